"""MXFP8 weights and projection inputs on the block-scaled tensor cores.

The released MXFP8 checkpoint ("Dory1.0-4B: A Looped Normalized-GPT", Key
Contributions item 4; MXFP8 by standard post-training quantisation,
Methodology in Plain English) is served with both operands of every
projection in MXFP8 (E4M3 elements, one E8M0 scale per 32 along K), products on
tcgen05.mma kind::mxf8f6f4.  Checked against oracle/quant.py:
  * the quantiser's codes and scales bit for bit (same bf16 inputs, the same
    rounding decision on both sides);
  * the block-scaled GEMM against the float64 product of the decoded
    operands, with ragged M and N and K splits;
  * sublayers and whole stacks (tiny: head_dim 64; head_dim 128: tcgen05
    attention) against the oracle with MXFP8 weights and MXFP8 projection
    inputs, at the same bars as the bf16 path.
"""

import numpy as np
import pytest
import torch

from oracle import Oracle
from oracle import quant as Q
from tests.gpu_util import build, inputs, to_np, assert_parity, oracle_cache

pytestmark = pytest.mark.gpu


def _rows(M, K, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    x = torch.randn(M, K, device="cuda", generator=g)
    # magnitudes spread over blocks, an all-zero block and a tiny block
    x = x * torch.exp2(torch.randint(-8, 8, (M, K // 32), device="cuda", generator=g)
                       .repeat_interleave(32, dim=1).float())
    x[0, :32] = 0
    x[min(1, M - 1), 32:64] *= 1e-30
    return x.to(torch.bfloat16)


def _unchunk(scales, rows, K):
    """Scale codes [rows, K/32] from the chunked layout (dory_quant_mxfp8)."""
    rb = (rows + 127) // 128
    ch = scales.reshape(K // 128, rb, 32, 4, 4)        # kc, rb, i, j, q
    s = ch.transpose(1, 3, 2, 0, 4).reshape(rb * 128, K // 32)   # row = rb*128 + 32 j + i
    return s[:rows], s[rows:]


# (3, 24576) and (3, 81920): rows too long for the CTA-per-row kernel's
# registers at 1024 threads go to the warp-per-row kernel (the second)
@pytest.mark.parametrize("M,K", [(300, 384), (1, 128), (128, 3072), (77, 9216), (3, 24576),
                                 (3, 81920)])
def test_quantiser_codes_and_scales_are_bit_exact(M, K):
    from looped_ngpt_transformer_fwd_b200 import build as libbuild
    from looped_ngpt_transformer_fwd_b200.model import quant_mxfp8
    libbuild.build()
    x = _rows(M, K, M + K)
    codes, scales = quant_mxfp8(x)
    torch.cuda.synchronize()
    want_c, want_s = Q.mxfp8_quantize(x.float().cpu().numpy().astype(np.float64))
    got_s, pad = _unchunk(scales.cpu().numpy(), M, K)
    assert np.array_equal(codes.cpu().numpy(), want_c)
    assert np.array_equal(got_s, want_s)
    assert np.all(pad == 127)


@pytest.mark.parametrize("M,N,K,splits", [(300, 512, 384, 1), (64, 384, 3072, 4), (1, 128, 128, 1),
                                          (129, 1286, 256, 1), (1000, 768, 1024, 2),
                                          (700, 1024, 3072, 1), (64, 2048, 1024, 3)])
# (N a multiple of 256: 256-column tiles with one accumulator; else 128-column tiles)
def test_block_scaled_gemm_matches_decoded_product(M, N, K, splits):
    from looped_ngpt_transformer_fwd_b200 import build as libbuild
    from looped_ngpt_transformer_fwd_b200.model import gemm_mxfp8
    libbuild.build()
    A = _rows(M, K, 3 * M + N)
    Bm = (torch.randn(N, K, device="cuda", generator=torch.Generator(device="cuda").manual_seed(N))
          * 0.02).to(torch.bfloat16)
    C = gemm_mxfp8(A, Bm, splits).double().sum(0).cpu().numpy()
    ref = Q.mxfp8_gemm(A.float().cpu().numpy(), Bm.float().cpu().numpy())
    err = np.abs(C - ref).max()
    assert err <= 1e-5 * np.abs(ref).max() + 1e-6, err
    # negative control: the bf16 product differs by the quantisation error
    exact = A.double().cpu().numpy() @ Bm.double().cpu().numpy().T
    assert np.abs(exact - ref).max() > 100 * err


def _mx_oracle(cfg, prov):
    return Oracle(cfg, Q.dequantized_provider(prov, "mxfp8"), act_quant=Q.mxfp8_fake_quant)


def _mx_model(cfg_name="tiny", seed=0, **over):
    from looped_ngpt_transformer_fwd_b200 import build as libbuild
    from looped_ngpt_transformer_fwd_b200.model import DoryModel
    from oracle import weights_from_generator
    from synthetic import load_config
    libbuild.build()
    cfg = load_config(cfg_name, **over)
    prov = weights_from_generator(cfg, seed, "random")
    return cfg, prov, DoryModel(cfg, prov, weight_format="mxfp8")


@pytest.fixture(scope="module")
def tiny_mx():
    return _mx_model("tiny", 21)


def test_mlp_sublayer_mxfp8(tiny_mx):
    cfg, prov, model = tiny_mx
    _, h = inputs(cfg, 81, 200)
    ht = torch.from_numpy(h.astype(np.float32)).cuda()
    model.mlp_sublayer(3, ht)
    torch.cuda.synchronize()
    assert model.device_status() == 0
    ref = _mx_oracle(cfg, prov).mlp_sublayer(3, h)
    assert_parity(to_np(ht), ref, tol_abs=5e-3, tol_cos=0.9999, what="MXFP8 MLP sublayer")


@pytest.mark.parametrize("layer", [0, 1])
def test_attention_sublayer_mxfp8(tiny_mx, layer):
    cfg, prov, model = tiny_mx
    _, h = inputs(cfg, 82, 150)
    kv = model.kv_cache("last_loop", 1, 160)
    ht = torch.from_numpy(h.astype(np.float32)).cuda()
    model.attention_sublayer(kv, layer, ht)
    torch.cuda.synchronize()
    ref = _mx_oracle(cfg, prov).attention_sublayer(layer, h, 0, 0, 1, oracle_cache(cfg, "last_loop"))
    assert_parity(to_np(ht), ref, tol_abs=5e-3, tol_cos=0.9999, what=f"MXFP8 attention {layer}")


@pytest.mark.parametrize("mode", ["per_loop", "last_loop"])
def test_stack_mxfp8_prefill_chunks_and_decode(tiny_mx, mode):
    cfg, prov, model = tiny_mx
    k = 2
    x, h = inputs(cfg, 83, 100)
    kv = model.kv_cache(mode, 1, 128, k_max=k)
    ocache = oracle_cache(cfg, mode, k_max=k)
    orc = _mx_oracle(cfg, prov)
    for a, b in ((0, 64), (64, 96)):
        out = model.prefill(kv, x[a:b], k, pos0=a)
        torch.cuda.synchronize()
        assert_parity(to_np(out), orc.forward(h[a:b], a, k, ocache), what=f"MXFP8 chunk {a} {mode}")
    for p in (96, 97, 98):
        d = torch.zeros(1, dtype=torch.int32, device="cuda")
        pp = torch.tensor([p], dtype=torch.int32, device="cuda")
        out = model.decode(kv, x[p:p + 1], d, pp, 127, k)
        assert_parity(to_np(out), orc.decode(h[p:p + 1], [0], [p], k, ocache),
                      what=f"MXFP8 decode {p} {mode}")
    assert model.device_status() == 0


def test_stack_mxfp8_head_dim_128_and_gqa3():
    """d_model 768, 6 / 2 heads of 128 (tcgen05 attention, the 4B head grouping),
    MXFP8 at k = 4: prefill of 300 tokens, then a decode batch."""
    cfg, prov, model = _mx_model("tiny", 22, d_model=768, n_q_heads=6, n_kv_heads=2, head_dim=128,
                                 d_ff=1024, window=128, softmax_scale=float(np.sqrt(128.0)))
    k = 4
    x, h = inputs(cfg, 84, 302)
    kv = model.kv_cache("last_loop", 1, 320, k_max=k)
    ocache = oracle_cache(cfg, "last_loop", k_max=k)
    orc = _mx_oracle(cfg, prov)
    out = model.prefill(kv, x[:300], k)
    torch.cuda.synchronize()
    assert model.attention_paths()["prefill_tc"] > 0
    assert_parity(to_np(out), orc.forward(h[:300], 0, k, ocache), what="MXFP8 hd128 prefill")
    for p in (300, 301):
        d = torch.zeros(1, dtype=torch.int32, device="cuda")
        pp = torch.tensor([p], dtype=torch.int32, device="cuda")
        out = model.decode(kv, x[p:p + 1], d, pp, 319, k)
        assert_parity(to_np(out), orc.decode(h[p:p + 1], [0], [p], k, ocache),
                      what=f"MXFP8 hd128 decode {p}")
    assert model.device_status() == 0
    model.close()


def test_mxfp8_tracks_the_bf16_model(tiny_mx):
    """Negative control of the oracle comparison: the MXFP8 model is close to the
    bf16 oracle but measurably different from it (the quantisation is live)."""
    cfg, prov, model = tiny_mx
    x, h = inputs(cfg, 85, 64)
    kv = model.kv_cache("last_loop", 1, 64, k_max=2)
    out = to_np(model.prefill(kv, x, 2))
    bf = Oracle(cfg, prov).forward(h, 0, 2, oracle_cache(cfg, "last_loop", k_max=2))
    mx = _mx_oracle(cfg, prov).forward(h, 0, 2, oracle_cache(cfg, "last_loop", k_max=2))
    assert np.abs(out - mx).max() < np.abs(out - bf).max()
