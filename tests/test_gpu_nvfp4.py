"""NVFP4 weights and projection inputs on the block-scaled tensor cores.

The released NVFP4 checkpoint ("Dory1.0-4B: A Looped Normalized-GPT", Key
Contributions item 4; Main Findings: NVFP4 after quantisation-aware
distillation) is served with both operands of every projection in NVFP4 (E2M1
elements, one E4M3 scale per 16 along K, an fp32 tensor scale), products on
tcgen05.mma kind::mxf4nvf4.  Checked against oracle/quant.py:
  * the quantiser's codes, block scales and tensor scale bit for bit, exact
    ties included;
  * the block-scaled GEMM against the float64 product of the decoded
    operands, with ragged M and N and K splits;
  * sublayers and whole stacks (tiny: head_dim 64; head_dim 128 with the 4B
    head grouping: tcgen05 attention) against the oracle with NVFP4 weights
    and NVFP4 projection inputs.
"""

import numpy as np
import pytest
import torch

from oracle import Oracle
from oracle import quant as Q
from tests.gpu_util import inputs, to_np, assert_parity, oracle_cache

pytestmark = pytest.mark.gpu

# Stack bar for NVFP4.  The GPU stores the attention output and the SwiGLU
# activations in bf16 (relative rounding up to 2^-9) before quantising them,
# the oracle keeps float64; E2M1 has one mantissa bit, so its decision points
# are 25-50 % apart, and an element whose bf16 value lands on the other side
# of one moves by a whole grid step (a third to a half of its value).  Such
# flips hit about one element in a few hundred per projection input and add up
# over the stack's sublayers: the per-token cosine bar is 0.998 (0.999 for the
# bf16 and MXFP8 paths, whose grids are 8x finer); max |diff| keeps 3e-2.
NV_TOL_COS = 0.998


def _lib():
    from looped_ngpt_transformer_fwd_b200 import build as libbuild
    libbuild.build()


def _rows(M, K, seed, unit=True):
    g = torch.Generator(device="cuda").manual_seed(seed)
    x = torch.randn(M, K, device="cuda", generator=g)
    # magnitudes spread over blocks, an all-zero block and a tiny block
    x = x * torch.exp2(torch.randint(-6, 3, (M, K // 16), device="cuda", generator=g)
                       .repeat_interleave(16, dim=1).float())
    x[0, :16] = 0
    x[min(1, M - 1), 16:32] *= 1e-6
    if unit:
        x = x / x.norm(dim=1, keepdim=True).clamp_min(1e-30)
    return x.to(torch.bfloat16)


def _unpack(codes):
    """[rows, K/2] packed bytes -> [rows, K] codes (element 2i in the low nibble)."""
    c = codes.astype(np.uint8)
    out = np.empty((c.shape[0], 2 * c.shape[1]), dtype=np.uint8)
    out[:, 0::2] = c & 0xF
    out[:, 1::2] = c >> 4
    return out


def _unchunk(scales, rows, K):
    """Scale codes [rows, K/16] from the chunked layout (dory_quant_nvfp4)."""
    rb = (rows + 127) // 128
    ch = scales.reshape(K // 256, rb, 4, 32, 4, 4)           # kc, rb, piece, i, j, q
    s = ch.transpose(1, 4, 3, 0, 2, 5).reshape(rb * 128, K // 16)
    return s[:rows], s[rows:]


# K up to 20480 (bf16): the block-per-thread kernel; (3, 24576): the
# CTA-per-row kernel with lane pairs per block; (3, 81920): the warp-per-row one
@pytest.mark.parametrize("M,K", [(300, 512), (1, 256), (128, 3072), (77, 9216), (3, 24576),
                                 (3, 81920)])
def test_quantiser_is_bit_exact_with_the_input_scale(M, K):
    from looped_ngpt_transformer_fwd_b200.model import quant_nvfp4
    _lib()
    x = _rows(M, K, M + K)
    codes, scales, d_g = quant_nvfp4(x, g=float(Q.NVFP4_ACT_G))
    torch.cuda.synchronize()
    want_c, want_s, _ = Q.nvfp4_quantize(x.float().cpu().numpy().astype(np.float64), Q.NVFP4_ACT_G)
    got_s, pad = _unchunk(scales.cpu().numpy(), M, K)
    assert np.array_equal(_unpack(codes.cpu().numpy()), want_c)
    assert np.array_equal(got_s, want_s)
    assert np.all(pad == 0x38)


@pytest.mark.parametrize("M,K", [(200, 768), (3072, 256)])
def test_quantiser_tensor_scale_from_the_data(M, K):
    """g = amax / (6 * 448) computed on the device equals the oracle's bit for
    bit, and so do the codes under it (weights: rows not unit vectors)."""
    from looped_ngpt_transformer_fwd_b200.model import quant_nvfp4
    _lib()
    x = (_rows(M, K, 7 * M + K, unit=False).float() * 0.03).to(torch.bfloat16)
    codes, scales, d_g = quant_nvfp4(x)
    torch.cuda.synchronize()
    xn = x.float().cpu().numpy().astype(np.float64)
    want_c, want_s, want_g = Q.nvfp4_quantize(xn)
    assert np.float32(d_g.item()) == want_g
    assert np.array_equal(_unpack(codes.cpu().numpy()), want_c)
    assert np.array_equal(_unchunk(scales.cpu().numpy(), M, K)[0], want_s)


def test_quantiser_exact_ties_round_to_even():
    """Inputs exactly halfway between E2M1 grid points (tensor scale 2^-12,
    block scale 1.5: every value exact in bf16) round like the oracle's."""
    from looped_ngpt_transformer_fwd_b200.model import quant_nvfp4
    _lib()
    g = 2.0 ** -12
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    blk = np.concatenate([[6.0], mids, -mids, [0.0]]) * 1.5 * g
    rows = np.stack([blk * 2.0 ** -e for e in range(8)])        # other block scales too
    x = np.tile(rows, (1, 16))                                  # K = 256
    xt = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).cuda()
    assert np.array_equal(xt.float().cpu().numpy(), x)
    codes, scales, _ = quant_nvfp4(xt, g=g)
    torch.cuda.synchronize()
    want_c, want_s, _ = Q.nvfp4_quantize(x, np.float32(g))
    assert np.array_equal(_unpack(codes.cpu().numpy()), want_c)
    assert np.array_equal(_unchunk(scales.cpu().numpy(), 8, 256)[0], want_s)


def test_quantiser_block_scale_ties_saturation_and_subnormals():
    """Blocks whose quotient amax / (6 g) lies exactly on an E4M3 midpoint
    (normal and subnormal, one carrying into the next binade), on the
    saturation point 448 and above it, and just beside such points; each
    block also holds the E2M1 midpoints of its own decoded scale.  The
    kernels decide most values from a bracketed fp32 quotient and hand these
    ones to the exact comparisons: codes and scales equal the oracle's."""
    from looped_ngpt_transformer_fwd_b200.model import quant_nvfp4
    _lib()
    g = 2.0 ** -12
    qs = [1.0625, 1.9375, 248.0, 432.0, 448.0, 456.0, 464.0, 1024.0,
          2.0 ** -10, 1.5 * 2.0 ** -9, 15 * 2.0 ** -10, 2.5 * 2.0 ** -9,
          1.0, 17.0, 0.3125, 96.0]
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    rng = np.random.default_rng(11)
    rows, K = 24, 512
    x = np.zeros((rows, K))
    for r in range(rows):
        for b in range(K // 16):
            q = qs[(b + 5 * r) % len(qs)] * (1.0 + 2.0 ** -7 * ((r // 8) - 1))   # on, below, above
            amax = 6.0 * g * q
            x[r, 16 * b:16 * b + 16] = rng.uniform(-amax, amax, 16)
            x[r, 16 * b + rng.integers(16)] = amax * rng.choice([-1.0, 1.0])
    x = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).float().numpy().astype(np.float64)
    # E2M1 midpoints of each block's scale (those not above the block's amax)
    _, s_codes, _ = Q.nvfp4_quantize(x, np.float32(g))
    s = Q.decode(s_codes, Q.E4M3)
    for r in range(rows):
        for b in range(K // 16):
            blk = x[r, 16 * b:16 * b + 16]
            amax = np.abs(blk).max()
            j = int(np.argmax(np.abs(blk)))
            free = [i for i in range(16) if i != j]
            for i, m in zip(free, mids):
                v = m * s[r, b] * g * (-1.0) ** i
                if 0.0 < abs(v) <= amax:
                    blk[i] = v
    xt = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).cuda()
    assert np.array_equal(xt.float().cpu().numpy(), x)
    codes, scales, _ = quant_nvfp4(xt, g=g)
    torch.cuda.synchronize()
    want_c, want_s, _ = Q.nvfp4_quantize(x, np.float32(g))
    assert np.array_equal(_unchunk(scales.cpu().numpy(), rows, K)[0], want_s)
    assert np.array_equal(_unpack(codes.cpu().numpy()), want_c)


@pytest.mark.parametrize("M,N,K,splits", [(300, 512, 512, 1), (64, 384, 3072, 4), (1, 128, 256, 1),
                                          (129, 1286, 256, 1), (1000, 768, 1024, 2),
                                          (700, 1024, 3072, 1), (64, 2048, 1536, 3)])
# (N a multiple of 256: 256-column tiles with one accumulator; else 128-column tiles;
# every K split owns at least one 256-K step)
def test_block_scaled_gemm_matches_decoded_product(M, N, K, splits):
    from looped_ngpt_transformer_fwd_b200.model import gemm_nvfp4
    _lib()
    A = _rows(M, K, 3 * M + N)
    Bm = (torch.randn(N, K, device="cuda", generator=torch.Generator(device="cuda").manual_seed(N))
          * 0.02).to(torch.bfloat16)
    An, Bn = A.float().cpu().numpy().astype(np.float64), Bm.float().cpu().numpy().astype(np.float64)
    g_a, g_b = Q.NVFP4_ACT_G, Q.nvfp4_tensor_scale(Bn)
    C = gemm_nvfp4(A, Bm, g_a, g_b, splits).double().sum(0).cpu().numpy()
    ref = Q.nvfp4_gemm(An, Bn, g_a, g_b)
    err = np.abs(C - ref).max()
    assert err <= 1e-5 * np.abs(ref).max() + 1e-7, err
    # negative control: the bf16 product differs by the quantisation error
    exact = An @ Bn.T
    assert np.abs(exact - ref).max() > 100 * err


def _nv_oracle(cfg, prov):
    return Oracle(cfg, Q.dequantized_provider(prov, "nvfp4"), act_quant=Q.nvfp4_fake_quant)


def _nv_model(cfg_name="tiny", seed=0, **over):
    from looped_ngpt_transformer_fwd_b200.model import DoryModel
    from oracle import weights_from_generator
    from synthetic import load_config
    _lib()
    cfg = load_config(cfg_name, **over)
    prov = weights_from_generator(cfg, seed, "random")
    return cfg, prov, DoryModel(cfg, prov, weight_format="nvfp4")


@pytest.fixture(scope="module")
def tiny_nv():
    return _nv_model("tiny", 31)


def test_mlp_sublayer_nvfp4(tiny_nv):
    cfg, prov, model = tiny_nv
    _, h = inputs(cfg, 91, 200)
    ht = torch.from_numpy(h.astype(np.float32)).cuda()
    model.mlp_sublayer(3, ht)
    torch.cuda.synchronize()
    assert model.device_status() == 0
    ref = _nv_oracle(cfg, prov).mlp_sublayer(3, h)
    assert_parity(to_np(ht), ref, tol_abs=5e-3, tol_cos=0.9999, what="NVFP4 MLP sublayer")


@pytest.mark.parametrize("layer", [0, 1])
def test_attention_sublayer_nvfp4(tiny_nv, layer):
    cfg, prov, model = tiny_nv
    _, h = inputs(cfg, 92, 150)
    kv = model.kv_cache("last_loop", 1, 160)
    ht = torch.from_numpy(h.astype(np.float32)).cuda()
    model.attention_sublayer(kv, layer, ht)
    torch.cuda.synchronize()
    ref = _nv_oracle(cfg, prov).attention_sublayer(layer, h, 0, 0, 1, oracle_cache(cfg, "last_loop"))
    assert_parity(to_np(ht), ref, tol_abs=5e-3, tol_cos=0.9999, what=f"NVFP4 attention {layer}")


@pytest.mark.parametrize("mode", ["per_loop", "last_loop"])
def test_stack_nvfp4_prefill_chunks_and_decode(tiny_nv, mode):
    cfg, prov, model = tiny_nv
    k = 2
    x, h = inputs(cfg, 93, 100)
    kv = model.kv_cache(mode, 1, 128, k_max=k)
    ocache = oracle_cache(cfg, mode, k_max=k)
    orc = _nv_oracle(cfg, prov)
    for a, b in ((0, 64), (64, 96)):
        out = model.prefill(kv, x[a:b], k, pos0=a)
        torch.cuda.synchronize()
        assert_parity(to_np(out), orc.forward(h[a:b], a, k, ocache), tol_cos=NV_TOL_COS,
                      what=f"NVFP4 chunk {a} {mode}")
    for p in (96, 97, 98):
        d = torch.zeros(1, dtype=torch.int32, device="cuda")
        pp = torch.tensor([p], dtype=torch.int32, device="cuda")
        out = model.decode(kv, x[p:p + 1], d, pp, 127, k)
        assert_parity(to_np(out), orc.decode(h[p:p + 1], [0], [p], k, ocache),
                      tol_cos=NV_TOL_COS, what=f"NVFP4 decode {p} {mode}")
    assert model.device_status() == 0


def test_stack_nvfp4_head_dim_128_and_gqa3():
    """d_model 768, 6 / 2 heads of 128 (tcgen05 attention, the 4B head grouping),
    NVFP4 at k = 4: prefill of 300 tokens, then decode steps."""
    cfg, prov, model = _nv_model("tiny", 32, d_model=768, n_q_heads=6, n_kv_heads=2, head_dim=128,
                                 d_ff=1024, window=128, softmax_scale=float(np.sqrt(128.0)))
    k = 4
    x, h = inputs(cfg, 94, 302)
    kv = model.kv_cache("last_loop", 1, 320, k_max=k)
    ocache = oracle_cache(cfg, "last_loop", k_max=k)
    orc = _nv_oracle(cfg, prov)
    out = model.prefill(kv, x[:300], k)
    torch.cuda.synchronize()
    assert model.attention_paths()["prefill_tc"] > 0
    assert_parity(to_np(out), orc.forward(h[:300], 0, k, ocache), tol_cos=NV_TOL_COS,
                  what="NVFP4 hd128 prefill")
    for p in (300, 301):
        d = torch.zeros(1, dtype=torch.int32, device="cuda")
        pp = torch.tensor([p], dtype=torch.int32, device="cuda")
        out = model.decode(kv, x[p:p + 1], d, pp, 319, k)
        assert_parity(to_np(out), orc.decode(h[p:p + 1], [0], [p], k, ocache),
                      tol_cos=NV_TOL_COS, what=f"NVFP4 hd128 decode {p}")
    assert model.device_status() == 0
    model.close()


def test_nvfp4_tracks_the_bf16_model(tiny_nv):
    """Negative control: the NVFP4 model is closer to the NVFP4 oracle than to
    the bf16 one (the quantisation is live)."""
    cfg, prov, model = tiny_nv
    x, h = inputs(cfg, 95, 64)
    kv = model.kv_cache("last_loop", 1, 64, k_max=2)
    out = to_np(model.prefill(kv, x, 2))
    bf = Oracle(cfg, prov).forward(h, 0, 2, oracle_cache(cfg, "last_loop", k_max=2))
    nv = _nv_oracle(cfg, prov).forward(h, 0, 2, oracle_cache(cfg, "last_loop", k_max=2))
    assert np.abs(out - nv).max() < np.abs(out - bf).max()


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp8"])
def test_mixed_k_decode_block_scaled(fmt):
    """A decode step with its own loop count per sequence on block-scaled
    weights: rows whose loops are done are skipped by the row kernel, so the
    stream's codes come from the stand-alone quantiser; each row equals that
    sequence decoded alone with its k by the oracle of the same format."""
    from looped_ngpt_transformer_fwd_b200.model import DoryModel
    from oracle import weights_from_generator
    from synthetic import load_config
    _lib()
    cfg = load_config("tiny")
    prov = weights_from_generator(cfg, 33, "random")
    model = DoryModel(cfg, prov, weight_format=fmt)
    orc = Oracle(cfg, Q.dequantized_provider(prov, fmt),
                 act_quant=Q.nvfp4_fake_quant if fmt == "nvfp4" else Q.mxfp8_fake_quant)
    ks = [1, 3, 2]
    k_hi = max(ks)
    kv = model.kv_cache("last_loop", 3, 96, k_max=k_hi)
    ocache = oracle_cache(cfg, "last_loop", k_max=k_hi)
    lens = [9, 40, 3]
    xs = [inputs(cfg, 80 + s, lens[s] + 1) for s in range(3)]
    for s, L in enumerate(lens):
        model.prefill(kv, xs[s][0][:L], ks[s], seq=s, pos0=0)
        orc.forward(xs[s][1][:L], 0, ks[s], ocache, seq=s)
    order = [1, 2, 0]
    rows_t = torch.cat([xs[s][0][lens[s]:lens[s] + 1] for s in order])
    d_seq = torch.tensor(order, dtype=torch.int32, device="cuda")
    d_pos = torch.tensor([lens[s] for s in order], dtype=torch.int32, device="cuda")
    d_k = torch.tensor([ks[s] for s in order], dtype=torch.int32, device="cuda")
    out = to_np(model.decode_mixed(kv, rows_t, d_seq, d_pos, d_k, 95, k_hi))
    torch.cuda.synchronize()
    assert model.device_status() == 0
    for i, s in enumerate(order):
        ref = orc.decode(xs[s][1][lens[s]:lens[s] + 1], [s], [lens[s]], ks[s], ocache)
        assert_parity(out[i:i + 1], ref, tol_cos=NV_TOL_COS, what=f"{fmt} mixed-k seq {s} k={ks[s]}")
    model.close()
