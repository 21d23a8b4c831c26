"""Backward of the MLP sublayer on the GPU against the float64 oracle.

Truncated depth-one back-propagation trains only the final recurrent
invocation ("Dory1.0-4B: A Looped Normalized-GPT", Methodology in Plain
English); dory_mlp_sublayer_backward is its MLP-sublayer step.  Checked:
  * the tcgen05 GEMM with operands read MN-major (the dgrad and wgrad
    products) against float64 matmuls, every transposed layout, ragged sizes;
  * every gradient (dh, dW_gate, dW_up, dW_down, dalpha) against
    oracle/backward.py on the tiny, head_dim-128 and 4B shapes;
  * an output gradient along h_out gives (nearly) zero gradients on the GPU
    too: the closed form the oracle is pinned by.
Bar (the forward is recomputed with the inference path's bf16 operands:
h, the SwiGLU activations and dL/dy are rounded to bf16, 2^-9 relative, before
their products): per gradient tensor, relative Frobenius error <= 2e-2 and
cosine (flattened) >= 0.9998.
"""

import numpy as np
import pytest
import torch

from oracle.backward import mlp_sublayer_backward
from tests.gpu_util import build, inputs, to_np

pytestmark = pytest.mark.gpu

REL_FRO, MIN_COS = 2e-2, 0.9998


@pytest.mark.parametrize("a_mn,b_mn", [(0, 1), (1, 0), (1, 1)])
@pytest.mark.parametrize("M,N,K", [(304, 384, 512), (3072, 1024, 200), (256, 256, 4096),
                                   (136, 1280, 1000)])
def test_gemm_with_transposed_operands(a_mn, b_mn, M, N, K):
    from looped_ngpt_transformer_fwd_b200 import build as libbuild
    from looped_ngpt_transformer_fwd_b200.model import gemm_bf16_mn
    libbuild.build()
    if (not a_mn or not b_mn) and K % 8:
        pytest.skip("a K-major operand needs 16-byte rows")
    g = torch.Generator(device="cuda").manual_seed(M + N + K)
    A = torch.randn(K, M, device="cuda", generator=g) if a_mn else torch.randn(M, K, device="cuda", generator=g)
    Bm = torch.randn(K, N, device="cuda", generator=g) if b_mn else torch.randn(N, K, device="cuda", generator=g)
    A, Bm = A.to(torch.bfloat16), Bm.to(torch.bfloat16)
    C = gemm_bf16_mn(A, Bm, M, N, K, a_mn, b_mn)
    torch.cuda.synchronize()
    An = A.double().cpu().numpy()
    Bn = Bm.double().cpu().numpy()
    ref = (An.T if a_mn else An) @ (Bn if b_mn else Bn.T)
    err = np.abs(C.double().cpu().numpy() - ref).max()
    assert err <= 1e-4 * np.abs(ref).max(), err


def _weights(prov, layer):
    from synthetic.bf16 import bf16_bits_to_f32
    raw = prov(layer)
    return {k: (bf16_bits_to_f32(v).astype(np.float64) if v.dtype == np.uint16
                else np.asarray(v, dtype=np.float64)) for k, v in raw.items()}


def _check(got, want, what):
    g, w = to_np(got).ravel(), np.asarray(want, np.float64).ravel()
    rel = np.linalg.norm(g - w) / np.linalg.norm(w)
    cos = float(g @ w / (np.linalg.norm(g) * np.linalg.norm(w)))
    assert rel <= REL_FRO and cos >= MIN_COS, f"{what}: rel {rel:.3e} cos {cos:.6f}"
    return rel, cos


def _run(cfg_name, seed, rows, layer, **over):
    cfg, prov, model = build(cfg_name, seed=seed, **over)
    _, h = inputs(cfg, seed + 1, rows)
    rng = np.random.default_rng(seed + 2)
    dh_out = rng.standard_normal(h.shape) * 0.1
    ht = torch.from_numpy(h.astype(np.float32)).cuda()
    gt = torch.from_numpy(dh_out.astype(np.float32)).cuda()
    out = model.mlp_sublayer_backward(layer, ht, gt)
    torch.cuda.synchronize()
    assert model.device_status() == 0
    ref = mlp_sublayer_backward(cfg, _weights(prov, layer), h, dh_out)
    res = {}
    for k, rk in (("dh", "dh"), ("d_w_gate", "d_w_gate"), ("d_w_up", "d_w_up"),
                  ("d_w_down", "d_w_down"), ("d_alpha", "d_alpha")):
        res[k] = _check(out[k], ref[rk], f"{cfg_name} {k}")
    model.close()
    return res


@pytest.mark.parametrize("rows,layer", [(200, 3), (64, 0), (1, 1)])
def test_mlp_backward_tiny(rows, layer):
    _run("tiny", 41, rows, layer)


def test_mlp_backward_head_dim_128_shapes():
    _run("tiny", 42, 300, 2, d_model=768, n_q_heads=6, n_kv_heads=2, head_dim=128, d_ff=1024,
         softmax_scale=float(np.sqrt(128.0)))


def test_mlp_backward_4b_shapes():
    """d_model 3072, d_ff 9216 (one block of each kind), 256 rows."""
    _run("dory4b", 43, 256, 1, n_in_blocks=1, n_rec_blocks=1, n_out_blocks=1)


def test_gradient_along_the_output_vanishes_on_the_gpu():
    """dL/dh_out = 3 h_out: the output is a unit vector, so every gradient is
    zero up to the bf16 rounding of the recomputed forward."""
    cfg, prov, model = build("tiny", seed=44)
    _, h = inputs(cfg, 45, 128)
    ht = torch.from_numpy(h.astype(np.float32)).cuda()
    h_out = ht.clone()
    model.mlp_sublayer(2, h_out)
    rng = np.random.default_rng(46)
    ref_scale = model.mlp_sublayer_backward(
        2, ht, torch.from_numpy((rng.standard_normal(h.shape) * 0.1).astype(np.float32)).cuda())
    along = model.mlp_sublayer_backward(2, ht, 3.0 * h_out)
    torch.cuda.synchronize()
    for k in ("dh", "d_w_gate", "d_w_up", "d_w_down"):
        typical = ref_scale[k].abs().max().item()
        assert along[k].abs().max().item() < 0.05 * typical, k
    model.close()


# ------------------------------------------------------------------ attention

def _run_attention(cfg_name, seed, rows, layer, **over):
    from oracle.backward import attention_sublayer_backward
    cfg, prov, model = build(cfg_name, seed=seed, **over)
    _, h = inputs(cfg, seed + 1, rows)
    dh_out = np.random.default_rng(seed + 2).standard_normal(h.shape) * 0.1
    ht = torch.from_numpy(h.astype(np.float32)).cuda()
    gt = torch.from_numpy(dh_out.astype(np.float32)).cuda()
    out = model.attention_sublayer_backward(layer, ht, gt)
    torch.cuda.synchronize()
    assert model.device_status() == 0
    ref = attention_sublayer_backward(cfg, _weights(prov, layer), h, dh_out, layer)
    for k in ("dh", "d_wq", "d_wk", "d_wv", "d_wg", "d_wo", "d_alpha", "d_s_qk"):
        _check(out[k], ref[k], f"{cfg_name} layer {layer} {k}")
    model.close()


@pytest.mark.parametrize("layer", [0, 1])        # sliding window (W = 32), full
@pytest.mark.parametrize("rows", [100, 7])
def test_attention_backward_tiny(layer, rows):
    _run_attention("tiny", 51, rows, layer)


@pytest.mark.parametrize("layer", [0, 1])        # W = 128, full; GQA group 3
def test_attention_backward_head_dim_128(layer):
    _run_attention("tiny", 52, 300, layer, d_model=768, n_q_heads=6, n_kv_heads=2, head_dim=128,
                   d_ff=1024, window=128, softmax_scale=float(np.sqrt(128.0)))


def test_attention_backward_4b_shapes():
    """d_model 3072, 24 / 8 heads of 128, window 4096 (full causal at 256 rows)."""
    _run_attention("dory4b", 53, 256, 1, n_in_blocks=1, n_rec_blocks=1, n_out_blocks=1)


def test_attention_gradient_along_the_output_vanishes_on_the_gpu():
    cfg, prov, model = build("tiny", seed=54)
    _, h = inputs(cfg, 55, 64)
    ht = torch.from_numpy(h.astype(np.float32)).cuda()
    kv = model.kv_cache("last_loop", 1, 64)
    h_out = ht.clone()
    model.attention_sublayer(kv, 1, h_out, loop=1, seq=0, pos0=0)
    rng = np.random.default_rng(56)
    typical = model.attention_sublayer_backward(
        1, ht, torch.from_numpy((rng.standard_normal(h.shape) * 0.1).astype(np.float32)).cuda())
    along = model.attention_sublayer_backward(1, ht, -2.0 * h_out)
    torch.cuda.synchronize()
    for k in ("dh", "d_wq", "d_wk", "d_wv", "d_wg", "d_wo"):
        assert along[k].abs().max().item() < 0.05 * typical[k].abs().max().item(), k
    model.close()


# ------------------------------------------------------------------ the stack

# Bar for the whole truncated backward: the rounding of every sublayer's
# recomputed forward and backward operands to bf16 adds up along the chain
# (12 sublayers for the tiny stack), so it could exceed one sublayer's error;
# measured it stays at the sublayer level (worst tensor 8.3e-3 relative,
# cosine 0.99997; dL/dx_k 1.4e-3), and the chain keeps the sublayer bar.
CHAIN_REL, CHAIN_COS = REL_FRO, MIN_COS


@pytest.mark.parametrize("k", [1, 2, 3])
def test_last_loop_backward_matches_the_oracle(k):
    from oracle.backward import last_loop_backward
    from tests.gpu_util import assert_parity
    cfg, prov, model = build("tiny", seed=61)
    _, h = inputs(cfg, 62, 64)
    dh_out = np.random.default_rng(63).standard_normal(h.shape) * 0.1
    kv = model.kv_cache("last_loop", 1, 64)
    res = model.last_loop_backward(kv, torch.from_numpy(h.astype(np.float32)).cuda(),
                                   torch.from_numpy(dh_out.astype(np.float32)).cuda(), k)
    torch.cuda.synchronize()
    assert model.device_status() == 0
    ref = last_loop_backward(cfg, prov, h, dh_out, k)
    assert_parity(to_np(res["h_out"]), ref["h_out"], what=f"training forward k={k}")
    worst = (0.0, 1.0)
    for b, gb in ref["grads"].items():
        for name, want in gb.items():
            g, w = to_np(res["grads"][b][name]).ravel(), np.asarray(want).ravel()
            rel = np.linalg.norm(g - w) / np.linalg.norm(w)
            cos = float(g @ w / (np.linalg.norm(g) * np.linalg.norm(w)))
            worst = (max(worst[0], rel), min(worst[1], cos))
            assert rel <= CHAIN_REL and cos >= CHAIN_COS, f"block {b} {name}: rel {rel:.3e} cos {cos:.6f}"
    g, w = to_np(res["dx"]).ravel(), ref["dx"].ravel()
    assert np.linalg.norm(g - w) / np.linalg.norm(w) <= CHAIN_REL
    model.close()


# ------------------------------------------------------------------ contracts

def test_backward_is_deterministic():
    """Two identical calls give bit-identical gradients: the dalpha and ds_qk
    sums run in a fixed order, and the concurrent KV heads write disjoint
    rows."""
    cfg, prov, model = build("tiny", seed=71, d_model=768, n_q_heads=6, n_kv_heads=2, head_dim=128,
                             d_ff=1024, window=128, softmax_scale=float(np.sqrt(128.0)))
    _, h = inputs(cfg, 72, 300)
    ht = torch.from_numpy(h.astype(np.float32)).cuda()
    gt = torch.from_numpy((np.random.default_rng(73).standard_normal(h.shape) * 0.1)
                          .astype(np.float32)).cuda()
    a1 = model.attention_sublayer_backward(0, ht, gt)
    a2 = model.attention_sublayer_backward(0, ht, gt)
    m1 = model.mlp_sublayer_backward(1, ht, gt)
    m2 = model.mlp_sublayer_backward(1, ht, gt)
    torch.cuda.synchronize()
    for k in a1:
        assert torch.equal(a1[k], a2[k]), k
    for k in m1:
        assert torch.equal(m1[k], m2[k]), k
    model.close()


def test_backward_refuses_what_it_does_not_cover():
    """Block-scaled weights have no backward (BAD_CONFIG), and a per-loop cache
    with fewer loop slots than k is refused (K_EXCEEDS_KMAX)."""
    from looped_ngpt_transformer_fwd_b200.binding import DoryError
    from looped_ngpt_transformer_fwd_b200.model import DoryModel
    from oracle import weights_from_generator
    from synthetic import load_config
    cfg = load_config("tiny")
    prov = weights_from_generator(cfg, 74, "random")
    mx = DoryModel(cfg, prov, weight_format="mxfp8")
    _, h = inputs(cfg, 75, 32)
    ht = torch.from_numpy(h.astype(np.float32)).cuda()
    with pytest.raises(DoryError, match="BAD_CONFIG"):
        mx.mlp_sublayer_backward(1, ht, ht.clone())
    with pytest.raises(DoryError, match="BAD_CONFIG"):
        mx.attention_sublayer_backward(1, ht, ht.clone())
    mx.close()
    model = DoryModel(cfg, prov)
    kv = model.kv_cache("per_loop", 1, 32, k_max=1)
    with pytest.raises(DoryError, match="K_EXCEEDS_KMAX"):
        model.last_loop_backward(kv, ht, ht.clone(), 2)
    model.close()
