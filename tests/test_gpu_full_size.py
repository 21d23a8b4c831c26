"""Full-size parity (4B shapes, the launch configurations bench.py times).

The oracle cannot run the whole 4B workloads in seconds, so these tests
compare what it can compute one by one and check properties for the rest:
  * prefill 1 x 4096 at k = 2: by causality rows [0, m) of the prefill equal a
    prefill of the first m tokens (pinned in test_oracle_pins), so the first
    rows are compared with the oracle; every row must lie on the unit sphere;
  * decode of 64 sequences x 32768 cached positions at k = 2 (last-loop): one
    sampled sequence is recomputed by the oracle from the same counter-hash
    cache contents; every row must be finite and unit-norm.
"""

import numpy as np
import pytest
import torch

from tests.gpu_util import inputs, to_np, assert_parity, oracle, oracle_cache

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def big():
    from looped_ngpt_transformer_fwd_b200 import build as libbuild
    from looped_ngpt_transformer_fwd_b200.model import DoryModel
    from oracle import weights_from_generator
    from synthetic import load_config
    libbuild.build()
    cfg = load_config("dory4b")
    prov = weights_from_generator(cfg, 2, cache_blocks=True)
    model = DoryModel(cfg, prov)
    yield cfg, prov, model
    model.close()
    torch.cuda.empty_cache()


def test_4b_prefill_4096_k2_prefix_rows_and_unit_norm(big):
    cfg, prov, model = big
    T, k, m = 4096, 2, 4
    x, h = inputs(cfg, 41, T)
    kv = model.kv_cache("last_loop", 1, T, k_max=k)
    out = model.prefill(kv, x, k)
    torch.cuda.synchronize()
    assert model.device_status() == 0
    norms = out.float().norm(dim=1)
    assert torch.isfinite(out.float()).all()
    assert (norms - 1).abs().max().item() < 1e-2
    ref = oracle(cfg, prov).forward(h[:m], 0, k, oracle_cache(cfg, "last_loop", k_max=k))
    assert_parity(to_np(out[:m]), ref, what="4B prefill prefix rows")


def test_4b_decode_b64_ctx32768_sampled_sequence(big):
    import bench
    from oracle import KVCache
    from synthetic import block_weights
    from synthetic.kvfill import kv_values
    cfg, prov, model = big
    B, ctx, k, mode, seed = 64, 32768, 2, "last_loop", 2
    kv = model.kv_cache(mode, B, ctx + 64, k_max=k)
    bench.fill_decode_cache(model, kv, cfg, seed, ctx, mode, k, B)
    x, h = inputs(cfg, 42, B)
    d_seq = torch.arange(B, dtype=torch.int32, device="cuda")
    d_pos = torch.full((B,), ctx, dtype=torch.int32, device="cuda")
    out = model.decode(kv, x, d_seq, d_pos, ctx, k)
    torch.cuda.synchronize()
    assert model.device_status() == 0
    assert torch.isfinite(out.float()).all()
    assert (out.float().norm(dim=1) - 1).abs().max().item() < 1e-2
    s = 37
    s_qk = {b: block_weights(cfg, seed, b, names=("s_qk",))["s_qk"] for b in range(36)}

    def pre(slot, seq, lo, hi):
        return kv_values(seed, slot, seq, np.arange(lo, hi), cfg["n_kv_heads"], cfg["head_dim"],
                         s_qk[slot // 16])
    cache = KVCache(cfg, mode, k_max=k, prefill=pre, prefilled_len={s: ctx})
    ref = oracle(cfg, prov).decode(h[s:s + 1], [s], [ctx], k, cache)
    assert_parity(to_np(out[s:s + 1]), ref, what="4B decode sampled sequence")
    del kv
    torch.cuda.empty_cache()


@pytest.mark.parametrize("mode", ["per_loop", "last_loop"])
def test_4b_shape_stack_matches_oracle_at_every_row(mode):
    """The 4B block shapes (d_model 3072, 24 / 8 heads of 128, MLP 9216, window
    4096) with one input, one recurrent and one output block, k = 2, on 300
    tokens: every row against the oracle, with the fused projections on (an
    8-CTA cluster per row and a ragged last band, 300 = 2 x 128 + 44)."""
    from looped_ngpt_transformer_fwd_b200 import build as libbuild
    from looped_ngpt_transformer_fwd_b200.model import DoryModel
    from oracle import weights_from_generator
    from synthetic import load_config
    libbuild.build()
    cfg = load_config("dory4b", n_in_blocks=1, n_rec_blocks=1, n_out_blocks=1, full_period=2)
    prov = weights_from_generator(cfg, 11, "random")
    model = DoryModel(cfg, prov)
    assert model.fused_update(True)        # the 8-CTA cluster path at the 4B shape
    k = 2
    x, h = inputs(cfg, 43, 302)
    kv = model.kv_cache(mode, 1, 400, k_max=k)
    ocache = oracle_cache(cfg, mode, k_max=k)
    orc = oracle(cfg, prov)
    out = model.prefill(kv, x[:300], k)
    torch.cuda.synchronize()
    assert model.device_status() == 0
    assert_parity(to_np(out), orc.forward(h[:300], 0, k, ocache), what=f"4B-shape prefill {mode}")
    for p in (300, 301):
        d = torch.zeros(1, dtype=torch.int32, device="cuda")
        pp = torch.tensor([p], dtype=torch.int32, device="cuda")
        out = model.decode(kv, x[p:p + 1], d, pp, 399, k)
        ref = orc.decode(h[p:p + 1], [0], [p], k, ocache)
        assert_parity(to_np(out), ref, what=f"4B-shape decode {p} {mode}")
    model.close()


@pytest.mark.parametrize("fmt", ["mxfp8", "nvfp4"])
def test_4b_shape_block_scaled_stack_matches_oracle(fmt):
    """The 4B block shapes (d_model 3072, 24 / 8 heads of 128, MLP 9216) with one
    input, one recurrent and one output block, k = 2, MXFP8 or NVFP4 weights and
    projection inputs, 300 tokens then two decode steps: every row against the
    oracle of the same format (NVFP4 at its stack bar, cosine 0.998)."""
    from looped_ngpt_transformer_fwd_b200 import build as libbuild
    from looped_ngpt_transformer_fwd_b200.model import DoryModel
    from oracle import Oracle, weights_from_generator
    from oracle import quant as Q
    from synthetic import load_config
    libbuild.build()
    cfg = load_config("dory4b", n_in_blocks=1, n_rec_blocks=1, n_out_blocks=1, full_period=2)
    prov = weights_from_generator(cfg, 12, "random")
    model = DoryModel(cfg, prov, weight_format=fmt)
    orc = Oracle(cfg, Q.dequantized_provider(prov, fmt),
                 act_quant=Q.nvfp4_fake_quant if fmt == "nvfp4" else Q.mxfp8_fake_quant)
    tol_cos = 0.998 if fmt == "nvfp4" else 0.999
    k = 2
    x, h = inputs(cfg, 44, 302)
    kv = model.kv_cache("last_loop", 1, 400, k_max=k)
    ocache = oracle_cache(cfg, "last_loop", k_max=k)
    out = model.prefill(kv, x[:300], k)
    torch.cuda.synchronize()
    assert model.device_status() == 0
    assert_parity(to_np(out), orc.forward(h[:300], 0, k, ocache), tol_cos=tol_cos,
                  what=f"4B-shape {fmt} prefill")
    for p in (300, 301):
        d = torch.zeros(1, dtype=torch.int32, device="cuda")
        pp = torch.tensor([p], dtype=torch.int32, device="cuda")
        out = model.decode(kv, x[p:p + 1], d, pp, 399, k)
        ref = orc.decode(h[p:p + 1], [0], [p], k, ocache)
        assert_parity(to_np(out), ref, tol_cos=tol_cos, what=f"4B-shape {fmt} decode {p}")
    model.close()
