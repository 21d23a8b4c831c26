"""GPU parity: the sm_100a library (through its C ABI) against the float64 oracle
on the same seeded inputs (tiny config: several tiles, ragged tails, ring wraps)."""

import numpy as np
import pytest
import torch

from tests.gpu_util import (build, inputs, to_np, assert_parity, oracle, oracle_cache, metrics)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny():
    return build("tiny", seed=0, variant="random")


# ------------------------------------------------------------------ GEMM
@pytest.mark.parametrize("M,N,K", [(300, 512, 384), (64, 384, 3072), (1, 128, 64), (1000, 768, 256),
                                   (129, 256, 128)])
def test_gemm_matches_fp64(M, N, K):
    from looped_ngpt_transformer_fwd_b200 import build as libbuild
    from looped_ngpt_transformer_fwd_b200.model import gemm_bf16
    libbuild.build()
    g = torch.Generator(device="cuda").manual_seed(M * 7 + N)
    A = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
    Bm = torch.randn(N, K, device="cuda", generator=g).to(torch.bfloat16)
    C = gemm_bf16(A, Bm)
    torch.cuda.synchronize()
    ref = (A.double() @ Bm.double().T)
    err = (C.double() - ref).abs().max().item()
    assert err <= 1e-4 * ref.abs().max().item() + 1e-4, err


# ------------------------------------------------------------------ sublayers
def test_d_model_4096_mlp_sublayer_matches_oracle():
    """d_model 4096 (32 heads of 128, the widest the library takes): the row
    update's wide forms -- the pipelined kernel for 200 rows and the
    512-thread one-row kernel for 100 -- against the oracle."""
    cfg, prov, model = build("tiny", seed=3, d_model=4096, n_q_heads=32, n_kv_heads=8,
                             head_dim=128, d_ff=512, n_in_blocks=1, n_rec_blocks=1,
                             n_out_blocks=1, window=64)
    for n in (200, 100):
        _, h = inputs(cfg, 21 + n, n)
        ht = torch.from_numpy(h.astype(np.float32)).cuda()
        model.mlp_sublayer(0, ht)
        torch.cuda.synchronize()
        assert model.device_status() == 0
        ref = oracle(cfg, prov).mlp_sublayer(0, h)
        assert_parity(to_np(ht), ref, tol_abs=5e-3, tol_cos=0.9999, what=f"mlp d4096 rows {n}")
    model.close()


def test_mlp_sublayer_matches_oracle(tiny):
    cfg, prov, model = tiny
    _, h = inputs(cfg, 11, 200)
    for layer in (0, 5):
        ht = torch.from_numpy(h.astype(np.float32)).cuda()
        model.mlp_sublayer(layer, ht)
        torch.cuda.synchronize()
        ref = oracle(cfg, prov).mlp_sublayer(layer, h)
        assert_parity(to_np(ht), ref, tol_abs=5e-3, tol_cos=0.9999, what=f"mlp layer {layer}")


@pytest.mark.parametrize("layer", [0, 1])     # SWA, full
def test_attention_sublayer_matches_oracle(tiny, layer):
    cfg, prov, model = tiny
    _, h = inputs(cfg, 12, 150)
    kv = model.kv_cache("last_loop", 2, 256)
    ocache = oracle_cache(cfg, "last_loop")
    orc = oracle(cfg, prov)
    # two calls: the second reads the first's committed keys (ring for SWA)
    for pos0, n in ((0, 90), (90, 60)):
        ht = torch.from_numpy(h[pos0:pos0 + n].astype(np.float32)).cuda()
        model.attention_sublayer(kv, layer, ht, loop=1, seq=1, pos0=pos0)
        torch.cuda.synchronize()
        ref = orc.attention_sublayer(layer, h[pos0:pos0 + n], pos0, 1, 1, ocache)
        assert_parity(to_np(ht), ref, tol_abs=5e-3, tol_cos=0.9999, what=f"attn {layer} @{pos0}")


# ------------------------------------------------------------------ whole stack
@pytest.mark.parametrize("mode", ["per_loop", "last_loop"])
@pytest.mark.parametrize("k", [1, 2, 3, 4])
def test_prefill_matches_oracle(tiny, mode, k):
    cfg, prov, model = tiny
    x, h = inputs(cfg, 13, 128)
    kv = model.kv_cache(mode, 1, 256, k_max=4)
    out = model.prefill(kv, x, k)
    torch.cuda.synchronize()
    assert model.device_status() == 0
    ref = oracle(cfg, prov).forward(h, 0, k, oracle_cache(cfg, mode, k_max=4))
    assert_parity(to_np(out), ref, what=f"prefill {mode} k={k}")
    launches, sub = model.last_call_stats()
    assert sub == 2 * (cfg["n_in_blocks"] + k * cfg["n_rec_blocks"] + cfg["n_out_blocks"])
    assert launches > sub


@pytest.mark.parametrize("mode", ["per_loop", "last_loop"])
@pytest.mark.parametrize("k", [2, 4])
def test_chunked_prefill_then_decode_matches_oracle(tiny, mode, k):
    """Chunks that straddle the 32-slot SWA ring several times, then decode steps
    (per-loop caching at k = 4 reads and writes all four loop slots)."""
    cfg, prov, model = tiny
    x, h = inputs(cfg, 14, 110)
    kv = model.kv_cache(mode, 3, 160, k_max=k)
    ocache = oracle_cache(cfg, mode, k_max=k)
    orc = oracle(cfg, prov)
    seq = 2
    for a, b in ((0, 45), (45, 46), (46, 100)):
        out = model.prefill(kv, x[a:b], k, seq=seq, pos0=a)
        torch.cuda.synchronize()
        ref = orc.forward(h[a:b], a, k, ocache, seq=seq)
        assert_parity(to_np(out), ref, what=f"chunk {a}:{b} {mode}")
    for step, p in enumerate(range(100, 110)):
        d_seq = torch.tensor([seq], dtype=torch.int32, device="cuda")
        d_pos = torch.tensor([p], dtype=torch.int32, device="cuda")
        out = model.decode(kv, x[p:p + 1], d_seq, d_pos, 159, k)
        torch.cuda.synchronize()
        ref = orc.decode(h[p:p + 1], [seq], [p], k, ocache)
        assert_parity(to_np(out), ref, what=f"decode step {step} {mode}")
    assert model.device_status() == 0


def test_decode_batch_of_sequences_matches_oracle(tiny):
    """A batch of sequences at different positions (ragged contexts) in one step."""
    cfg, prov, model = tiny
    k = 2
    mode = "last_loop"
    kv = model.kv_cache(mode, 5, 200, k_max=2)
    ocache = oracle_cache(cfg, mode, k_max=2)
    orc = oracle(cfg, prov)
    lens = [3, 40, 77, 1, 64]
    xs = [inputs(cfg, 20 + s, lens[s] + 2) for s in range(5)]
    for s, L in enumerate(lens):
        model.prefill(kv, xs[s][0][:L], k, seq=s, pos0=0)
        orc.forward(xs[s][1][:L], 0, k, ocache, seq=s)
    order = [3, 0, 4, 1, 2]          # rows in a different order than the sequences
    for step in range(2):
        rows_t = torch.cat([xs[s][0][lens[s] + step:lens[s] + step + 1] for s in order])
        rows_h = np.concatenate([xs[s][1][lens[s] + step:lens[s] + step + 1] for s in order])
        d_seq = torch.tensor(order, dtype=torch.int32, device="cuda")
        d_pos = torch.tensor([lens[s] + step for s in order], dtype=torch.int32, device="cuda")
        out = model.decode(kv, rows_t, d_seq, d_pos, 199, k)
        torch.cuda.synchronize()
        ref = orc.decode(rows_h, order, [lens[s] + step for s in order], k, ocache)
        assert_parity(to_np(out), ref, what=f"batched decode step {step}")


def test_window_mask_is_exact():
    """W = 4: an off-by-one in the sliding window or causal mask moves a fifth of the
    softmax mass and fails the bar."""
    cfg, prov, model = build("tiny", seed=3, variant="random", window=4)
    x, h = inputs(cfg, 15, 70)
    kv = model.kv_cache("last_loop", 1, 128)
    out = model.prefill(kv, x[:60], 2)
    ocache = oracle_cache(cfg, "last_loop")
    orc = oracle(cfg, prov)
    ref = orc.forward(h[:60], 0, 2, ocache)
    assert_parity(to_np(out), ref, tol_cos=0.9995, what="W=4 prefill")
    for p in range(60, 66):
        d = torch.tensor([0], dtype=torch.int32, device="cuda")
        pp = torch.tensor([p], dtype=torch.int32, device="cuda")
        out = model.decode(kv, x[p:p + 1], d, pp, 127, 2)
        ref = orc.decode(h[p:p + 1], [0], [p], 2, ocache)
        assert_parity(to_np(out), ref, tol_cos=0.9995, what=f"W=4 decode {p}")


def test_modes_identical_at_k1(tiny):
    """Per-loop and last-loop caching run the same kernels on the same slots at k = 1."""
    cfg, prov, model = tiny
    x, _ = inputs(cfg, 16, 96)
    outs, caches = [], []
    for mode in ("per_loop", "last_loop"):
        kv = model.kv_cache(mode, 1, 128, k_max=1)
        kv.buf.zero_()
        outs.append(model.prefill(kv, x[:80], 1).clone())
        torch.cuda.synchronize()
        caches.append(kv.buf.clone())
    assert torch.equal(outs[0], outs[1])
    assert torch.equal(caches[0], caches[1])


def test_kv_cache_slots_and_contents(tiny):
    """Cache indexing is exact: full layers fill slots 0..T-1 and leave the rest
    untouched (bit-exact sentinel); SWA rings hold positions T-W..T-1 at pos % W;
    the stored k_hat / v match the oracle's entries for those positions."""
    cfg, prov, model = tiny
    T, ctx = 100, 128
    x, h = inputs(cfg, 17, T)
    kv = model.kv_cache("last_loop", 2, ctx, k_max=1)
    kv.buf.view(torch.int16).fill_(0x7F7F)
    model.prefill(kv, x, 2, seq=1)
    torch.cuda.synchronize()
    ocache = oracle_cache(cfg, "last_loop")
    oracle(cfg, prov).forward(h, 0, 2, ocache, seq=1)
    sentinel = torch.tensor(0x7F7F, dtype=torch.int16)
    for layer in range(8):
        full = layer % cfg["full_period"] == cfg["full_period"] - 1
        for head in range(cfg["n_kv_heads"]):
            kview = kv.entry_view(layer, 1, 1, head, "k")
            vview = kv.entry_view(layer, 1, 1, head, "v")
            other = kv.entry_view(layer, 1, 0, head, "k")     # sequence 0: never written
            assert bool((other.view(torch.int16).cpu() == sentinel).all())
            if full:
                assert bool((kview[T:].view(torch.int16).cpu() == sentinel).all())
                positions = list(range(T))
                slots = positions
            else:
                positions = list(range(T - cfg["window"], T))
                slots = [p % cfg["window"] for p in positions]
            K, V = ocache.read(layer, 1, 1, positions[0], positions[-1] + 1)
            gk = to_np(kview[slots])
            gv = to_np(vview[slots])
            assert np.abs(gk - K[:, head]).max() < 3e-2, (layer, head)
            assert np.abs(gv - V[:, head]).max() < 3e-2, (layer, head)


def test_host_buffers_give_the_same_result(tiny):
    """dory_prefill with pinned host h_in / h_out equals the device-buffer call."""
    cfg, prov, model = tiny
    x, _ = inputs(cfg, 18, 64)
    kv = model.kv_cache("last_loop", 1, 64)
    dev = model.prefill(kv, x, 2).cpu()
    hin = x.cpu().pin_memory()
    hout = torch.empty_like(hin).pin_memory()
    model.prefill(kv, hin, 2, h_out=hout)
    torch.cuda.synchronize()
    assert torch.equal(dev, hout)


def test_argument_errors(tiny):
    from looped_ngpt_transformer_fwd_b200.binding import DoryError
    cfg, prov, model = tiny
    x, _ = inputs(cfg, 19, 16)
    kv = model.kv_cache("per_loop", 1, 32, k_max=2)
    with pytest.raises(DoryError) as e:
        model.prefill(kv, x, 3)
    assert e.value.status == -4
    with pytest.raises(DoryError) as e:
        model.prefill(kv, x, 0)
    assert e.value.status == -3
    with pytest.raises(DoryError) as e:
        model.prefill(kv, x, 1, pos0=20)
    assert e.value.status == -5
    assert model.device_status() == 0


def test_kernel_profiling_counts_every_launch(tiny):
    """Instrumented graphs time every kernel; counts add up to the call's launches."""
    cfg, prov, model = tiny
    x, _ = inputs(cfg, 21, 64)
    kv = model.kv_cache("last_loop", 1, 64, k_max=2)
    model.profile(True)
    try:
        out_p = model.prefill(kv, x, 2).clone()
        prof = model.profile_read()
    finally:
        model.profile(False)
    out = model.prefill(kv, x, 2)
    torch.cuda.synchronize()
    assert torch.equal(out, out_p)
    launches, sub = model.last_call_stats()
    assert sum(n for _, n in prof.values()) == launches
    assert prof["gateup"][1] == prof["down"][1] == sub // 2
    assert all(t > 0 for t, n in prof.values() if n)


# ------------------------------------------------------------------ head_dim 128
# (d 512, 4/2 heads of 128, window 128): prefill attention runs on the tcgen05
# kernel at any chunk start and window (key tiles across the chunk start or a
# ring's end gathered row by row), on the mma.sync online-softmax kernel when
# the static softmax maximum would underflow; both must match the oracle.
HD128 = dict(d_model=512, n_q_heads=4, n_kv_heads=2, head_dim=128, d_ff=1024, window=128,
             softmax_scale=float(np.sqrt(128.0)))


@pytest.fixture(scope="module")
def hd128():
    return build("tiny", seed=7, variant="random", **HD128)


@pytest.mark.parametrize("mode", ["per_loop", "last_loop"])
@pytest.mark.parametrize("k", [2, 4])
def test_hd128_prefill_matches_oracle(hd128, mode, k):
    cfg, prov, model = hd128
    x, h = inputs(cfg, 51, 300)
    kv = model.kv_cache(mode, 1, 400, k_max=k)
    out = model.prefill(kv, x, k)
    torch.cuda.synchronize()
    assert model.device_status() == 0
    ref = oracle(cfg, prov).forward(h, 0, k, oracle_cache(cfg, mode, k_max=k))
    assert_parity(to_np(out), ref, what=f"hd128 prefill {mode} k={k}")
    assert model.attention_paths()["prefill_tc"] > 0


@pytest.mark.parametrize("mode", ["per_loop", "last_loop"])
@pytest.mark.parametrize("k", [2, 4])
def test_hd128_chunked_prefill_and_decode(hd128, mode, k):
    """Chunks at multiples of 128 (tensor-core attention reading cached tiles and
    ring slots), unaligned chunks (the same kernel, gathering the key tile that
    holds both cached and fresh keys), then decode steps."""
    cfg, prov, model = hd128
    x, h = inputs(cfg, 52, 420)
    kv = model.kv_cache(mode, 2, 480, k_max=k)
    ocache = oracle_cache(cfg, mode, k_max=k)
    orc = oracle(cfg, prov)
    seq = 1
    for a, b in ((0, 128), (128, 256), (256, 384), (384, 405), (405, 416)):
        out = model.prefill(kv, x[a:b], k, seq=seq, pos0=a)
        torch.cuda.synchronize()
        paths = model.attention_paths()
        assert paths["prefill_tc"] > 0 and paths["prefill_mma"] == 0, (a, paths)
        ref = orc.forward(h[a:b], a, k, ocache, seq=seq)
        assert_parity(to_np(out), ref, what=f"hd128 chunk {a}:{b} {mode}")
    for p in range(416, 420):
        d_seq = torch.tensor([seq], dtype=torch.int32, device="cuda")
        d_pos = torch.tensor([p], dtype=torch.int32, device="cuda")
        out = model.decode(kv, x[p:p + 1], d_seq, d_pos, 479, k)
        ref = orc.decode(h[p:p + 1], [seq], [p], k, ocache)
        assert_parity(to_np(out), ref, what=f"hd128 decode {p} {mode}")
    assert model.device_status() == 0


def _alpha_one_model(cfg, seed, sqk=None):
    """A model and its weight provider with alpha_attn = 1 (and optionally every
    s_qk entry set to `sqk`), in the generator's storage format."""
    from tests.oracle_util import modified
    from oracle import weights_from_generator
    from looped_ngpt_transformer_fwd_b200.model import DoryModel
    from synthetic import f32_to_bf16_bits
    base = weights_from_generator(cfg, seed, "random")

    def change(b, w):
        w["alpha_attn"][:] = 1.0
        if sqk is not None:
            w["s_qk"][:] = sqk
    prov = modified(base, change)

    def as_generator_format(b):
        w = prov(b)
        return {k_: (v.astype(np.float32) if k_ in ("alpha_attn", "alpha_mlp", "s_qk")
                     else f32_to_bf16_bits(v.astype(np.float32))) for k_, v in w.items()}
    return DoryModel(cfg, as_generator_format), as_generator_format


@pytest.mark.parametrize("window", [100, 128])
def test_hd128_unaligned_chunks_alpha_one_on_tensor_cores(window):
    """Chunks starting off the 128-key tile grid, and a window that is not a
    multiple of 128 (ring tiles that run past the ring's end), on the tcgen05
    kernel with alpha = 1: the attention output is compared almost undiluted,
    so a wrong row in a gathered key tile would show."""
    from synthetic import load_config
    cfg = load_config("tiny", **dict(HD128, window=window))
    model, prov = _alpha_one_model(cfg, 9)
    _, h = inputs(cfg, 54, 460)
    kv = model.kv_cache("last_loop", 1, 512)
    ocache = oracle_cache(cfg, "last_loop")
    orc = oracle(cfg, prov)
    for layer in (0, 1):                        # SWA, full
        for pos0, n in ((0, 200), (200, 57), (257, 130), (387, 73)):
            ht = torch.from_numpy(h[pos0:pos0 + n].astype(np.float32)).cuda()
            model.attention_sublayer(kv, layer, ht, loop=1, seq=0, pos0=pos0)
            torch.cuda.synchronize()
            paths = model.attention_paths()
            assert paths["prefill_tc"] > 0 and paths["prefill_mma"] == 0, paths
            ref = orc.attention_sublayer(layer, h[pos0:pos0 + n], pos0, 0, 1, ocache)
            assert_parity(to_np(ht), ref, tol_abs=1e-2, tol_cos=0.99995,
                          what=f"alpha=1 W={window} layer {layer} @{pos0}")
    assert model.device_status() == 0
    model.close()


def test_hd128_large_sqk_runs_the_online_softmax_kernel():
    """s_qk = 3 everywhere bounds the logits by softmax_scale * 9 ~ 102, too wide
    for the static softmax maximum (2 B log2(e) > 120), so prefill attention runs
    the mma.sync online-softmax kernel, aligned and unaligned chunks alike.  At
    logits near 100 the bf16 rounding of q and k (2^-9 relative) moves an
    exponent by up to ~0.2, so this case's bar is cos >= 0.999."""
    from synthetic import load_config
    cfg = load_config("tiny", **HD128)
    model, prov = _alpha_one_model(cfg, 10, sqk=3.0)
    _, h = inputs(cfg, 55, 300)
    kv = model.kv_cache("last_loop", 1, 320)
    ocache = oracle_cache(cfg, "last_loop")
    orc = oracle(cfg, prov)
    for pos0, n in ((0, 128), (128, 77), (205, 95)):
        ht = torch.from_numpy(h[pos0:pos0 + n].astype(np.float32)).cuda()
        model.attention_sublayer(kv, 1, ht, loop=1, seq=0, pos0=pos0)
        torch.cuda.synchronize()
        paths = model.attention_paths()
        assert paths["prefill_mma"] > 0 and paths["prefill_tc"] == 0, paths
        ref = orc.attention_sublayer(1, h[pos0:pos0 + n], pos0, 0, 1, ocache)
        assert_parity(to_np(ht), ref, tol_abs=2e-2, tol_cos=0.999,
                      what=f"online softmax @{pos0}")
    assert model.device_status() == 0
    model.close()


@pytest.mark.parametrize("layer", [0, 1])      # SWA (W = 128), full
def test_hd128_attention_sublayer_alpha_one_is_tight(layer):
    """alpha = 1 makes the sublayer output Norm(o W_o^T) itself, so the attention
    output is compared almost undiluted: a key added or dropped at a mask edge
    (one of ~128) would move it by ~0.8 %, far above the bf16 error."""
    from tests.oracle_util import modified
    from oracle import weights_from_generator
    from looped_ngpt_transformer_fwd_b200.model import DoryModel
    from synthetic import load_config
    cfg = load_config("tiny", **HD128)
    base = weights_from_generator(cfg, 8, "random")

    def alpha_one(b, w):
        w["alpha_attn"][:] = 1.0
    prov = modified(base, alpha_one)

    def as_generator_format(b):
        w = prov(b)
        from synthetic import f32_to_bf16_bits
        out = {}
        for k_, v in w.items():
            if k_ in ("alpha_attn", "alpha_mlp", "s_qk"):
                out[k_] = v.astype(np.float32)
            else:
                out[k_] = f32_to_bf16_bits(v.astype(np.float32))
        return out
    model = DoryModel(cfg, as_generator_format)
    _, h = inputs(cfg, 53, 448)
    kv = model.kv_cache("last_loop", 1, 512)
    ocache = oracle_cache(cfg, "last_loop")
    orc = oracle(cfg, as_generator_format)
    for pos0, n in ((0, 256), (256, 192)):
        ht = torch.from_numpy(h[pos0:pos0 + n].astype(np.float32)).cuda()
        model.attention_sublayer(kv, layer, ht, loop=1, seq=0, pos0=pos0)
        torch.cuda.synchronize()
        ref = orc.attention_sublayer(layer, h[pos0:pos0 + n], pos0, 0, 1, ocache)
        assert_parity(to_np(ht), ref, tol_abs=1e-2, tol_cos=0.99995,
                      what=f"alpha=1 attention layer {layer} @{pos0}")
    model.close()


def test_recycled_cache_handles_do_not_reuse_stale_graphs(tiny):
    """Caches freed and re-created with another mode may land on the same handle
    and buffer addresses; every call must still run the graph of its own cache."""
    import gc
    cfg, prov, model = tiny
    x, h = inputs(cfg, 22, 80)
    for mode in ("per_loop", "last_loop", "per_loop", "last_loop"):
        kv = model.kv_cache(mode, 1, 96, k_max=2)
        ocache = oracle_cache(cfg, mode, k_max=2)
        orc = oracle(cfg, prov)
        for a, b in ((0, 40), (40, 80)):
            out = model.prefill(kv, x[a:b], 2, pos0=a)
            torch.cuda.synchronize()
            assert_parity(to_np(out), orc.forward(h[a:b], a, 2, ocache), what=f"{mode} {a}:{b}")
        kv.free()
        del kv
        gc.collect()


# ------------------------------------------------------- loop count per sequence
@pytest.mark.parametrize("mode", ["last_loop", "per_loop"])
def test_mixed_k_decode_matches_oracle(tiny, mode):
    """One decode step with its own loop count per sequence: each row equals that
    sequence decoded alone with its k (rows in another order than sequences)."""
    cfg, prov, model = tiny
    ks = [1, 4, 2, 3]
    k_hi = max(ks)
    kv = model.kv_cache(mode, 4, 128, k_max=k_hi)
    ocache = oracle_cache(cfg, mode, k_max=k_hi)
    orc = oracle(cfg, prov)
    lens = [5, 33, 70, 2]
    xs = [inputs(cfg, 40 + s, lens[s] + 2) for s in range(4)]
    for s, L in enumerate(lens):
        model.prefill(kv, xs[s][0][:L], ks[s], seq=s, pos0=0)
        orc.forward(xs[s][1][:L], 0, ks[s], ocache, seq=s)
    order = [2, 0, 3, 1]
    for step in range(2):
        rows_t = torch.cat([xs[s][0][lens[s] + step:lens[s] + step + 1] for s in order])
        d_seq = torch.tensor(order, dtype=torch.int32, device="cuda")
        d_pos = torch.tensor([lens[s] + step for s in order], dtype=torch.int32, device="cuda")
        d_k = torch.tensor([ks[s] for s in order], dtype=torch.int32, device="cuda")
        out = to_np(model.decode_mixed(kv, rows_t, d_seq, d_pos, d_k, 127, k_hi))
        torch.cuda.synchronize()
        for i, s in enumerate(order):
            p = lens[s] + step
            ref = orc.decode(xs[s][1][p:p + 1], [s], [p], ks[s], ocache)
            assert_parity(out[i:i + 1], ref, what=f"mixed-k decode step {step} seq {s} k={ks[s]} {mode}")
    assert model.device_status() == 0


def test_mixed_k_decode_with_equal_counts_is_the_plain_step(tiny):
    """Every row with the same count: bit for bit the plain decode step."""
    cfg, prov, model = tiny
    k = 2
    caches = [model.kv_cache("last_loop", 3, 64, k_max=k) for _ in range(2)]
    lens = [7, 20, 41]
    xs = [inputs(cfg, 60 + s, lens[s] + 1)[0] for s in range(3)]
    for kv in caches:
        for s, L in enumerate(lens):
            model.prefill(kv, xs[s][:L], k, seq=s, pos0=0)
    rows = torch.cat([xs[s][lens[s]:lens[s] + 1] for s in range(3)])
    d_seq = torch.arange(3, dtype=torch.int32, device="cuda")
    d_pos = torch.tensor(lens, dtype=torch.int32, device="cuda")
    d_k = torch.full((3,), k, dtype=torch.int32, device="cuda")
    plain = model.decode(caches[0], rows, d_seq, d_pos, 63, k)
    mixed = model.decode_mixed(caches[1], rows, d_seq, d_pos, d_k, 63, k)
    torch.cuda.synchronize()
    assert torch.equal(plain.view(torch.int16), mixed.view(torch.int16))
    assert model.device_status() == 0


def test_mixed_k_decode_rejects_bad_counts(tiny):
    """Host-checked k_hi errors, and a device count outside 1..k_hi reported as a
    bounds error (the row's recurrent loops are skipped, nothing faults)."""
    from looped_ngpt_transformer_fwd_b200.binding import DoryError
    cfg, prov, model = tiny
    kv = model.kv_cache("per_loop", 2, 32, k_max=2)
    x, _ = inputs(cfg, 70, 4)
    for s in range(2):
        model.prefill(kv, x[2 * s:2 * s + 1], 2, seq=s, pos0=0)
    rows = x[1:3]
    d_seq = torch.arange(2, dtype=torch.int32, device="cuda")
    d_pos = torch.ones(2, dtype=torch.int32, device="cuda")
    with pytest.raises(DoryError) as e:
        model.decode_mixed(kv, rows, d_seq, d_pos, torch.full((2,), 2, dtype=torch.int32,
                                                               device="cuda"), 31, 3)
    assert e.value.status == -4          # k_hi above the per-loop cache's k_max
    with pytest.raises(DoryError) as e:
        model.decode_mixed(kv, rows, d_seq, d_pos, torch.full((2,), 1, dtype=torch.int32,
                                                               device="cuda"), 31, 0)
    assert e.value.status == -3          # k_hi out of range
    bad = torch.tensor([2, 0], dtype=torch.int32, device="cuda")
    model.decode_mixed(kv, rows, d_seq, d_pos, bad, 31, 2)
    torch.cuda.synchronize()
    assert model.device_status() == -11
    assert model.device_status() == 0    # the status word was cleared


@pytest.mark.parametrize("mode", ["per_loop", "last_loop"])
def test_hd128_chunks_twice_the_window(hd128, mode):
    """Chunks of 2W (W = 128) at chunk-aligned starts, as the long-context prefill
    runs 8192-token chunks over a 4096-slot ring: every chunk overwrites the whole
    ring and reads the previous chunk's last W keys from it."""
    cfg, prov, model = hd128
    k = 4
    x, h = inputs(cfg, 54, 1024 + 2)
    kv = model.kv_cache(mode, 1, 1100, k_max=k)
    ocache = oracle_cache(cfg, mode, k_max=k)
    orc = oracle(cfg, prov)
    for a in range(0, 1024, 256):
        out = model.prefill(kv, x[a:a + 256], k, pos0=a)
        torch.cuda.synchronize()
        paths = model.attention_paths()
        assert paths["prefill_mma"] == 0
        assert paths["prefill_tc"] == cfg["n_in_blocks"] + k * cfg["n_rec_blocks"] + cfg["n_out_blocks"]
        ref = orc.forward(h[a:a + 256], a, k, ocache)
        assert_parity(to_np(out), ref, what=f"2W chunk at {a} {mode}")
    for p in (1024, 1025):
        d = torch.zeros(1, dtype=torch.int32, device="cuda")
        pp = torch.tensor([p], dtype=torch.int32, device="cuda")
        out = model.decode(kv, x[p:p + 1], d, pp, 1099, k)
        ref = orc.decode(h[p:p + 1], [0], [p], k, ocache)
        assert_parity(to_np(out), ref, what=f"decode {p} after 2W chunks {mode}")
    assert model.device_status() == 0


# ------------------------------------------------------- GQA group of 3 (the 4B grouping)
# 6 query heads over 2 KV heads of 128: three query heads per KV head, as in the
# 24/8 4B shape, at sizes the oracle runs in seconds (many query tiles, so the
# late, full-window tiles of the tensor-core kernel are compared too).
G3 = dict(d_model=768, n_q_heads=6, n_kv_heads=2, head_dim=128, d_ff=1024, window=128,
          softmax_scale=float(np.sqrt(128.0)))


@pytest.fixture(scope="module")
def g3():
    return build("tiny", seed=9, variant="random", **G3)


@pytest.mark.parametrize("mode", ["per_loop", "last_loop"])
@pytest.mark.parametrize("k", [1, 4])
def test_gqa3_prefill_matches_oracle(g3, mode, k):
    cfg, prov, model = g3
    x, h = inputs(cfg, 55, 640)
    kv = model.kv_cache(mode, 1, 700, k_max=k)
    out = model.prefill(kv, x, k)
    torch.cuda.synchronize()
    assert model.device_status() == 0
    assert model.attention_paths()["prefill_tc"] > 0
    ref = oracle(cfg, prov).forward(h, 0, k, oracle_cache(cfg, mode, k_max=k))
    assert_parity(to_np(out), ref, what=f"GQA-3 prefill {mode} k={k}")


@pytest.mark.parametrize("mode", ["per_loop", "last_loop"])
def test_gqa3_chunks_and_decode_batch(g3, mode):
    cfg, prov, model = g3
    k = 2
    kv = model.kv_cache(mode, 3, 700, k_max=k)
    ocache = oracle_cache(cfg, mode, k_max=k)
    orc = oracle(cfg, prov)
    lens = [384, 300, 513]
    xs = [inputs(cfg, 56 + s, lens[s] + 2) for s in range(3)]
    for s, L in enumerate(lens):
        cut = 256 if L > 256 else L
        for a, b in ((0, cut), (cut, L)):
            if b > a:
                out = model.prefill(kv, xs[s][0][a:b], k, seq=s, pos0=a)
                ref = orc.forward(xs[s][1][a:b], a, k, ocache, seq=s)
                assert_parity(to_np(out), ref, what=f"GQA-3 seq {s} chunk {a}:{b} {mode}")
    for step in range(2):
        rows_t = torch.cat([xs[s][0][lens[s] + step:lens[s] + step + 1] for s in range(3)])
        rows_h = np.concatenate([xs[s][1][lens[s] + step:lens[s] + step + 1] for s in range(3)])
        d_seq = torch.arange(3, dtype=torch.int32, device="cuda")
        d_pos = torch.tensor([L + step for L in lens], dtype=torch.int32, device="cuda")
        out = model.decode(kv, rows_t, d_seq, d_pos, 699, k)
        torch.cuda.synchronize()
        assert model.attention_paths()["decode_tma"] > 0
        ref = orc.decode(rows_h, [0, 1, 2], [L + step for L in lens], k, ocache)
        assert_parity(to_np(out), ref, what=f"GQA-3 decode step {step} {mode}")
    assert model.device_status() == 0


# ------------------------------------------------------- extrapolated loop counts
@pytest.fixture(scope="module")
def tiny_extrap():
    return build("tiny", seed=10, variant="random", allow_extrapolated_k=True)


@pytest.mark.parametrize("mode", ["per_loop", "last_loop"])
@pytest.mark.parametrize("k", [6, 8])
def test_extrapolated_k_prefill_and_decode(tiny_extrap, mode, k):
    """Loop counts beyond the trained 1..4 ("Dory1.0-4B: A Looped Normalized-GPT",
    Main Findings: base scores at k = 6 and 8), accepted with allow_extrapolated_k:
    the same stack with more passes of the shared block."""
    cfg, prov, model = tiny_extrap
    x, h = inputs(cfg, 57, 82)
    kv = model.kv_cache(mode, 1, 96, k_max=k)
    ocache = oracle_cache(cfg, mode, k_max=k)
    orc = oracle(cfg, prov)
    out = model.prefill(kv, x[:80], k)
    torch.cuda.synchronize()
    assert_parity(to_np(out), orc.forward(h[:80], 0, k, ocache), what=f"k={k} prefill {mode}")
    _, sub = model.last_call_stats()
    assert sub == 2 * (cfg["n_in_blocks"] + k * cfg["n_rec_blocks"] + cfg["n_out_blocks"])
    for p in (80, 81):
        d = torch.zeros(1, dtype=torch.int32, device="cuda")
        pp = torch.tensor([p], dtype=torch.int32, device="cuda")
        out = model.decode(kv, x[p:p + 1], d, pp, 95, k)
        ref = orc.decode(h[p:p + 1], [0], [p], k, ocache)
        assert_parity(to_np(out), ref, what=f"k={k} decode {p} {mode}")
    assert model.device_status() == 0


def test_extrapolated_k_needs_the_flag(tiny):
    from looped_ngpt_transformer_fwd_b200.binding import DoryError
    cfg, prov, model = tiny
    x, _ = inputs(cfg, 58, 8)
    kv = model.kv_cache("last_loop", 1, 16, k_max=1)
    with pytest.raises(DoryError) as e:
        model.prefill(kv, x, 6)
    assert e.value.status == -3


# ------------------------------------------------------- failure path: bounded waits
def test_bounded_wait_timeout_is_reported_and_the_model_stays_usable(tiny):
    """A kernel's wait that runs out records a timeout in the device status word
    instead of hanging the GPU.  The test kernel waits on a barrier nothing
    completes, with a 5 ms limit; the status reads DORY_ERR_DEVICE_TIMEOUT once,
    and the next prefill still matches the oracle."""
    cfg, prov, model = tiny
    assert model.device_status() == 0
    model.wait_timeout(5000)
    torch.cuda.synchronize()
    assert model.device_status() == -9
    assert model.device_status() == 0
    x, h = inputs(cfg, 59, 64)
    kv = model.kv_cache("last_loop", 1, 64, k_max=2)
    out = model.prefill(kv, x, 2)
    torch.cuda.synchronize()
    assert model.device_status() == 0
    ref = oracle(cfg, prov).forward(h, 0, 2, oracle_cache(cfg, "last_loop", k_max=2))
    assert_parity(to_np(out), ref, what="prefill after a timeout")


# ------------------------------------------------------- fused projection + nGPT update
@pytest.mark.parametrize("mode", ["per_loop", "last_loop"])
def test_fused_update_matches_unfused_path_and_oracle(hd128, mode):
    """The output / down projections with the nGPT update (and the re-injection)
    in their epilogue, a 2-CTA cluster per row at d_model 512, against the
    unfused path (projection, then the row kernel) and against the oracle."""
    cfg, prov, model = hd128
    k = 3
    x, h = inputs(cfg, 61, 300)
    outs = []
    for fused in (True, False):
        assert model.fused_update(fused) == fused
        kv = model.kv_cache(mode, 1, 320, k_max=k)
        # every workspace byte is written before it is read: fill it with junk first
        model.workspace(300).fill_(0x3F)
        outs.append(to_np(model.prefill(kv, x, k)))
        torch.cuda.synchronize()
    model.fused_update(False)
    ref = oracle(cfg, prov).forward(h, 0, k, oracle_cache(cfg, mode, k_max=k))
    assert_parity(outs[0], ref, what=f"fused {mode}")
    assert_parity(outs[1], ref, what=f"unfused {mode}")
    assert_parity(outs[0], outs[1], tol_abs=2e-2, tol_cos=0.9995, what="fused vs unfused")
    assert model.device_status() == 0


def test_fused_update_is_deterministic(g3):
    """Row sums are added in a fixed order: two runs give the same bits (d_model
    768: a 2-CTA cluster of 384 columns each), and match the oracle."""
    cfg, prov, model = g3
    x, h = inputs(cfg, 62, 400)
    kv = model.kv_cache("last_loop", 1, 400, k_max=2)
    model.workspace(400).fill_(0x3F)
    assert model.fused_update(True)
    try:
        a = model.prefill(kv, x, 2).clone()
        b = model.prefill(kv, x, 2)
        torch.cuda.synchronize()
    finally:
        model.fused_update(False)
    assert torch.equal(a, b)
    ref = oracle(cfg, prov).forward(h, 0, 2, oracle_cache(cfg, "last_loop", k_max=2))
    assert_parity(to_np(a), ref, what="fused, GQA-3 shape")
