"""Pins of the oracle's block-scaled weight formats (oracle/quant.py).

The element and scale codecs are checked against PyTorch's own float8 types
(a library routine) and against exhaustive nearest-value searches; the block
formats against invariants that a dropped term, a wrong exponent or a
transposed block would break.  The formats are those of the released MXFP8 /
NVFP4 checkpoints ("Dory1.0-4B: A Looped Normalized-GPT", Key Contributions
item 4), read as the public format definitions.
"""

import numpy as np
import pytest
import torch

from oracle import quant as Q


def _nearest_even(x, fmt):
    """Exhaustive search: the closest finite value of the format; on a tie the
    one with the even code; beyond the largest value, the largest value."""
    ebits = 4 if fmt == Q.E4M3 else 2
    codes = np.arange(1 << (ebits + fmt[1]))         # the non-negative codes
    vals = Q.decode(codes, fmt)
    ok = np.isfinite(vals)
    codes, vals = codes[ok], vals[ok]
    out = []
    for v in np.asarray(x, dtype=np.float64):
        a = min(abs(v), fmt[2])
        d = np.abs(vals - a)
        best = np.flatnonzero(d == d.min())
        if len(best) > 1:
            best = [c for c in best if codes[c] % 2 == 0]
        out.append(np.copysign(vals[best[0]], v))
    return np.array(out)


def test_e4m3_decode_matches_torch_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = Q.decode(codes, Q.E4M3)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(got[fin], ref[fin])
    assert np.nanmax(got) == 448.0 and np.nanmin(np.abs(got[got != 0])) == 2.0 ** -9


def test_e4m3_rounding_matches_torch_in_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.uniform(-460, 460, 4000),
        rng.standard_normal(2000) * 1e-2,
        np.exp2(rng.uniform(-12, 8.8, 2000)) * rng.choice([-1, 1], 2000),
        # exact ties go to the even code: 1 + 1/16 -> 1, 1 + 3/16 -> 1.25; in the
        # subnormal range (step 2^-9) 2^-10 -> 0 and 3 * 2^-10 -> 2^-8
        [1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10, 0.0, -0.0, 448.0, 460.0],
    ])
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = Q.round_to_format(x.astype(np.float32).astype(np.float64), Q.E4M3)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("fmt", [Q.E4M3, Q.E2M1], ids=["e4m3", "e2m1"])
def test_rounding_matches_exhaustive_search(fmt):
    rng = np.random.default_rng(1)
    vmax = fmt[2]
    x = np.concatenate([rng.uniform(-1.2 * vmax, 1.2 * vmax, 3000),
                        np.exp2(rng.uniform(-12, np.log2(vmax) + 0.5, 3000)),
                        Q.decode(np.arange(1 << (5 if fmt == Q.E2M1 else 8)), fmt)])
    x = x[np.isfinite(x)]
    # midpoints between consecutive representable values are exact ties
    vals = np.unique(np.abs(x[np.isin(x, Q.decode(np.arange(128 if fmt == Q.E4M3 else 8), fmt))]))
    x = np.concatenate([x, (vals[1:] + vals[:-1]) / 2])
    assert np.array_equal(Q.round_to_format(x, fmt), _nearest_even(x, fmt))


@pytest.mark.parametrize("fmt,n", [(Q.E4M3, 256), (Q.E2M1, 16)], ids=["e4m3", "e2m1"])
def test_encode_inverts_decode(fmt, n):
    codes = np.arange(n)
    vals = Q.decode(codes, fmt)
    fin = np.isfinite(vals)
    assert np.array_equal(Q.encode(vals[fin], fmt), codes[fin])


def test_e2m1_value_set():
    # 1 sign, 2 exponent (bias 1), 1 mantissa bit: eight magnitudes, largest 6,
    # smallest positive 0.5 (subnormal), all exactly representable in E4M3
    mags = Q.decode(np.arange(8), Q.E2M1)
    assert len(set(mags)) == 8 and mags.max() == 6.0 and mags[mags > 0].min() == 0.5
    assert np.array_equal(Q.round_to_format(mags, Q.E4M3), mags)
    assert np.array_equal(Q.decode(np.arange(8, 16), Q.E2M1), -mags)


def test_e8m0_decode_matches_torch():
    codes = np.arange(255, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    assert np.array_equal(Q.e8m0_value(codes), ref)


def _weights(n=12, k=128, seed=3):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((n, k)) * 0.02
    w[0, :32] = 0.0                                  # an all-zero block
    w[1, 32:64] *= 1e-6                              # a tiny block
    return w


def test_mxfp8_block_scale_and_error_bound():
    w = _weights()
    codes, scales = Q.mxfp8_quantize(w)
    assert codes.shape == w.shape and scales.shape == (12, 4)
    x = Q.e8m0_value(scales)
    blocks = w.reshape(12, 4, 32)
    amax = np.abs(blocks).max(axis=2)
    nz = amax > 0
    # the block's largest magnitude lands in [256, 512) in scale units
    assert np.all((amax[nz] / x[nz] >= 256) & (amax[nz] / x[nz] < 512))
    w_hat = Q.mxfp8_dequantize(codes, scales).reshape(12, 4, 32)
    scaled = np.abs(blocks) / x[:, :, None]
    err = np.abs(blocks - w_hat)
    normal = (scaled >= 2.0 ** -6) & (scaled <= 448)
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(blocks[normal]) * (1 + 1e-12))
    sat = scaled > 448
    assert np.allclose(err[sat], (scaled[sat] - 448) * np.broadcast_to(x[:, :, None], sat.shape)[sat])
    assert np.all(w_hat[0, 0] == 0)


def test_mxfp8_power_of_two_scaling_only_moves_the_scales():
    w = _weights(seed=4)
    c1, s1 = Q.mxfp8_quantize(w)
    c2, s2 = Q.mxfp8_quantize(w * 2.0 ** 5)
    assert np.array_equal(c1, c2)
    nz = np.abs(w.reshape(12, 4, 32)).max(axis=2) > 0
    assert np.array_equal(s2.astype(int)[nz], s1.astype(int)[nz] + 5)


def test_mxfp8_round_trip_of_values_on_the_grid():
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 0x78, size=(4, 64)).astype(np.uint8)   # magnitudes below 256
    codes[:, ::32] = 0x78 | 0x80 * (rng.integers(0, 2, (4, 2)))   # one of 256 per block
    codes[:, 1::2] |= 0x80                                         # negative odd columns
    scales = rng.integers(100, 130, size=(4, 2)).astype(np.uint8)
    w = Q.mxfp8_dequantize(codes, scales)
    c2, s2 = Q.mxfp8_quantize(w)
    assert np.array_equal(s2, scales)
    assert np.array_equal(Q.decode(c2, Q.E4M3), Q.decode(codes, Q.E4M3))


def test_nvfp4_elements_are_nearest_and_scales_consistent():
    w = _weights(k=64, seed=6)
    codes, scales, g = Q.nvfp4_quantize(w)
    assert codes.max() < 16 and scales.shape == (12, 4) and g.dtype == np.float32
    s = Q.decode(scales, Q.E4M3)
    assert np.all(np.isfinite(s)) and s.max() <= 448
    blocks = w.reshape(12, 4, 16)
    denom = s * float(g)
    for i in range(12):
        for j in range(4):
            if denom[i, j] == 0:
                assert np.all(codes.reshape(12, 4, 16)[i, j] == 0)
                continue
            want = _nearest_even(blocks[i, j] / denom[i, j], Q.E2M1)
            got = Q.decode(codes.reshape(12, 4, 16)[i, j], Q.E2M1)
            assert np.array_equal(np.abs(got), np.abs(want))
    # the block scale is the E4M3 value nearest to amax_block / (6 g)
    bmax = np.abs(blocks).max(axis=2)
    assert np.array_equal(s.ravel(), _nearest_even((bmax / (6 * float(g))).ravel(), Q.E4M3))


def test_nvfp4_power_of_two_scaling_only_moves_the_tensor_scale():
    w = _weights(k=64, seed=7)
    c1, s1, g1 = Q.nvfp4_quantize(w)
    c2, s2, g2 = Q.nvfp4_quantize(w * 2.0 ** -3)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)
    assert float(g2) == float(g1) * 2.0 ** -3
    d1 = Q.nvfp4_dequantize(c1, s1, g1)
    assert np.array_equal(Q.nvfp4_dequantize(c2, s2, g2), d1 * 2.0 ** -3)


def test_quantized_gemm_uses_the_dequantised_weights():
    rng = np.random.default_rng(8)
    a = rng.standard_normal((5, 64))
    codes, scales = Q.mxfp8_quantize(_weights(n=7, k=64, seed=9))
    w_hat = Q.mxfp8_dequantize(codes, scales)
    c = Q.quantized_gemm(a, w_hat)
    brute = np.array([[sum(a[i, t] * w_hat[j, t] for t in range(64)) for j in range(7)]
                      for i in range(5)])
    assert np.allclose(c, brute, rtol=1e-12, atol=1e-15)


def test_quantised_stacks_track_the_bf16_stack():
    """[P1] Main Findings: MXFP8 weights (post-training quantisation) score roughly
    on par with BF16, NVFP4 needed distillation to close its gap.  The tiny stack
    (k = 2) with dequantised weights stays close to the bf16 one, MXFP8 (3
    mantissa bits) closer than NVFP4 (1 bit); a wrong scale exponent or block
    axis would not."""
    from oracle import Oracle, KVCache, weights_from_generator
    from oracle.quant import dequantized_provider
    from synthetic import load_config, hidden_in
    from synthetic.bf16 import bf16_bits_to_f32
    cfg = load_config("tiny")
    prov = weights_from_generator(cfg, 11)
    h = bf16_bits_to_f32(hidden_in(cfg, 12, 48)).astype(np.float64)
    ref = Oracle(cfg, prov).forward(h, 0, 2, KVCache(cfg, "last_loop", k_max=2))
    err = {}
    for fmt, min_cos in (("mxfp8", 0.9995), ("nvfp4", 0.995)):
        out = Oracle(cfg, dequantized_provider(prov, fmt)).forward(
            h, 0, 2, KVCache(cfg, "last_loop", k_max=2))
        cos = (out * ref).sum(1) / np.linalg.norm(out, axis=1) / np.linalg.norm(ref, axis=1)
        assert cos.min() > min_cos, (fmt, cos.min())
        assert np.allclose(np.linalg.norm(out, axis=1), 1.0, atol=1e-9)
        err[fmt] = np.abs(out - ref).max()
    assert 0 < err["mxfp8"] < err["nvfp4"] / 2


def test_fake_quant_equals_quantise_then_dequantise_per_row():
    rng = np.random.default_rng(13)
    x = rng.standard_normal((3, 5, 96)) * np.exp2(rng.integers(-6, 6, (3, 5, 1)))
    fq = Q.mxfp8_fake_quant(x)
    for i in range(3):
        for j in range(5):
            c, s = Q.mxfp8_quantize(x[i, j][None, :])
            assert np.array_equal(fq[i, j], Q.mxfp8_dequantize(c, s)[0])
    assert np.array_equal(Q.mxfp8_fake_quant(fq), fq)          # idempotent on the grid


def test_mxfp8_gemm_brute_force():
    """Both operands quantised along K, then an exact product: a brute-force sum
    over decoded codes times their two block scales."""
    rng = np.random.default_rng(14)
    a = rng.standard_normal((4, 64))
    w = rng.standard_normal((6, 64)) * 0.03
    ca, sa = Q.mxfp8_quantize(a)
    cw, sw = Q.mxfp8_quantize(w)
    va, vw = Q.decode(ca, Q.E4M3), Q.decode(cw, Q.E4M3)
    brute = np.array([[sum(va[i, t] * 2.0 ** (int(sa[i, t // 32]) - 127) *
                           vw[j, t] * 2.0 ** (int(sw[j, t // 32]) - 127) for t in range(64))
                       for j in range(6)] for i in range(4)])
    assert np.allclose(Q.mxfp8_gemm(a, w), brute, rtol=1e-13, atol=1e-15)
    # relative error of the quantised product stays within a few e4m3 half-ulps
    exact = a @ w.T
    assert np.abs(Q.mxfp8_gemm(a, w) - exact).max() < 0.1 * np.abs(exact).max()


def test_activation_quantised_stack():
    """The oracle with MXFP8 weights and MXFP8 projection inputs (the MX serving
    recipe) stays on the sphere and close to the bf16 stack, closer than NVFP4
    weights alone; quantising the inputs changes the result (the hook is live)."""
    from oracle import Oracle, KVCache, weights_from_generator
    from oracle.quant import dequantized_provider, mxfp8_fake_quant
    from synthetic import load_config, hidden_in
    from synthetic.bf16 import bf16_bits_to_f32
    cfg = load_config("tiny")
    prov = weights_from_generator(cfg, 11)
    h = bf16_bits_to_f32(hidden_in(cfg, 12, 48)).astype(np.float64)
    run = lambda p, aq=None: Oracle(cfg, p, act_quant=aq).forward(
        h, 0, 2, KVCache(cfg, "last_loop", k_max=2))
    ref = run(prov)
    w8 = dequantized_provider(prov, "mxfp8")
    wonly = run(w8)
    both = run(w8, mxfp8_fake_quant)
    cos = (both * ref).sum(1) / np.linalg.norm(both, axis=1) / np.linalg.norm(ref, axis=1)
    assert cos.min() > 0.999
    assert np.allclose(np.linalg.norm(both, axis=1), 1.0, atol=1e-9)
    assert np.abs(both - wonly).max() > 1e-5


def _nvfp4_brute(x, g):
    """NVFP4 values of x [K] (K a multiple of 16) under tensor scale g by
    exhaustive search: each block's scale is the nearest E4M3 value to
    amax / (6 g), each element the nearest E2M1 value to x / (s g), times s g."""
    out = []
    for blk in np.asarray(x, dtype=np.float64).reshape(-1, 16):
        s = _nearest_even([np.abs(blk).max() / (6.0 * float(g))], Q.E4M3)[0]
        unit = s * float(g)
        if unit == 0:
            out.append(np.zeros(16))
            continue
        out.append(_nearest_even(blk / unit, Q.E2M1) * unit)
    return np.concatenate(out)


def test_nvfp4_given_tensor_scale_matches_brute_force():
    """With the tensor scale given (as for the projection inputs), every block
    scale and element is the exhaustive nearest value; unit-norm rows under
    NVFP4_ACT_G = 1 / (6 * 448) never need a block scale above 448."""
    rng = np.random.default_rng(21)
    x = rng.standard_normal((3, 64))
    x[1] *= np.exp2(rng.integers(-8, 0, 64))          # mixed magnitudes, tiny blocks
    x[2, :16] = 0.0                                   # an all-zero block
    x /= np.linalg.norm(x, axis=1, keepdims=True)
    codes, scales, g = Q.nvfp4_quantize(x, Q.NVFP4_ACT_G)
    assert g == Q.NVFP4_ACT_G
    assert Q.decode(scales, Q.E4M3).max() <= 448
    got = Q.nvfp4_dequantize(codes, scales, g)
    for i in range(3):
        assert np.array_equal(got[i], _nvfp4_brute(x[i], g))
    assert np.array_equal(Q.nvfp4_fake_quant(x), got)
    assert np.all(codes[2, :16] == 0) and np.all(scales[2, 0] == 0)


def test_nvfp4_exact_ties_round_to_even():
    """Values exactly halfway between two E2M1 grid points (t s g with t a
    midpoint, all exact in float64) go to the even code: 0.25 -> 0, 0.75 -> 1,
    1.25 -> 1, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4 (times s g)."""
    g = np.float32(2.0 ** -12)
    s = 1.5
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    want = np.array([0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0])
    blk = np.concatenate([[6.0], mids, -mids, [0.0]]) * s * float(g)   # amax / (6 g) = s exactly
    codes, scales, _ = Q.nvfp4_quantize(blk[None, :], g)
    assert Q.decode(scales, Q.E4M3)[0, 0] == s
    vals = Q.decode(codes, Q.E2M1)[0]
    assert np.array_equal(vals[1:8], want) and np.array_equal(vals[8:15], -want)
    assert vals[0] == 6.0


def test_nvfp4_group_shares_the_largest_tensor_scale():
    """Matrices of one GEMM share one g: the block holding the group's largest
    value gets scale 448, and no block of a matrix whose values are at most half
    the group's maximum comes near it (with a per-matrix g every matrix would
    have a 448 block)."""
    from oracle.quant import dequantized_provider, NVFP4_GROUPS
    rng = np.random.default_rng(22)
    names = [n for grp in NVFP4_GROUPS for n in grp]
    base = {n: rng.standard_normal((32, 64)) for n in names}
    for n, top_val in (("wq", 0.02), ("wg", 0.018), ("wk", 0.01), ("wv", 0.005)):
        base[n] *= top_val / np.abs(base[n]).max()      # the group's maxima: 1, 0.9, 0.5, 0.25
    prov = lambda b: base
    deq = dequantized_provider(prov, "nvfp4")(0)
    g = Q.nvfp4_tensor_scale(base["wq"], base["wk"], base["wv"], base["wg"])
    assert g == Q.nvfp4_tensor_scale(np.concatenate([base[n] for n in ("wq", "wk", "wv", "wg")]))
    for n in ("wq", "wk", "wv", "wg"):
        c, sc, _ = Q.nvfp4_quantize(base[n], g)
        assert np.array_equal(deq[n], Q.nvfp4_dequantize(c, sc, g))
    assert Q.decode(Q.nvfp4_quantize(base["wq"], g)[1], Q.E4M3).max() == 448
    assert Q.decode(Q.nvfp4_quantize(base["wg"], g)[1], Q.E4M3).max() < 448
    for n in ("wk", "wv"):
        assert Q.decode(Q.nvfp4_quantize(base[n], g)[1], Q.E4M3).max() <= 240


def test_nvfp4_gemm_brute_force():
    """Both operands quantised along K under their tensor scales, then an exact
    product: a brute-force sum over decoded codes times block and tensor
    scales."""
    rng = np.random.default_rng(23)
    a = rng.standard_normal((3, 32))
    a /= np.linalg.norm(a, axis=1, keepdims=True)
    w = rng.standard_normal((4, 32)) * 0.05
    ca, sa, ga = Q.nvfp4_quantize(a, Q.NVFP4_ACT_G)
    cw, sw, gw = Q.nvfp4_quantize(w)
    va, vw = Q.decode(ca, Q.E2M1), Q.decode(cw, Q.E2M1)
    fa, fw = Q.decode(sa, Q.E4M3), Q.decode(sw, Q.E4M3)
    brute = np.array([[sum(va[i, t] * fa[i, t // 16] * float(ga) * vw[j, t] * fw[j, t // 16] *
                           float(gw) for t in range(32)) for j in range(4)] for i in range(3)])
    assert np.allclose(Q.nvfp4_gemm(a, w), brute, rtol=1e-13, atol=1e-16)
    exact = a @ w.T
    assert np.abs(Q.nvfp4_gemm(a, w) - exact).max() < 0.3 * np.abs(exact).max()


def test_nvfp4_activation_quantised_stack():
    """NVFP4 weights and NVFP4 projection inputs: the tiny stack stays on the
    sphere and near the bf16 stack, further from it than with MXFP8 (1 mantissa
    bit against 3)."""
    from oracle import Oracle, KVCache, weights_from_generator
    from oracle.quant import dequantized_provider, mxfp8_fake_quant, nvfp4_fake_quant
    from synthetic import load_config, hidden_in
    from synthetic.bf16 import bf16_bits_to_f32
    cfg = load_config("tiny")
    prov = weights_from_generator(cfg, 11)
    h = bf16_bits_to_f32(hidden_in(cfg, 12, 48)).astype(np.float64)
    run = lambda p, aq=None: Oracle(cfg, p, act_quant=aq).forward(
        h, 0, 2, KVCache(cfg, "last_loop", k_max=2))
    ref = run(prov)
    nv = run(dequantized_provider(prov, "nvfp4"), nvfp4_fake_quant)
    mx = run(dequantized_provider(prov, "mxfp8"), mxfp8_fake_quant)
    cos = lambda u: ((u * ref).sum(1) / np.linalg.norm(u, axis=1) / np.linalg.norm(ref, axis=1)).min()
    assert cos(nv) > 0.98
    assert np.allclose(np.linalg.norm(nv, axis=1), 1.0, atol=1e-9)
    assert cos(mx) > cos(nv)
