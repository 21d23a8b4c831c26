"""Pins of the CPU oracle against facts the Dory pages and the mathematics fix.

Each test names the passage or the mathematical fact it checks.  Pages:
  [P1] "Dory1.0-4B: A Looped Normalized-GPT" (ai.info AI summary)
  [P4] "Dory 1.0 4B Benchmarks: How Do 1, 2 and 4 Loops Compare?" (goremy.ai)
  [P5] "NVIDIA Nemotron Labs Dory 1.0 4B: ..." (observer.broadside.tech card)
"""

import json
import math
import os

import numpy as np
import pytest

from oracle import (Oracle, KVCache, l2norm, rope, is_full_layer, block_role,
                    kv_cache_bytes, layer_applications, weights_from_generator)
from tests.oracle_util import (tiny, shaped_like_4b, micro, random_float_weights, modified,
                               unit_rows)
from synthetic import load_config

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "dory_structure.json")


def _run(cfg, provider, h, k, mode="per_loop", k_max=4, pos0=0, cache=None, **kw):
    orc = Oracle(cfg, provider, **kw)
    cache = cache or KVCache(cfg, mode, k_max=k_max)
    return orc.forward(h, pos0, k, cache), orc, cache


# ---------------------------------------------------------------- structure

def test_depth_and_pattern_match_golden():
    """[P1] Key Contributions 1 / Main Findings: 72, 112, 192 layer applications at
    k = 1, 2, 4; [P1] Methodology: 27 SWA + 9 full attention layers, 36 MLP layers;
    [P4] What is Dory1.0-4B?: 8 / 20 / 8 blocks."""
    g = json.load(open(GOLDEN))
    cfg = shaped_like_4b()
    assert (cfg["n_in_blocks"], cfg["n_rec_blocks"], cfg["n_out_blocks"]) == (
        g["blocks"]["input"], g["blocks"]["recurrent"], g["blocks"]["output"])
    nb = 36
    kinds = ["full" if is_full_layer(cfg, b) else "swa" for b in range(nb)]
    assert kinds.count("swa") == g["attention_layers"]["sliding_window"]
    assert kinds.count("full") == g["attention_layers"]["full"]
    assert kinds[:4] == ["swa" if p == "swa" else "full" for p in g["pattern"]]
    prov = random_float_weights(cfg, 1)
    h = unit_rows(cfg, 3, 2)
    for k, apps in g["layer_applications"].items():
        k = int(k)
        _, orc, _ = _run(cfg, prov, h, k, k_max=k)
        assert orc.sublayer_apps == apps
        assert layer_applications(cfg, k) == apps
        assert apps == g["depth_formula"]["constant"] + g["depth_formula"]["per_loop"] * k
        assert orc.sublayer_apps // 2 * 1 == 16 + 20 * k   # blocks = 16 + 20k


@pytest.mark.parametrize("k", [6, 8])
def test_depth_formula_holds_at_extrapolated_loop_counts(k):
    """[P1] Main Findings: base scores are reported at k = 6 and 8, loop counts never
    trained on (inference-depth extrapolation).  The stack is the same at any k:
    32 + 40k sublayer applications ([P1] Key Contributions 1's closed form) and
    16 + 20k block passes, with the recurrent weights read k times."""
    g = json.load(open(GOLDEN))
    cfg = shaped_like_4b()
    prov = random_float_weights(cfg, 1)
    _, orc, _ = _run(cfg, prov, unit_rows(cfg, 5, 1), k, k_max=k)
    apps = g["depth_formula"]["constant"] + g["depth_formula"]["per_loop"] * k
    assert orc.sublayer_apps == apps == layer_applications(cfg, k)
    assert orc.sublayer_apps // 2 == 16 + 20 * k


def test_recurrent_weights_are_shared_across_loops():
    """[P5] Key ideas / [P4] looping at inference: the same weights serve every k —
    the set of weight blocks read is the 36 physical blocks for every k."""
    cfg = shaped_like_4b()
    base = random_float_weights(cfg, 2)
    for k in (1, 3):
        seen = []

        def prov(b):
            seen.append(b)
            return base(b)
        _run(cfg, prov, unit_rows(cfg, 4, 1), k, k_max=k)
        assert sorted(set(seen)) == list(range(36))
        rec_reads = [b for b in seen if block_role(cfg, b) == "recurrent"]
        assert len(rec_reads) == 2 * 20 * k    # attn + mlp read each recurrent block each loop


def test_loop_equals_unrolled_stack_with_reinjection():
    """[P1] Methodology: the input block's fixed output is re-injected before every pass
    of the shared block and the recurrent output is L2-normalised.  The looped forward
    equals an explicitly unrolled list of 8 + 20k + 8 tied blocks."""
    cfg = tiny()
    prov = random_float_weights(cfg, 5)
    h = unit_rows(cfg, 6, 24)
    k = 3
    out, _, _ = _run(cfg, prov, h, k, mode="per_loop", k_max=k)

    orc = Oracle(cfg, prov)
    cache = KVCache(cfg, "per_loop", k_max=k)
    n_in, n_rec = cfg["n_in_blocks"], cfg["n_rec_blocks"]
    program = [("blk", b, 1) for b in range(n_in)] + [("save_e",)]
    for j in range(1, k + 1):
        program += [("inject",)] + [("blk", b, j) for b in range(n_in, n_in + n_rec)]
    program += [("blk", b, 1) for b in range(n_in + n_rec, n_in + n_rec + cfg["n_out_blocks"])]
    x, e = h, None
    for op in program:
        if op[0] == "blk":
            x = orc.block(op[1], x, 0, 0, op[2], cache)
        elif op[0] == "save_e":
            e = x
        else:
            x = l2norm(x + e)
    np.testing.assert_allclose(out, x, rtol=0, atol=1e-13)
    # re-injection matters once k > 1: dropping it changes the result
    orc2 = Oracle(cfg, prov)
    c2 = KVCache(cfg, "per_loop", k_max=k)
    x = h
    for op in program:
        if op[0] == "blk":
            x = orc2.block(op[1], x, 0, 0, op[2], c2)
    assert np.abs(out - x).max() > 1e-3


# ---------------------------------------------------------------- KV modes

def test_kv_bytes_last_loop_constant_in_k():
    """[P1] Key Contributions 4 / [P4] KV cache modes: last-loop KV memory stays at its
    one-loop size for any k; per-loop memory grows with the loop count."""
    cfg = load_config("dory4b")
    one = kv_cache_bytes(cfg, "per_loop", 64, 32768, 1)
    for k in (1, 2, 3, 4, 8):
        assert kv_cache_bytes(cfg, "last_loop", 64, 32768, k) == one
    rec = sum(1 for b in range(36) if block_role(cfg, b) == "recurrent")
    assert rec == 20
    grow = kv_cache_bytes(cfg, "per_loop", 64, 32768, 2) - one
    # recurrent blocks: 15 SWA (4096 slots) + 5 full (32768 slots), 4096 B per slot
    assert grow == 64 * (15 * 4096 + 5 * 32768) * 4096
    # the 4B decode cache at 32768 positions: 9 full + 27 SWA layers
    assert one == 64 * (9 * 32768 + 27 * 4096) * 4096


def test_modes_identical_at_k1_and_on_fresh_single_call():
    """[P4] KV cache modes: with one loop there is one cache either way, so the two
    modes agree exactly; they can only differ once a later call reads entries an
    earlier call left (negative control at k = 2)."""
    cfg = tiny()
    prov = random_float_weights(cfg, 7)
    h = unit_rows(cfg, 8, 40)
    for k in (1, 2):
        a, _, ca = _run(cfg, prov, h[:24], k, mode="per_loop", k_max=k)
        b, _, cb = _run(cfg, prov, h[:24], k, mode="last_loop", k_max=k)
        assert np.array_equal(a, b)                      # fresh single call: identical
        for blk in range(8):
            ka, va = ca.read(blk, k, 0, 0, 24)
            kb, vb = cb.read(blk, k, 0, 0, 24)
            assert np.array_equal(ka, kb) and np.array_equal(va, vb)
        # second call (chunk 2) sees the first call's cache
        a2 = Oracle(cfg, prov).forward(h[24:], 24, k, ca)
        b2 = Oracle(cfg, prov).forward(h[24:], 24, k, cb)
        if k == 1:
            assert np.array_equal(a2, b2)
        else:
            assert np.abs(a2 - b2).max() > 1e-4


def test_last_loop_cache_holds_final_loop_entries():
    """[P5] Key ideas: in last_loop mode the cache holds only the final loop's keys and
    values — equal to per-loop caching's loop-k cache."""
    cfg = tiny()
    prov = random_float_weights(cfg, 9)
    h = unit_rows(cfg, 10, 16)
    _, _, cp = _run(cfg, prov, h, 3, mode="per_loop", k_max=3)
    _, _, cl = _run(cfg, prov, h, 3, mode="last_loop", k_max=3)
    for blk in range(2, 6):
        kl, vl = cl.read(blk, 1, 0, 0, 16)
        k3, v3 = cp.read(blk, 3, 0, 0, 16)
        k1, _ = cp.read(blk, 1, 0, 0, 16)
        assert np.array_equal(kl, k3) and np.array_equal(vl, v3)
        assert np.abs(kl - k1).max() > 1e-4


def test_chunked_prefill_equals_one_shot_per_loop():
    """Per-loop caching stores every loop's keys, so splitting a prefill into chunks
    changes nothing (each query still sees loop-j keys of all earlier positions)."""
    cfg = tiny()
    prov = random_float_weights(cfg, 11)
    h = unit_rows(cfg, 12, 100)
    one, _, _ = _run(cfg, prov, h, 2, mode="per_loop", k_max=2)
    cache = KVCache(cfg, "per_loop", k_max=2)
    orc = Oracle(cfg, prov)
    parts = [orc.forward(h[a:b], a, 2, cache) for a, b in ((0, 37), (37, 40), (40, 100))]
    np.testing.assert_allclose(np.concatenate(parts), one, rtol=0, atol=1e-12)


def test_prefix_rows_are_causal():
    """Causal attention: rows [0, m) of a T-token prefill equal the prefill of the first
    m tokens (both KV modes, any k).  Used to sample full-size outputs."""
    cfg = tiny()
    prov = random_float_weights(cfg, 13)
    h = unit_rows(cfg, 14, 90)
    for mode in ("per_loop", "last_loop"):
        full, _, _ = _run(cfg, prov, h, 2, mode=mode, k_max=2)
        pre, _, _ = _run(cfg, prov, h[:33], 2, mode=mode, k_max=2)
        np.testing.assert_allclose(full[:33], pre, rtol=0, atol=1e-12)


@pytest.mark.parametrize("k", [1, 2, 3])
def test_decode_after_prefill_equals_longer_prefill(k):
    """A decode step is a one-token call: under per-loop caching, prefill(T) then one
    decode step gives the last row of prefill(T + 1), for any loop count."""
    cfg = tiny()
    prov = random_float_weights(cfg, 15)
    h = unit_rows(cfg, 16, 51)
    ref, _, _ = _run(cfg, prov, h, k, mode="per_loop", k_max=3)
    cache = KVCache(cfg, "per_loop", k_max=3)
    orc = Oracle(cfg, prov)
    orc.forward(h[:50], 0, k, cache)
    step = orc.decode(h[50:51], [0], [50], k, cache)
    np.testing.assert_allclose(step[0], ref[50], rtol=0, atol=1e-12)


@pytest.mark.parametrize("mode", ["per_loop", "last_loop"])
def test_decode_rows_are_independent(mode):
    """Each row of a decode step attends only to its own sequence's cache: a batched
    step equals every row decoded alone.  (So a step may give each row its own loop
    count: the loop count is a per-request dial, [P5] Why it matters here.)"""
    cfg = tiny()
    prov = random_float_weights(cfg, 21)
    lens = [7, 30, 12]
    hs = [unit_rows(cfg, 30 + s, lens[s] + 1) for s in range(3)]
    runs = []
    for _ in range(2):
        cache = KVCache(cfg, mode, k_max=2)
        orc = Oracle(cfg, prov)
        for s in range(3):
            orc.forward(hs[s][:lens[s]], 0, 2, cache, seq=s)
        runs.append((orc, cache))
    rows = np.stack([hs[s][lens[s]] for s in range(3)])
    orc, cache = runs[0]
    batched = orc.decode(rows, [0, 1, 2], lens, 2, cache)
    orc, cache = runs[1]
    single = np.stack([orc.decode(rows[s:s + 1], [s], [lens[s]], 2, cache)[0] for s in range(3)])
    np.testing.assert_allclose(batched, single, rtol=0, atol=1e-12)
    # and the rows really differ (a step that ignored its sequence would not)
    assert np.abs(batched[0] - batched[1]).max() > 1e-3


def test_unwritten_reads_raise():
    cfg = tiny()
    cache = KVCache(cfg, "last_loop")
    with pytest.raises(KeyError):
        Oracle(cfg, random_float_weights(cfg, 1)).forward(unit_rows(cfg, 1, 2), 5, 1, cache)


# ---------------------------------------------------------------- nGPT update

def test_ngpt_update_closed_forms():
    """[P1] Methodology, nGPT residual: h <- Norm(h + alpha (Norm(y) - h)).
    alpha = 0.5 between orthogonal unit vectors gives their normalised midpoint;
    alpha = 1 gives Norm(y); alpha = 0 gives h."""
    orc = Oracle(tiny(), None)
    h = np.array([[1.0, 0.0, 0.0]])
    y = np.array([[0.0, 5.0, 0.0]])
    out = orc._ngpt_update(h, y, np.full(3, 0.5))
    np.testing.assert_allclose(out, [[math.sqrt(0.5), math.sqrt(0.5), 0.0]], atol=1e-15)
    out = orc._ngpt_update(h, np.array([[0.0, -2.0, 2.0]]), np.ones(3))
    np.testing.assert_allclose(out, [[0.0, -math.sqrt(0.5), math.sqrt(0.5)]], atol=1e-15)
    out = orc._ngpt_update(h, y, np.array([0.0, 1.0, 1.0]))   # per-channel alpha
    np.testing.assert_allclose(out, [[math.sqrt(0.5), math.sqrt(0.5), 0.0]], atol=1e-15)


def test_every_state_on_unit_sphere():
    """[P1] Methodology: everything is L2-normalised — every post-sublayer state has
    unit norm (to 1e-5, here to float64 rounding)."""
    cfg = tiny()
    worst = [0.0]

    def hook(h):
        worst[0] = max(worst[0], float(np.abs(np.linalg.norm(h, axis=1) - 1).max()))
    _run(cfg, random_float_weights(cfg, 17), unit_rows(cfg, 18, 64), 3, k_max=3, on_state=hook)
    assert worst[0] < 1e-12


def test_alpha_zero_is_identity():
    """alpha = 0 freezes the stream: h_out = Norm(h_in) (re-injection gives Norm(2e) = e)."""
    cfg = tiny()
    h = unit_rows(cfg, 19, 20)
    out, _, _ = _run(cfg, random_float_weights(cfg, 20, alpha=0.0), h, 2, k_max=2)
    np.testing.assert_allclose(out, l2norm(h), rtol=0, atol=1e-14)


def test_alpha_one_outputs_normalised_sublayer():
    """alpha = 1: the sublayer returns Norm(f(h)), a unit vector; with W_gate = 0 the MLP
    output f(h) is zero and the update keeps only the (1 - alpha)-shrunk stream."""
    cfg = tiny()
    prov = random_float_weights(cfg, 21, alpha=1.0)
    orc = Oracle(cfg, prov)
    h = unit_rows(cfg, 22, 4)
    out = orc.mlp_sublayer(0, h)
    assert np.abs(np.linalg.norm(out, axis=1) - 1).max() < 1e-14
    # W_gate = 0: SiLU(0) = 0, so f(h) = 0, Norm(0) = 0 and the update leaves
    # Norm((1 - alpha) * h), the stream shrunk channel-wise and renormalised.
    base = random_float_weights(cfg, 23)
    zero_gate = modified(base, lambda b, w: w["w_gate"].fill(0.0))
    alpha = base(0)["alpha_mlp"]
    np.testing.assert_allclose(Oracle(cfg, zero_gate).mlp_sublayer(0, l2norm(h)),
                               l2norm((1 - alpha) * l2norm(h)), atol=1e-15)


# ---------------------------------------------------------------- norm placement

@pytest.mark.parametrize("name,invariant", [
    ("wq", True), ("wk", True), ("wv", True), ("wo", True), ("w_up", True), ("w_down", True),
    ("w_gate", False), ("wg", False),
])
def test_scale_invariances(name, invariant):
    """[P1] Methodology: q/k are L2-normalised per head (nGPT QK norm), the gated
    attention output and the SwiGLU activations are L2-normalised before their
    projections, and every sublayer output is normalised inside the update.  So
    scaling Wq, Wk, Wv, Wo, W_up or W_down by c > 0 changes nothing, while the
    nonlinear gate paths (W_gate of SwiGLU, the attention gate Wg) do change."""
    cfg = tiny()
    base = random_float_weights(cfg, 24)
    h = unit_rows(cfg, 25, 40)
    ref, _, _ = _run(cfg, base, h, 2, k_max=2)
    scaled = modified(base, lambda b, w: w.__setitem__(name, w[name] * 3.7))
    out, _, _ = _run(cfg, scaled, h, 2, k_max=2)
    err = np.abs(out - ref).max()
    if invariant:
        assert err < 1e-12
    else:
        assert err > 1e-4


# ---------------------------------------------------------------- attention

def test_swa_equals_full_when_window_covers_sequence():
    """[P1] Methodology: sliding-window attention is causal attention restricted to the
    last W keys; with W >= T it is full causal attention (negative control: W < T)."""
    h = unit_rows(tiny(), 26, 64)
    prov = random_float_weights(tiny(), 27)
    full_only, _, _ = _run(tiny(full_period=1), prov, h, 2, k_max=2)
    wide, _, _ = _run(tiny(window=64), prov, h, 2, k_max=2)
    narrow, _, _ = _run(tiny(window=16), prov, h, 2, k_max=2)
    assert np.array_equal(full_only, wide)
    assert np.abs(full_only - narrow).max() > 1e-4


def test_gqa_equals_mha_with_repeated_kv_heads():
    """[P1] Methodology: grouped-query attention — query head h reads KV head
    floor(h / (Hq/Hkv)).  Equal to multi-head attention whose K/V weights repeat
    each KV head for its group."""
    cfg = tiny()
    group = cfg["n_q_heads"] // cfg["n_kv_heads"]
    hd = cfg["head_dim"]
    gqa = random_float_weights(cfg, 28)

    def rep(b, w):
        for nm in ("wk", "wv"):
            heads = w[nm].reshape(cfg["n_kv_heads"], hd, -1)
            w[nm] = np.repeat(heads, group, axis=0).reshape(cfg["n_q_heads"] * hd, -1)
    mha_cfg = tiny(n_kv_heads=cfg["n_q_heads"])
    mha = modified(gqa, rep)
    h = unit_rows(cfg, 29, 50)
    a, _, _ = _run(cfg, gqa, h, 2, k_max=2)
    b, _, _ = _run(mha_cfg, mha, h, 2, k_max=2)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)


def test_rope_closed_forms():
    """RoPE (pages: RoPE with base 1e4 / 1e7): position 0 is the identity; a basis vector
    e_i rotates into e_{i+hd/2} by angle p * base^(-2i/hd); dot products depend only
    on the position difference."""
    x = np.random.default_rng(0).standard_normal((3, 2, 64))
    np.testing.assert_array_equal(rope(x, [0, 0, 0], 1e4), x)
    e0 = np.zeros((1, 1, 64)); e0[0, 0, 0] = 1.0
    r = rope(e0, [1], 1e4)[0, 0]
    assert abs(r[0] - 0.5403023058681398) < 1e-15 and abs(r[32] - 0.8414709848078965) < 1e-15
    e31 = np.zeros((1, 1, 64)); e31[0, 0, 31] = 1.0
    r = rope(e31, [1000], 1e4)[0, 0]
    ang = 1000 * 10000.0 ** (-62.0 / 64.0)           # = 1000 / 10000^(31/32)
    assert abs(ang - 0.1333521432163324) < 1e-15
    assert abs(r[31] - math.cos(ang)) < 1e-15 and abs(r[63] - math.sin(ang)) < 1e-15
    q, k = x[0:1], x[1:2]
    d1 = np.sum(rope(q, [7], 1e7) * rope(k, [3], 1e7))
    d2 = np.sum(rope(q, [1004], 1e7) * rope(k, [1000], 1e7))
    assert abs(d1 - d2) < 1e-12


def _brute_attention_sublayer(cfg, w, h, pos0, prev_k, prev_v, full=False):
    """Loop-by-loop restatement of one gated GQA attention sublayer for a fresh
    (pos0 = 0, prev empty) or continued call; pure Python floats."""
    d, hq, hkv, hd = cfg["d_model"], cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    n = len(h)
    half = hd // 2

    def matvec(m, x):
        return [sum(m[r][c] * x[c] for c in range(len(x))) for r in range(len(m))]

    def unit(v):
        s = math.sqrt(sum(t * t for t in v))
        return [t / s for t in v]

    def rot(v, p, base):
        out = [0.0] * hd
        for i in range(half):
            a = p * base ** (-2.0 * i / hd)
            out[i] = v[i] * math.cos(a) - v[i + half] * math.sin(a)
            out[i + half] = v[i + half] * math.cos(a) + v[i] * math.sin(a)
        return out

    base = cfg["rope_base_full"] if full else cfg["rope_base_swa"]
    keys, vals = list(prev_k), list(prev_v)
    qs, gates = [], []
    for t in range(n):
        p = pos0 + t
        qf, kf, vf = matvec(w["wq"], h[t]), matvec(w["wk"], h[t]), matvec(w["wv"], h[t])
        g = [1.0 / (1.0 + math.exp(-z)) for z in matvec(w["wg"], h[t])]
        qh = [[w["s_qk"][i] * z for i, z in enumerate(unit(rot(qf[j * hd:(j + 1) * hd], p, base)))]
              for j in range(hq)]
        kh = [[w["s_qk"][i] * z for i, z in enumerate(unit(rot(kf[j * hd:(j + 1) * hd], p, base)))]
              for j in range(hkv)]
        vh = [vf[j * hd:(j + 1) * hd] for j in range(hkv)]
        keys.append(kh); vals.append(vh); qs.append(qh); gates.append(g)
    outs = []
    for t in range(n):
        p = pos0 + t
        o = []
        for j in range(hq):
            kv = j // (hq // hkv)
            allowed = [s for s in range(p + 1) if full or p - s < cfg["window"]]
            logits = [cfg["softmax_scale"] * sum(a * b for a, b in zip(qs[t][j], keys[s][kv]))
                      for s in allowed]
            m = max(logits)
            ex = [math.exp(z - m) for z in logits]
            tot = sum(ex)
            acc = [0.0] * hd
            for e_, s in zip(ex, allowed):
                for i in range(hd):
                    acc[i] += e_ / tot * vals[s][kv][i]
            o.extend(gates[t][j] * z for z in acc)
        y = matvec(w["wo"], unit(o))
        yn = unit(y)
        u = [h[t][i] + w["alpha_attn"][i] * (yn[i] - h[t][i]) for i in range(d)]
        outs.append(unit(u))
    return outs


def test_attention_sublayer_brute_force():
    """Brute-force restatement (Python loops, math.exp) of the gated GQA sliding-window
    attention sublayer on a micro model, over two calls (second call reads the cache)."""
    cfg = micro()
    prov = random_float_weights(cfg, 30)
    w = {k: v.tolist() for k, v in prov(0).items()}
    h = l2norm(np.random.default_rng(31).standard_normal((5, cfg["d_model"])))
    orc = Oracle(cfg, prov)
    cache = KVCache(cfg, "last_loop")
    got1 = orc.attention_sublayer(0, h[:3], 0, 0, 1, cache)
    got2 = orc.attention_sublayer(0, h[3:], 3, 0, 1, cache)
    want = _brute_attention_sublayer(cfg, w, h.tolist(), 0, [], [])
    np.testing.assert_allclose(np.concatenate([got1, got2]), np.array(want), rtol=0, atol=1e-13)


def test_full_layer_brute_force_uses_full_base_and_no_window():
    """[P1] Methodology: full-attention layers see every earlier key and use their own
    RoPE base (1e7), unlike the SWA layers (window W, base 1e4)."""
    cfg = micro(rope_base_full=1e7)
    prov = random_float_weights(cfg, 36)
    w = {k: v.tolist() for k, v in prov(1).items()}      # block 1 is a full layer
    assert is_full_layer(cfg, 1) and not is_full_layer(cfg, 0)
    h = l2norm(np.random.default_rng(37).standard_normal((5, cfg["d_model"])))
    got = Oracle(cfg, prov).attention_sublayer(1, h, 0, 0, 1, KVCache(cfg, "last_loop"))
    want = _brute_attention_sublayer(cfg, w, h.tolist(), 0, [], [], full=True)
    np.testing.assert_allclose(got, np.array(want), rtol=0, atol=1e-13)
    swa_like = _brute_attention_sublayer(cfg, w, h.tolist(), 0, [], [], full=False)
    assert np.abs(np.array(swa_like) - got).max() > 1e-6


def test_mlp_sublayer_brute_force():
    """Brute-force SwiGLU sublayer: a_i = SiLU(gate_scale * g_i) * u_i, Norm(a) before the
    down-projection, then the nGPT update (Python loops)."""
    cfg = micro(gate_scale=1.7)
    prov = random_float_weights(cfg, 32)
    w = {k: v.tolist() for k, v in prov(0).items()}
    h = l2norm(np.random.default_rng(33).standard_normal((3, cfg["d_model"])))
    got = Oracle(cfg, prov).mlp_sublayer(0, h)
    for t in range(3):
        x = h[t].tolist()
        a = []
        for r in range(cfg["d_ff"]):
            g = 1.7 * sum(w["w_gate"][r][c] * x[c] for c in range(cfg["d_model"]))
            u = sum(w["w_up"][r][c] * x[c] for c in range(cfg["d_model"]))
            a.append(g / (1.0 + math.exp(-g)) * u)
        na = math.sqrt(sum(z * z for z in a))
        y = [sum(w["w_down"][r][c] * a[c] / na for c in range(cfg["d_ff"])) for r in range(cfg["d_model"])]
        ny = math.sqrt(sum(z * z for z in y))
        u = [x[i] + w["alpha_mlp"][i] * (y[i] / ny - x[i]) for i in range(cfg["d_model"])]
        nu = math.sqrt(sum(z * z for z in u))
        np.testing.assert_allclose(got[t], [z / nu for z in u], rtol=0, atol=1e-14)


def test_window_one_attends_to_self_only():
    """W = 1: softmax over the single visible key is 1, so the attention sublayer does
    not depend on any other token (changing earlier tokens leaves row t unchanged)."""
    cfg = micro(window=1, full_period=1000)
    prov = random_float_weights(cfg, 34)
    rng = np.random.default_rng(35)
    h = l2norm(rng.standard_normal((6, cfg["d_model"])))
    h2 = h.copy()
    h2[:5] = l2norm(rng.standard_normal((5, cfg["d_model"])))
    a = Oracle(cfg, prov).attention_sublayer(0, h, 0, 0, 1, KVCache(cfg, "last_loop"))
    b = Oracle(cfg, prov).attention_sublayer(0, h2, 0, 0, 1, KVCache(cfg, "last_loop"))
    np.testing.assert_allclose(a[5], b[5], atol=1e-15)
    assert np.abs(a[4] - b[4]).max() > 1e-6


def test_generator_weights_are_bf16_and_unit_rows():
    cfg = tiny()
    from synthetic import bf16_bits_to_f32
    w = weights_from_generator(cfg, 0)(3)
    for name in ("wq", "wk", "wv", "wg", "wo", "w_gate", "w_up", "w_down"):
        m = bf16_bits_to_f32(w[name]).astype(np.float64)
        assert np.abs(np.linalg.norm(m, axis=1) - 1).max() < 1e-2
    assert np.all(w["alpha_attn"] == np.float32(0.05)) and np.all(w["s_qk"] == 1)


# ---------------------------------------------------------------- pre-filled caches

def _prefill_values(cfg):
    """Deterministic K/V contents per (slot, seq, position), independent of how a
    range is requested (so a range read equals the same positions read one by one).
    float32 values: the cache holds filled entries in float32, as the GPU caches'
    bf16 contents are."""
    hkv, hd = cfg["n_kv_heads"], cfg["head_dim"]

    def pre(slot, seq, lo, hi):
        ks, vs = [], []
        for p in range(lo, hi):
            r = np.random.default_rng([slot, seq, p, 99])
            ks.append(r.standard_normal((hkv, hd)).astype(np.float32))
            vs.append(r.standard_normal((hkv, hd)).astype(np.float32))
        shape = (0, hkv, hd)
        return (np.stack(ks) if ks else np.zeros(shape)), (np.stack(vs) if vs else np.zeros(shape))
    return pre


@pytest.mark.parametrize("mode", ["per_loop", "last_loop"])
def test_prefilled_cache_equals_explicit_writes(mode):
    """The decode workloads start from caches whose earlier positions come from a
    fill callback instead of earlier calls.  A cache filled that way must read back
    exactly like a cache into which the same values were written explicitly: the
    last W positions of a sliding-window layer, every position of a full layer, in
    every loop slot, and a position rewritten after the fill returns the new value
    ([P4] How does looping work at inference time?: each cache keeps a layer's
    keys/values; SWA layers keep the last W positions)."""
    cfg = tiny()                      # W = 32, blocks alternate SWA / full
    W, k = cfg["window"], 2
    lens = {0: 70, 1: 40}             # seq 0 beyond the window, seq 1 partly
    pre = _prefill_values(cfg)
    filled = KVCache(cfg, mode, k_max=k, prefill=pre, prefilled_len=lens)
    written = KVCache(cfg, mode, k_max=k)
    for slot in written.slot_ids():
        b, loop = slot // 16, slot % 16 + 1
        for seq, n in lens.items():
            lo = 0 if is_full_layer(cfg, b) else max(0, n - W)
            K, V = pre(slot, seq, lo, n)
            written.write(b, loop, seq, lo, K, V)
    assert is_full_layer(cfg, 1) and not is_full_layer(cfg, 2)
    loops = (1, 2) if mode == "per_loop" else (1,)
    for b in (0, 1, 2, 3):            # input SWA, input full, recurrent SWA, recurrent full
        for loop in (loops if block_role(cfg, b) == "recurrent" else (1,)):
            for seq, n in lens.items():
                ranges = ([(0, n), (5, n - 3), (n - 1, n)] if is_full_layer(cfg, b)
                          else [(max(0, n - W), n), (max(0, n - W) + 4, n - 2)])
                for lo, hi in ranges:
                    ka, va = filled.read(b, loop, seq, lo, hi)
                    kb, vb = written.read(b, loop, seq, lo, hi)
                    assert np.array_equal(ka, kb) and np.array_equal(va, vb), (b, loop, seq, lo)
    # a continued call (both modes write and read within the call) and decode steps
    prov = random_float_weights(cfg, 40)
    h = unit_rows(cfg, 41, 9)
    outs = []
    for cache in (filled, written):
        orc = Oracle(cfg, prov)
        o1 = orc.forward(h[:6], lens[0], k, cache, seq=0)
        o2 = orc.decode(h[6:8], [0, 1], [lens[0] + 6, lens[1]], k, cache)
        outs.append(np.concatenate([o1, o2]))
    assert np.array_equal(outs[0], outs[1])
    # a position inside the filled range rewritten afterwards reads back the new value
    newk = np.full((1, cfg["n_kv_heads"], cfg["head_dim"]), 0.25)
    newv = np.full_like(newk, -0.5)
    for cache in (filled, written):
        cache.write(2, 1, 1, lens[1] - 3, newk, newv)
        cache.write(1, 1, 1, 7, newk, newv)
    for b, lo, hi in ((2, lens[1] - W + 8, lens[1]), (1, 0, lens[1])):
        ka, va = filled.read(b, 1, 1, lo, hi)
        kb, vb = written.read(b, 1, 1, lo, hi)
        assert np.array_equal(ka, kb) and np.array_equal(va, vb)
    ka, va = filled.read(2, 1, 1, lens[1] - 3, lens[1] - 2)
    assert np.all(ka == 0.25) and np.all(va == -0.5)
    # negative control: a fill that ignores the sequence index reads differently
    wrong = KVCache(cfg, mode, k_max=k, prefill=lambda s, q, lo, hi: pre(s, 0, lo, hi),
                    prefilled_len=lens)
    kw, _ = wrong.read(1, 1, 1, 0, lens[1])
    kb, _ = written.read(1, 1, 1, 0, lens[1])
    assert not np.array_equal(kw[:7], kb[:7])


# ---------------------------------------------------------------- output gate

def _gate_inputs(cfg, w_dir, n, seed):
    """Rows h = Norm(w_dir + noise) with h . w_dir >= 0.5 for every row."""
    rng = np.random.default_rng(seed)
    h = l2norm(w_dir[None, :] + 0.25 * rng.standard_normal((n, cfg["d_model"]))
               / np.sqrt(cfg["d_model"]))
    assert (h @ w_dir).min() > 0.5
    return h


def test_gate_equal_across_heads_is_removed_by_the_output_norm():
    """[P1] Methodology: the sigmoid output gates multiply each head's output, and the
    concatenated gated output is L2-normalised before the output projection.  When
    every head of a token gets the same gate value, the gate is a per-token uniform
    scale that the norm removes: the sublayer equals the one with W_g = 0 (all gates
    1/2).  A gate read for the wrong token would break this."""
    cfg = tiny()
    base = random_float_weights(cfg, 42)
    w_dir = l2norm(np.random.default_rng(43).standard_normal(cfg["d_model"]))
    same = modified(base, lambda b, w: w.__setitem__("wg", np.tile(3.0 * w_dir, (cfg["n_q_heads"], 1))))
    zero = modified(base, lambda b, w: w["wg"].fill(0.0))
    h = unit_rows(cfg, 44, 40)
    for layer in (0, 1):
        a = Oracle(cfg, same).attention_sublayer(layer, h, 0, 0, 1, KVCache(cfg, "last_loop"))
        z = Oracle(cfg, zero).attention_sublayer(layer, h, 0, 0, 1, KVCache(cfg, "last_loop"))
        np.testing.assert_allclose(a, z, rtol=0, atol=1e-13)


@pytest.mark.parametrize("head", [0, 1, 2, 3])
def test_one_hot_gate_selects_that_head(head):
    """[P1] Methodology: head j's output is scaled by sigmoid(h . W_g[j]).  With
    W_g[j] = +c u and every other row -c u, on inputs with h . u >= 1/2 and c = 400,
    head j's gate is 1 and the others are below e^-200: the sublayer keeps head j's
    attention output alone.  Because the output norm and the nGPT update see only
    the direction of y = Norm(o) W_o^T, that equals the W_g = 0 sublayer whose W_o
    keeps only head j's columns.  A gate applied to the wrong head, or sigmoid(-x),
    fails it."""
    cfg = tiny()
    hq, hd = cfg["n_q_heads"], cfg["head_dim"]
    base = random_float_weights(cfg, 45)
    u = l2norm(np.random.default_rng(46).standard_normal(cfg["d_model"]))

    def one_hot(b, w):
        g = np.tile(-400.0 * u, (hq, 1))
        g[head] = 400.0 * u
        w["wg"] = g

    def only_head(b, w):
        w["wg"].fill(0.0)
        keep = np.zeros(hq * hd)
        keep[head * hd:(head + 1) * hd] = 1.0
        w["wo"] = w["wo"] * keep[None, :]
    h = _gate_inputs(cfg, u, 24, 47)
    for layer in (0, 1):
        a = Oracle(cfg, modified(base, one_hot)).attention_sublayer(
            layer, h, 0, 0, 1, KVCache(cfg, "last_loop"))
        b = Oracle(cfg, modified(base, only_head)).attention_sublayer(
            layer, h, 0, 0, 1, KVCache(cfg, "last_loop"))
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
        # and the choice of head matters
        other = (head + 1) % hq

        def only_other(bb, w, other=other):
            w["wg"].fill(0.0)
            keep = np.zeros(hq * hd)
            keep[other * hd:(other + 1) * hd] = 1.0
            w["wo"] = w["wo"] * keep[None, :]
        c = Oracle(cfg, modified(base, only_other)).attention_sublayer(
            layer, h, 0, 0, 1, KVCache(cfg, "last_loop"))
        assert np.abs(a - c).max() > 1e-4


def test_mask_rule_closed_forms():
    """[P1] Methodology: causal attention, sliding-window layers see the last W
    positions including the query's own.  Visible keys of query q: [max(0, q-W+1), q]
    (W keys once q >= W - 1) for a window, [0, q] for a full layer."""
    from oracle import mask_allows
    for W in (1, 2, 4, 7):
        for q in range(12):
            vis = [j for j in range(20) if mask_allows(q, j, W)]
            assert vis == list(range(max(0, q - W + 1), q + 1))
            assert len(vis) == min(q + 1, W)
    assert [j for j in range(20) if mask_allows(9, j)] == list(range(10))
    grid = mask_allows(np.arange(6)[:, None], np.arange(6)[None, :], 2)
    assert np.array_equal(grid, np.tril(np.ones((6, 6), bool)) & ~np.tril(np.ones((6, 6), bool), -2))
