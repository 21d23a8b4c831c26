"""Helpers for the oracle tests: small configs and weight providers (no method arithmetic)."""

import copy

import numpy as np

from synthetic import load_config, bf16_bits_to_f32, hidden_in


def tiny(**over):
    return load_config("tiny", **over)


def shaped_like_4b(**over):
    """The 4B block structure (8/20/8 blocks, 3:1 SWA:full) with toy widths."""
    cfg = load_config("dory4b")
    cfg.update(d_model=64, n_q_heads=2, n_kv_heads=1, head_dim=32, d_ff=128, window=8,
               softmax_scale=float(np.sqrt(32)))
    cfg.update(over)
    return cfg


def micro(**over):
    cfg = load_config("tiny")
    cfg.update(d_model=8, n_q_heads=2, n_kv_heads=1, head_dim=4, d_ff=12,
               n_in_blocks=1, n_rec_blocks=1, n_out_blocks=1, window=2, full_period=2,
               softmax_scale=2.0)
    cfg.update(over)
    return cfg


def random_float_weights(cfg, seed, alpha=None, s_qk_random=True):
    """Provider b -> dict of float64 arrays (not bf16-rounded; for pure-oracle tests)."""
    d, hq, hkv, hd, ff = (cfg["d_model"], cfg["n_q_heads"], cfg["n_kv_heads"],
                          cfg["head_dim"], cfg["d_ff"])
    shapes = {"wq": (hq * hd, d), "wk": (hkv * hd, d), "wv": (hkv * hd, d), "wg": (hq, d),
              "wo": (d, hq * hd), "w_gate": (ff, d), "w_up": (ff, d), "w_down": (d, ff)}
    memo = {}

    def provide(b):
        if b not in memo:
            r = np.random.default_rng([seed, b])
            w = {n: r.standard_normal(s) / np.sqrt(s[1]) for n, s in shapes.items()}
            w["alpha_attn"] = (r.uniform(0.03, 0.3, d) if alpha is None else np.full(d, alpha))
            w["alpha_mlp"] = (r.uniform(0.03, 0.3, d) if alpha is None else np.full(d, alpha))
            w["s_qk"] = r.uniform(0.5, 1.5, hd) if s_qk_random else np.ones(hd)
            memo[b] = w
        return memo[b]
    return provide


def modified(provider, fn):
    """Provider whose blocks are deep-copied and passed through fn(b, w)."""
    memo = {}

    def provide(b):
        if b not in memo:
            w = copy.deepcopy(provider(b))
            w = {k: (bf16_bits_to_f32(v).astype(np.float64) if v.dtype == np.uint16 else
                     np.asarray(v, np.float64)) for k, v in w.items()}
            fn(b, w)
            memo[b] = w
        return memo[b]
    return provide


def unit_rows(cfg, seed, n):
    return bf16_bits_to_f32(hidden_in(cfg, seed, n)).astype(np.float64)
