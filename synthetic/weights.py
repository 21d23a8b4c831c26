"""Seeded synthetic weights and input hidden states.

Recipe (the configs' data description):
  * every projection matrix [out, in] is drawn i.i.d. N(0, weight_std), each row
    is scaled to unit L2 norm over `in` (nGPT-style row normalisation of the
    stored matrix), then rounded to bfloat16 (RNE).  The oracle uses these
    bf16 values exactly, so weight quantisation is not part of parity error;
  * alpha vectors are `alpha_init` per dimension ("default") or U(0.03, 0.07)
    per dimension ("random", used by tests to catch indexing errors);
  * the per-head-dimension query/key scale s_qk is 1 ("default") or
    U(0.5, 1.5) ("random");
  * input hidden states are N(0, 1) rows scaled to unit L2 norm, then rounded
    to bf16.

Draws are keyed by (seed, block, tensor, row chunk), so results do not depend
on thread count or on how many rows are requested.
"""

from concurrent.futures import ThreadPoolExecutor
import os

import numpy as np

from .bf16 import f32_to_bf16_bits

_ROW_CHUNK = 256
_TENSOR_IDS = {
    "wq": 1, "wk": 2, "wv": 3, "wg": 4, "wo": 5,
    "w_gate": 6, "w_up": 7, "w_down": 8,
    "alpha_attn": 9, "alpha_mlp": 10, "s_qk": 11,
    "emb_in": 12, "emb_out": 13, "logit_scale": 14,
}
MATRICES = ("wq", "wk", "wv", "wg", "wo", "w_gate", "w_up", "w_down")
VECTORS = ("alpha_attn", "alpha_mlp", "s_qk")

_POOL = None


def _pool():
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max(1, min(32, os.cpu_count() or 1)))
    return _POOL


def _rng(*key):
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) for k in key])))


def matrix_shapes(cfg):
    d, hq, hkv, hd, ff = (cfg["d_model"], cfg["n_q_heads"], cfg["n_kv_heads"],
                          cfg["head_dim"], cfg["d_ff"])
    return {
        "wq": (hq * hd, d), "wk": (hkv * hd, d), "wv": (hkv * hd, d), "wg": (hq, d),
        "wo": (d, hq * hd), "w_gate": (ff, d), "w_up": (ff, d), "w_down": (d, ff),
    }


def _matrix_chunk(seed, block, tid, chunk, rows, cols, std):
    z = _rng(seed, block, tid, chunk).standard_normal((rows, cols), dtype=np.float32)
    z *= np.float32(std)
    nrm = np.sqrt(np.einsum("ij,ij->i", z.astype(np.float64), z.astype(np.float64)))
    z = (z / nrm[:, None]).astype(np.float32)
    return f32_to_bf16_bits(z)


def _matrix(seed, block, name, shape, std):
    rows, cols = shape
    tid = _TENSOR_IDS[name]
    starts = list(range(0, rows, _ROW_CHUNK))
    parts = list(_pool().map(
        lambda c: _matrix_chunk(seed, block, tid, c // _ROW_CHUNK,
                                min(_ROW_CHUNK, rows - c), cols, std), starts))
    return np.concatenate(parts, axis=0)


def block_weights(cfg, seed, block, variant="default", names=None):
    """Weights of one transformer block (global block index `block`).

    Returns a dict: matrices as uint16 bf16 bit patterns of shape [out, in]
    (wq [Hq*hd, d], wk/wv [Hkv*hd, d], wg [Hq, d], wo [d, Hq*hd],
    w_gate/w_up [d_ff, d], w_down [d, d_ff]); vectors as float32
    (alpha_attn [d], alpha_mlp [d], s_qk [hd]).
    """
    shapes = matrix_shapes(cfg)
    names = names or (MATRICES + VECTORS)
    out = {}
    for name in names:
        if name in shapes:
            out[name] = _matrix(seed, block, name, shapes[name], cfg["weight_std"])
        elif name in ("alpha_attn", "alpha_mlp"):
            n = cfg["d_model"]
            if variant == "random":
                out[name] = _rng(seed, block, _TENSOR_IDS[name]).uniform(0.03, 0.07, n).astype(np.float32)
            else:
                out[name] = np.full(n, cfg["alpha_init"], dtype=np.float32)
        elif name == "s_qk":
            n = cfg["head_dim"]
            if variant == "random":
                out[name] = _rng(seed, block, _TENSOR_IDS[name]).uniform(0.5, 1.5, n).astype(np.float32)
            else:
                out[name] = np.ones(n, dtype=np.float32)
        else:
            raise KeyError(name)
    return out


def hidden_in(cfg, seed, n, row0=0):
    """Rows [row0, row0+n) of the seeded unit-norm input stream, as uint16 bf16 bits [n, d]."""
    d = cfg["d_model"]
    if n == 0:
        return np.zeros((0, d), dtype=np.uint16)
    c0, c1 = row0 // _ROW_CHUNK, (row0 + n - 1) // _ROW_CHUNK
    parts = []
    for c in range(c0, c1 + 1):
        z = _rng(seed, 0xD0, c).standard_normal((_ROW_CHUNK, d)).astype(np.float64)
        z /= np.sqrt((z * z).sum(axis=1, keepdims=True))
        parts.append(f32_to_bf16_bits(z.astype(np.float32)))
    allrows = np.concatenate(parts, axis=0)
    off = row0 - c0 * _ROW_CHUNK
    return np.ascontiguousarray(allrows[off:off + n])


def vocab_weights(cfg, seed, vocab=None):
    """Token embedding tables around the stack (the vocabulary size is not on the
    pages: `vocab_size` of the config): emb_in, emb_out [V, d] as bf16 bits with
    N(0, weight_std) rows scaled to unit norm (as the block matrices), and
    logit_scale [V] float32 drawn U(10, 20)."""
    V = int(vocab or cfg["vocab_size"])
    d = cfg["d_model"]
    out = {name: _matrix(seed, 0xE0, name, (V, d), cfg["weight_std"])
           for name in ("emb_in", "emb_out")}
    out["logit_scale"] = _rng(seed, 0xE0, _TENSOR_IDS["logit_scale"]).uniform(10.0, 20.0, V).astype(np.float32)
    return out
