"""Embedding lookup, LM head and sampling around the looped stack (oracle side).

TEST INFRASTRUCTURE ONLY, like the rest of `oracle/`: only `tests/`,
`__graft_entry__.smoke()` and the CPU legs of `bench.py` may use it.

The pages describe the model only between the first and last hidden states
("Dory1.0-4B: A Looped Normalized-GPT", Overview: a 4B-parameter language
model; no vocabulary size, no head).  The plainest reading for the nGPT
backbone the card cites ("NVIDIA Nemotron Labs Dory 1.0 4B ...", Key ideas,
nGPT: every vector on the unit sphere):
  * embedding: the token's row of the input table, L2-normalised, is the
    stack's unit-norm input h_in;
  * LM head: logits z_v = s_z[v] * (E_out[v] . h) with unit-norm output rows
    and a learned per-token scale s_z (nGPT's logit scaling);
  * sampling: temperature T = 0 takes argmax_v z_v (the lowest index on a
    tie); T > 0 draws by the Gumbel-max rule, argmax_v z_v / T + G_v with
    G_v = -log(-log U_v), which samples softmax(z / T).  U_v comes from a
    counter-based hash of (seed, the row's step counter, v), so a sample is a
    pure function of its inputs; the hash is lowbias32 (C. Wellons,
    "Prospecting for Hash Functions", 2018: xorshift 16, multiply 0x7feb352d,
    xorshift 15, multiply 0x846ca68b, xorshift 16), written out below.
The vocabulary size is a config value (`vocab_size`), an assumption.
"""

import numpy as np

_M32 = 0xFFFFFFFF


def lowbias32(x):
    """The lowbias32 integer hash on uint64 arrays holding 32-bit values."""
    x = np.asarray(x, dtype=np.uint64) & _M32
    x ^= x >> np.uint64(16)
    x = (x * np.uint64(0x7FEB352D)) & _M32
    x ^= x >> np.uint64(15)
    x = (x * np.uint64(0x846CA68B)) & _M32
    x ^= x >> np.uint64(16)
    return x


def uniform(seed, step, v):
    """U in (0, 1) of (seed, step, token v): (h + 0.5) / 2^32 with
    h = H(H(H(seed) ^ step) ^ v), H = lowbias32."""
    h = lowbias32(lowbias32(lowbias32(np.uint64(seed)) ^ np.uint64(step)) ^ np.asarray(v, np.uint64))
    return (h.astype(np.float64) + 0.5) / 4294967296.0


def embed(emb_in, tokens):
    """h_in rows: Norm(E_in[token]) in float64."""
    rows = np.asarray(emb_in, dtype=np.float64)[np.asarray(tokens)]
    return rows / np.sqrt(np.maximum((rows * rows).sum(axis=1, keepdims=True), 1e-20))


def lm_head(emb_out, logit_scale, h):
    """z = s_z * (h E_out^T) in float64: [n, V]."""
    return np.asarray(h, np.float64) @ np.asarray(emb_out, np.float64).T * \
        np.asarray(logit_scale, np.float64)[None, :]


def sample(z, temperature, seed, steps):
    """One token per row of z [n, V]: greedy at T = 0, else Gumbel-max with the
    row's step counter steps[i].  Computed in float64."""
    z = np.asarray(z, dtype=np.float64)
    n, V = z.shape
    out = np.empty(n, dtype=np.int64)
    v = np.arange(V, dtype=np.uint64)
    for i in range(n):
        if temperature <= 0:
            key = z[i]
        else:
            u = uniform(seed, int(steps[i]), v)
            key = z[i] / temperature - np.log(-np.log(u))
        out[i] = int(np.argmax(key))          # first maximum: the lowest index
    return out
