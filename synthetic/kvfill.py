"""Counter-based contents for pre-filled KV caches (decode workloads).

The decode workloads start from caches holding tens of thousands of cached
positions per sequence, far too many to draw on the host.  Each cached entry is
therefore a pure function of its coordinates, evaluated by one published
32-bit integer hash ("lowbias32", C. Wellons, *Prospecting for Hash Functions*,
2018: xorshift 16, multiply 0x7feb352d, xorshift 15, multiply 0x846ca68b,
xorshift 16).  The same integer arithmetic runs in NumPy (oracle side) and in
torch on the GPU (harness side) and yields bit-identical values.

For cache slot `slot` (an integer naming a layer and loop), sequence `seq`,
position `p`, KV head `h`, dimension `i`:
    w    = (p * n_kv + h) * head_dim + i            (a 32-bit counter)
    hash = lowbias32(w XOR salt(seed, slot, seq, K-or-V))
    K    = (+1 or -1 from the top hash bit) * kscale[i]
    V    = (((hash >> 8) & 255) - 128) / 128         (exact in bf16)
with kscale[i] = bf16(float32(s_qk[i]) * float32(1/sqrt(head_dim))), so every
cached key is s_qk times a unit vector, as the method's keys are.
"""

import numpy as np

from .bf16 import round_bf16

_M32 = 0xFFFFFFFF


def _mul32(x, c):
    # (x * c) mod 2^32 for 0 <= x < 2^32, keeping every product below 2^63 so
    # that signed 64-bit integer arithmetic (NumPy or torch) is exact.
    lo, hi = c & 0xFFFF, c >> 16
    return (x * lo + (((x * hi) & 0xFFFF) << 16)) & _M32


def lowbias32(x):
    """The lowbias32 hash on int64 arrays / tensors / Python ints holding 32-bit values."""
    x = x ^ (x >> 16)
    x = _mul32(x, 0x7FEB352D)
    x = x ^ (x >> 15)
    x = _mul32(x, 0x846CA68B)
    x = x ^ (x >> 16)
    return x


def salt(seed, slot, seq, which):
    """which: 0 for K, 1 for V."""
    s = lowbias32(int(seed) & _M32)
    s = lowbias32(s ^ (int(slot) & _M32))
    s = lowbias32(s ^ (int(seq) & _M32))
    return lowbias32(s ^ int(which))


def kscale(s_qk, head_dim):
    s = np.asarray(s_qk, dtype=np.float32) * np.float32(1.0 / np.sqrt(head_dim))
    return round_bf16(s.astype(np.float32))


def kv_values(seed, slot, seq, positions, n_kv, head_dim, s_qk):
    """NumPy: K, V float32 arrays [len(positions), n_kv, head_dim] (bf16-exact values)."""
    pos = np.asarray(positions, dtype=np.int64)
    w = ((pos[:, None, None] * n_kv + np.arange(n_kv, dtype=np.int64)[None, :, None]) * head_dim
         + np.arange(head_dim, dtype=np.int64)[None, None, :])
    hk = lowbias32(w ^ salt(seed, slot, seq, 0))
    hv = lowbias32(w ^ salt(seed, slot, seq, 1))
    sign = (1 - 2 * (hk >> 31)).astype(np.float32)
    k = sign * kscale(s_qk, head_dim)[None, None, :]
    v = (((hv >> 8) & 255) - 128).astype(np.float32) / np.float32(128.0)
    return k.astype(np.float32), v


def kv_values_torch(seed, slot, seq, positions, n_kv, head_dim, s_qk, device):
    """torch twin of `kv_values`: bf16 tensors [len(positions), n_kv, head_dim] on `device`."""
    import torch
    pos = torch.as_tensor(positions, dtype=torch.int64, device=device)
    w = ((pos[:, None, None] * n_kv + torch.arange(n_kv, dtype=torch.int64, device=device)[None, :, None])
         * head_dim + torch.arange(head_dim, dtype=torch.int64, device=device)[None, None, :])
    hk = lowbias32(w ^ salt(seed, slot, seq, 0))
    hv = lowbias32(w ^ salt(seed, slot, seq, 1))
    ks = torch.from_numpy(kscale(s_qk, head_dim)).to(device)
    k = (1 - 2 * (hk >> 31)).to(torch.float32) * ks[None, None, :]
    v = (((hv >> 8) & 255) - 128).to(torch.float32) / 128.0
    return k.to(torch.bfloat16), v.to(torch.bfloat16)
