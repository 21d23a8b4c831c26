"""Block-scaled weight formats of the quantised checkpoints (oracle side).

TEST INFRASTRUCTURE ONLY, like the rest of `oracle/`: only `tests/`,
`__graft_entry__.smoke()` and the CPU legs of `bench.py` may use it.

"Dory1.0-4B: A Looped Normalized-GPT" (ai.info AI summary), Key Contributions
item 4: the model is released as BF16, MXFP8 and NVFP4 checkpoints (Main
Findings: MXFP8 by post-training quantisation, NVFP4 after
quantisation-aware distillation).  The pages give no bit layout; the plainest
reading is the public definition of each format:

* MXFP8: blocks of 32 consecutive values along the reduction (K) axis share a
  power-of-two scale stored as E8M0 (code e means 2^(e - 127)); elements are
  FP8 E4M3 (exponent bias 7, 3 mantissa bits, subnormals, no infinities,
  largest finite 448).  The block's scale exponent is floor(log2(amax)) - 8,
  8 being the largest E4M3 exponent; elements round to nearest (ties to even)
  and saturate at 448.
* NVFP4: blocks of 16 share an E4M3 scale and the whole tensor one fp32 scale
  g = amax / (6 * 448); elements are FP4 E2M1 (exponent bias 1, 1 mantissa
  bit, largest 6).  Block scale s = E4M3(amax_block / (6 g)); elements
  E2M1(x / (s g)), nearest even, saturating at 6.  "The whole tensor" is read
  as the weight one projection GEMM reads: the matrices the forward pass
  multiplies with the same input in one product (q, k, v and the output-gate
  rows; the SwiGLU gate and up rows) share one g, the maximum over the group
  (NVFP4_GROUPS), as the released NVFP4 format does for fused projections.
  Serving is read like MXFP8's: both operands of every projection in NVFP4.
  A projection input's tensor scale is fixed at g = 1 / (6 * 448): its rows
  are unit vectors (the stream, and the attention output and SwiGLU
  activations after their norm), so no element exceeds 1 and every block
  scale stays within E4M3's range (NVFP4_ACT_G); a static input scale is what
  the format's checkpoints carry for activations.

Dequantisation multiplies back; a quantised GEMM is C = A @ W_hat^T with W_hat
the dequantised weights, in float64.  Serving an MXFP8 checkpoint ("standard
post-training quantisation", same page, Methodology in Plain English) is read
as the public MX recipe: the weights are stored in MXFP8 and every projection's
input is quantised to MXFP8 along K as well (mxfp8_gemm), so both operands of
the block-scaled product are E4M3 with E8M0 block scales.  Rounding here is done at the bit level
(exponent, then a round-half-even on the grid of that binade); the tests check
it against an exhaustive nearest-value search and, for E4M3, against
PyTorch's own float8 conversion.
"""

import numpy as np

# (exponent bias, mantissa bits, largest finite value) of the element formats
E4M3 = (7, 3, 448.0)
E2M1 = (1, 1, 6.0)


def round_to_format(x, fmt):
    """Nearest value of the format (ties to the even grid point), saturating at
    the largest finite value; keeps the sign (and -0)."""
    bias, mbits, vmax = fmt
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    emin = 1 - bias                                  # exponent of the smallest normal
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, emin)                          # subnormals share emin's grid
    ulp = np.exp2(e - mbits)
    q = np.rint(a / ulp) * ulp                       # np.rint: half to even
    q = np.minimum(q, vmax)
    return np.copysign(q, x)


def decode(codes, fmt):
    """Values of element codes (sign bit at 1 << (exponent + mantissa bits));
    for E4M3 the all-ones magnitude is NaN."""
    bias, mbits, _ = fmt
    ebits = 4 if fmt == E4M3 else 2
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where((c >> (ebits + mbits)) & 1, -1.0, 1.0)
    field = (c >> mbits) & ((1 << ebits) - 1)
    mant = c & ((1 << mbits) - 1)
    sub = mant * np.exp2(1 - bias - mbits)
    nrm = (1.0 + mant / (1 << mbits)) * np.exp2(field - bias)
    v = sign * np.where(field == 0, sub, nrm)
    if fmt == E4M3:
        v = np.where((field == 15) & (mant == 7), np.nan, v)
    return v


def encode(x, fmt):
    """Codes of values already on the format's grid (see round_to_format)."""
    bias, mbits, _ = fmt
    ebits = 4 if fmt == E4M3 else 2
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    neg = np.signbit(x).astype(np.int64)
    emin = 1 - bias
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    normal = a >= np.exp2(emin)
    field = np.where(normal, e + bias, 0).astype(np.int64)
    mant = np.where(normal, (a / np.exp2(e) - 1.0) * (1 << mbits),
                    a / np.exp2(emin - mbits))
    mant = np.rint(mant).astype(np.int64)
    return (neg << (ebits + mbits)) | (field << mbits) | mant


def e8m0_value(codes):
    """E8M0 scale codes -> 2^(e - 127) (code 255 is NaN)."""
    c = np.asarray(codes, dtype=np.int64)
    return np.where(c == 255, np.nan, np.exp2(c - 127.0))


# ----------------------------------------------------------------- MXFP8

MX_BLOCK = 32


def mxfp8_quantize(w):
    """w [N, K] (K a multiple of 32) -> (element codes [N, K] uint8 E4M3,
    scale codes [N, K/32] uint8 E8M0)."""
    w = np.asarray(w, dtype=np.float64)
    n, k = w.shape
    assert k % MX_BLOCK == 0
    blocks = w.reshape(n, k // MX_BLOCK, MX_BLOCK)
    amax = np.abs(blocks).max(axis=2)
    with np.errstate(divide="ignore"):
        sexp = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 8, -127)
    sexp = np.clip(sexp, -127, 127)
    q = round_to_format(blocks / np.exp2(sexp)[:, :, None], E4M3)
    return (encode(q, E4M3).astype(np.uint8).reshape(n, k),
            (sexp + 127).astype(np.uint8))


def mxfp8_dequantize(codes, scales):
    n, k = codes.shape
    v = decode(codes, E4M3).reshape(n, k // MX_BLOCK, MX_BLOCK)
    return (v * e8m0_value(scales)[:, :, None]).reshape(n, k)


# ----------------------------------------------------------------- NVFP4

NV_BLOCK = 16


NVFP4_ACT_G = np.float32(1.0 / (6.0 * 448.0))
NVFP4_GROUPS = (("wq", "wk", "wv", "wg"), ("wo",), ("w_gate", "w_up"), ("w_down",))


def nvfp4_tensor_scale(*mats):
    """g = amax / (6 * 448) over all elements of the matrices (the quotient in
    float64, then rounded to float32); 1 when every element is zero."""
    amax = max(float(np.abs(np.asarray(m, dtype=np.float64)).max()) for m in mats)
    return np.float32(amax / (6.0 * 448.0)) if amax > 0 else np.float32(1.0)


def nvfp4_quantize(w, g=None):
    """w [N, K] (K a multiple of 16) -> (element codes [N, K] uint8 holding
    E2M1 codes in the low nibble, block scale codes [N, K/16] uint8 E4M3,
    tensor scale g as float32).  g None: the tensor's own (nvfp4_tensor_scale)."""
    w = np.asarray(w, dtype=np.float64)
    n, k = w.shape
    assert k % NV_BLOCK == 0
    g = nvfp4_tensor_scale(w) if g is None else np.float32(g)
    blocks = w.reshape(n, k // NV_BLOCK, NV_BLOCK)
    bmax = np.abs(blocks).max(axis=2)
    s = round_to_format(bmax / (6.0 * float(g)), E4M3)
    denom = (s * float(g))[:, :, None]
    q = np.where(denom > 0, round_to_format(blocks / np.where(denom > 0, denom, 1.0), E2M1), 0.0)
    return (encode(q, E2M1).astype(np.uint8).reshape(n, k),
            encode(s, E4M3).astype(np.uint8), g)


def nvfp4_dequantize(codes, scales, g):
    n, k = codes.shape
    v = decode(codes, E2M1).reshape(n, k // NV_BLOCK, NV_BLOCK)
    return (v * decode(scales, E4M3)[:, :, None] * float(g)).reshape(n, k)


def nvfp4_fake_quant(x, g=NVFP4_ACT_G):
    """x [..., K] (K a multiple of 16) -> the values an NVFP4 encoding of x
    under tensor scale g holds (blocks of 16 along the last axis)."""
    x = np.asarray(x, dtype=np.float64)
    flat = x.reshape(-1, x.shape[-1])
    return nvfp4_dequantize(*nvfp4_quantize(flat, g)).reshape(x.shape)


def nvfp4_gemm(a, w, g_a=NVFP4_ACT_G, g_w=None):
    """Both operands in NVFP4 along K, products summed in float64:
    C = Q(A; g_a) Q(W; g_w)^T (g_w None: W's own tensor scale)."""
    return nvfp4_fake_quant(a, g_a) @ nvfp4_dequantize(*nvfp4_quantize(w, g_w)).T


def mxfp8_fake_quant(x):
    """x [..., K] (K a multiple of 32) -> the values an MXFP8 encoding of x holds:
    blocks of 32 consecutive values along the last axis get their E8M0 scale and
    E4M3 elements (mxfp8_quantize), then are decoded back."""
    x = np.asarray(x, dtype=np.float64)
    flat = x.reshape(-1, x.shape[-1])
    return mxfp8_dequantize(*mxfp8_quantize(flat)).reshape(x.shape)


def mxfp8_gemm(a, w):
    """Both operands in MXFP8 along the reduction axis K, products summed in
    float64: C = Q(A) Q(W)^T, Q = mxfp8_fake_quant.  This is what a block-scaled
    MMA computes on an MXFP8 weight and an activation quantised on the fly."""
    return mxfp8_fake_quant(a) @ mxfp8_fake_quant(w).T


def quantized_gemm(a, w_hat):
    """C = A W_hat^T in float64 (W_hat: dequantised [N, K])."""
    return np.asarray(a, dtype=np.float64) @ np.asarray(w_hat, dtype=np.float64).T


# ------------------------------------------------------ whole-model weights

MATRIX_NAMES = ("wq", "wk", "wv", "wg", "wo", "w_gate", "w_up", "w_down")


def dequantized_provider(provider, fmt):
    """Wrap a weight provider (block -> dict) so that every matrix [out, in] is
    replaced by its quantise -> dequantise version in `fmt` ("mxfp8" or
    "nvfp4"), blocks running along `in` (the GEMM reduction axis); the vectors
    (alpha, s_qk) are left as they are.  NVFP4 matrices of one NVFP4_GROUPS
    entry share the group's tensor scale."""
    from synthetic.bf16 import bf16_bits_to_f32
    if fmt not in ("mxfp8", "nvfp4"):
        raise ValueError(fmt)
    memo = {}

    def provide(b):
        if b not in memo:
            w = dict(provider(b))
            mats = {}
            for n in MATRIX_NAMES:
                m = w[n]
                mats[n] = bf16_bits_to_f32(m).astype(np.float64) if m.dtype == np.uint16 else \
                    np.asarray(m, dtype=np.float64)
            if fmt == "mxfp8":
                for n in MATRIX_NAMES:
                    w[n] = mxfp8_dequantize(*mxfp8_quantize(mats[n]))
            else:
                for group in NVFP4_GROUPS:
                    g = nvfp4_tensor_scale(*(mats[n] for n in group))
                    for n in group:
                        w[n] = nvfp4_dequantize(*nvfp4_quantize(mats[n], g))
            memo[b] = w
        return memo[b]
    return provide
