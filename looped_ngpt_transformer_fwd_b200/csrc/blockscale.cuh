// Element and block-scale decisions of the two block-scaled formats, shared by
// the stand-alone quantiser (quant.cu) and the row kernel that quantises the
// updated stream in place (rowops.cu), so both give the same codes.
// Requires sm_100a (the E2M1 conversion instruction).
//
// Formats: the released MXFP8 and NVFP4 checkpoints ("Dory1.0-4B: A Looped
// Normalized-GPT", Key Contributions item 4), read as the public definitions:
//   MXFP8: blocks of 32 share the E8M0 scale 2^(floor(log2 amax) - 8); E4M3
//          elements, nearest (ties to even), saturating at 448;
//   NVFP4: blocks of 16 share the E4M3 scale s = E4M3(amax / (6 g)) under an
//          fp32 tensor scale g; E2M1 elements nearest to x / (s g) (ties to
//          even), saturating at 6.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace dory {

// ------------------------------------------------------------------ MXFP8

// Block scale exponent floor(log2 amax) - 8 from the float's exponent field
// (a subnormal amax gives -135, clamped like any value below 2^-119 to -127).
__device__ __forceinline__ int mx_block_exponent(float amax) {
  if (!(amax > 0.f)) return -127;
  const int e = ((__float_as_int(amax) >> 23) & 0xFF) - 127;
  return min(127, max(-127, e - 8));
}
// The exact power of two 2^-sexp that maps the block into E4M3 range
// (sexp in [-127, 119]: a normal float).
__device__ __forceinline__ float mx_pow2_neg(int sexp) {
  return __int_as_float((127 - sexp) << 23);
}
// Four E4M3 codes (byte i from v_i * f), nearest, saturating.
__device__ __forceinline__ uint32_t mx_codes4(float v0, float v1, float v2, float v3, float f) {
  const __nv_fp8x2_storage_t lo =
      __nv_cvt_float2_to_fp8x2(make_float2(v0 * f, v1 * f), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hi =
      __nv_cvt_float2_to_fp8x2(make_float2(v2 * f, v3 * f), __NV_SATFINITE, __NV_E4M3);
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// ------------------------------------------------------------------ NVFP4

struct NvScale {
  uint32_t code;   // E4M3 code of s
  float s;         // its value (at most 4 significant bits: exact in fp32)
};

// s = E4M3(amax / (6 g)), nearest with ties to even, saturating at 448.  The
// quotient is rounded once to float64; an E4M3 midpoint has 5 significant
// bits, so a quotient of two fp32 values that is not exactly on one lies
// further from it than float64's rounding error, and the decision is that of
// the exact quotient.
__device__ __forceinline__ NvScale nv_block_scale(float amax, float g) {
  NvScale r{0u, 0.f};
  const double q = static_cast<double>(amax) / (6.0 * static_cast<double>(g));
  if (!(q > 0.0)) return r;
  if (q >= 448.0) {
    r.code = 0x7Eu;
    r.s = 448.f;
    return r;
  }
  const long long bits = __double_as_longlong(q);
  const int e = static_cast<int>((bits >> 52) & 0x7FF) - 1023;   // binade of q (q is normal)
  if (e < -6) {
    // E4M3 subnormals: multiples of 2^-9 (n = 8 is 2^-6, the first normal,
    // whose code is 8 as well)
    const int n = static_cast<int>(rint(q * 512.0));
    r.code = static_cast<uint32_t>(n);
    r.s = static_cast<float>(n) * 0.001953125f;
    return r;
  }
  // 1.m of q scaled to [8, 16): three mantissa bits, half to even; n = 16
  // carries into the next binade, which the code arithmetic absorbs
  const double m = __longlong_as_double((bits & 0x000FFFFFFFFFFFFFLL) | 0x3FF0000000000000LL);
  const int n = static_cast<int>(rint(m * 8.0));
  r.code = static_cast<uint32_t>(((e + 7) << 3) + n - 8);
  r.s = static_cast<float>(n) * __int_as_float((e - 3 + 127) << 23);
  return r;
}

// The seven E2M1 grid midpoints 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5 times s
// (each at most 7 significant bits: exact in fp32).
struct NvThresholds {
  float t[7];
};
__device__ __forceinline__ NvThresholds nv_thresholds(float s) {
  NvThresholds r;
  r.t[0] = 0.25f * s; r.t[1] = 0.75f * s; r.t[2] = 1.25f * s; r.t[3] = 1.75f * s;
  r.t[4] = 2.5f * s;  r.t[5] = 3.5f * s;  r.t[6] = 5.0f * s;
  return r;
}

// E2M1 code of x for the block's thresholds: the magnitude code counts the
// midpoints t_i s g that |x| passes, a midpoint itself going to the even
// neighbour (0, 1, 1, 2, 2, 4, 4).  fmaf(-t_i s, g, |x|) forms |x| - t_i s g
// exactly before its one rounding, so its sign is exact (for g above 2^-100,
// where no difference can underflow to zero).
__device__ __forceinline__ uint32_t nv_code(float x, const NvThresholds& th, float g) {
  const float a = fabsf(x);
  const uint32_t m = (fmaf(-th.t[0], g, a) > 0.f) + (fmaf(-th.t[1], g, a) >= 0.f) +
                     (fmaf(-th.t[2], g, a) > 0.f) + (fmaf(-th.t[3], g, a) >= 0.f) +
                     (fmaf(-th.t[4], g, a) > 0.f) + (fmaf(-th.t[5], g, a) >= 0.f) +
                     (fmaf(-th.t[6], g, a) > 0.f);
  return m | (signbit(x) ? 8u : 0u);
}

// ------------------------------------------------------------------ NVFP4, fast path
//
// Both decisions above are roundings of exact quotients (amax / (6 g) to E4M3,
// x / (s g) to E2M1).  The kernels take them from the hardware's
// round-to-nearest-even conversions applied to an fp32 bracket lo <= q <= hi
// of the quotient: a conversion is monotone, so where lo and hi give the same
// code it is the code of q, and only where they differ (q within about 2^-20
// of a decision point: exact ties, and roughly one value in 10^5 otherwise)
// the exact decisions above are taken, out of line.  A bracket end is formed
// as x * fl(r * (1 -+ 2^-20)) with r the reciprocal of fl(a b): fl(a b), the
// reciprocal (rcp.approx: relative error at most 2^-22), the widening and the
// product add up to under 2^-21 of relative error, inside the 2^-20 margin.
// Products that leave the normal fp32 range (saturated scales, s g below
// 2^-120) take the exact path.  The element conversion keeps the sign, a
// negative value that rounds to zero included (code 8, as nv_code gives).

constexpr float kNvBracketLo = 1.f - 0x1p-20f;
constexpr float kNvBracketHi = 1.f + 0x1p-20f;

// 1 / (6 g), the factor of the block-scale bracket
__device__ __forceinline__ float nv_scale_factor(float g) { return __frcp_rn(6.f * g); }

// Reciprocal of a normal float whose reciprocal is normal (rcp.approx.ftz.f32).
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Value of a non-negative, finite E4M3 code (exact in fp32).
__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : static_cast<float>(m) * 0x1p-9f;
}

// The exact decisions, out of line: they are rare, and inlined into every
// unrolled step of a kernel they would crowd the instruction cache.
static __device__ __noinline__ NvScale nv_block_scale_exact(float amax, float g) {
  return nv_block_scale(amax, g);
}
static __device__ __noinline__ uint32_t nv_codes4_exact(float a, float b, float c, float d, float s,
                                                        float g) {
  const NvThresholds th = nv_thresholds(s);
  return nv_code(a, th, g) | (nv_code(b, th, g) << 4) | (nv_code(c, th, g) << 8) |
         (nv_code(d, th, g) << 12);
}

// nv_block_scale(amax, g) with r6 = nv_scale_factor(g).
__device__ __forceinline__ NvScale nv_block_scale_fast(float amax, float g, float r6) {
  NvScale r{0u, 0.f};
  if (!(amax > 0.f)) return r;
  const float q = amax * r6;
  if (q < 440.f) {
    const uint32_t lo = __nv_cvt_float_to_fp8(q * kNvBracketLo, __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float_to_fp8(q * kNvBracketHi, __NV_SATFINITE, __NV_E4M3);
    if (lo == hi) {
      r.code = lo;
      r.s = e4m3_value(lo);
      return r;
    }
  }
  return nv_block_scale_exact(amax, g);
}

// E2M1 codes of a f, b f, c f, d f (nearest, ties to even, saturating at 6,
// sign kept), the first value in the low nibble of the 16-bit result.
__device__ __forceinline__ uint32_t e2m1_codes4(float a, float b, float c, float d, float f) {
  uint32_t w;
  // cvt ... e2m1x2 d, hi, lo puts its first source in the upper nibble
  asm("{\n\t.reg .b8 p0, p1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 p0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 p1, %4, %3;\n\t"
      "mov.b32 %0, {p0, p1, p0, p1};\n\t}"
      : "=r"(w)
      : "f"(a * f), "f"(b * f), "f"(c * f), "f"(d * f));
  return w & 0xFFFFu;
}
// The same for eight values (32-bit result).
__device__ __forceinline__ uint32_t e2m1_codes8(const float (&v)[8], float f) {
  uint32_t w;
  asm("{\n\t.reg .b8 p0, p1, p2, p3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 p0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 p1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 p2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 p3, %8, %7;\n\t"
      "mov.b32 %0, {p0, p1, p2, p3};\n\t}"
      : "=r"(w)
      : "f"(v[0] * f), "f"(v[1] * f), "f"(v[2] * f), "f"(v[3] * f), "f"(v[4] * f),
        "f"(v[5] * f), "f"(v[6] * f), "f"(v[7] * f));
  return w;
}

// Whether the block's scale admits the bracketed element decisions; `rs` is
// then the reciprocal of s g.
__device__ __forceinline__ bool nv_fast_scale(const NvScale& sc, float g, float& rs) {
  const float sg = sc.s * g;
  rs = rcp_approx(sg);
  return sc.code != 0x7Eu && sg >= 0x1p-120f;
}

// Codes of four values of a block with scale sc (16 bits, first value in the
// low nibble): the same codes as nv_code under nv_thresholds(sc.s).
__device__ __forceinline__ uint32_t nv_codes4(float a, float b, float c, float d,
                                              const NvScale& sc, float g) {
  if (!(sc.s > 0.f)) return 0u;
  float rs;
  if (nv_fast_scale(sc, g, rs)) {
    const uint32_t lo = e2m1_codes4(a, b, c, d, rs * kNvBracketLo);
    if (lo == e2m1_codes4(a, b, c, d, rs * kNvBracketHi)) return lo;
  }
  return nv_codes4_exact(a, b, c, d, sc.s, g);
}

// The same for eight values (32 bits).
__device__ __forceinline__ uint32_t nv_codes8(const float (&v)[8], const NvScale& sc, float g) {
  if (!(sc.s > 0.f)) return 0u;
  float rs;
  if (nv_fast_scale(sc, g, rs)) {
    const uint32_t lo = e2m1_codes8(v, rs * kNvBracketLo);
    if (lo == e2m1_codes8(v, rs * kNvBracketHi)) return lo;
  }
  return nv_codes4_exact(v[0], v[1], v[2], v[3], sc.s, g) |
         (nv_codes4_exact(v[4], v[5], v[6], v[7], sc.s, g) << 16);
}

}  // namespace dory
