// Element and block-scale decisions of the two block-scaled formats, shared by
// the stand-alone quantiser (quant.cu) and the row kernel that quantises the
// updated stream in place (rowops.cu), so both give the same codes.
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

}  // namespace dory
