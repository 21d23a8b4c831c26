// MXFP8 quantisation of GEMM operands (the released MXFP8 checkpoint format,
// "Dory1.0-4B: A Looped Normalized-GPT", Key Contributions item 4, served with
// both operands of every projection in MXFP8): blocks of 32 consecutive values
// along K share an E8M0 scale 2^(floor(log2 amax) - 8); each value becomes the
// E4M3 code nearest to x / scale (ties to even, saturating at 448).
//
// Output layout, chosen for the block-scaled tensor-core GEMM:
//   codes  [rows, K] bytes, row-major (a TMA box of 128 rows x 128 bytes is one
//          K step of the GEMM);
//   scales in 512-byte chunks, one per (128 rows, 128 K): chunk (kc, rb) at
//          ((kc * row_blocks) + rb) * 512, and inside it the scale of row
//          r = rb*128 + 32*j + i and K block q (0..3) at byte i*16 + j*4 + q.
//          tcgen05.cp of a chunk (32 rows of 16 bytes, copied to every group of
//          32 TMEM lanes) puts the scales of row r in column r / 32 of lane
//          r % 32, byte q: the layout the block-scaled MMA reads.
// Rows past `rows` (up to the next multiple of 128, or of 256 for weights read
// as 256-row tiles) get scale code 127 (1.0), so the MMA never multiplies the
// zero-filled padding by an undefined scale.
#include <cuda_fp8.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"

namespace dory {

namespace {

// Where output row r comes from: rows [seg_row[i], seg_row[i+1]) are rows of
// seg[i]; with `group` > 0 the rows instead alternate in groups of `group`
// between seg[0] and seg[1] (gate and up projections of one SwiGLU tile).
template <typename T>
struct QuantSrc {
  const T* seg[4];
  int seg_row[5];
  int n_seg;
  int group;
};

template <typename T>
__device__ __forceinline__ const T* source_row(const QuantSrc<T>& q, int r, int K) {
  if (q.group > 0) {
    const int t = r / (2 * q.group), i = r % (2 * q.group);
    return (i < q.group ? q.seg[0] : q.seg[1]) +
           static_cast<size_t>(t * q.group + (i < q.group ? i : i - q.group)) * K;
  }
  int i = 0;
  while (i + 1 < q.n_seg && r >= q.seg_row[i + 1]) ++i;
  return q.seg[i] + static_cast<size_t>(r - q.seg_row[i]) * K;
}

__device__ __forceinline__ void load4(const __nv_bfloat16* p, float (&v)[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
}
__device__ __forceinline__ void load4(const float* p, float (&v)[4]) {
  const float4 u = *reinterpret_cast<const float4*>(p);
  v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
}

constexpr int kQuantWarps = 8;      // rows per CTA (one warp per row)
constexpr int kQuantUnroll = 8;     // 128-value steps whose loads are in flight together

// Block scale exponent floor(log2 amax) - 8 from the float's exponent field
// (a subnormal amax gives -135, clamped like any value below 2^-119 to -127),
// and the exact power of two 2^-sexp that maps the block into E4M3 range.
__device__ __forceinline__ int block_exponent(float amax) {
  if (!(amax > 0.f)) return -127;
  const int e = ((__float_as_int(amax) >> 23) & 0xFF) - 127;
  return min(127, max(-127, e - 8));
}
__device__ __forceinline__ float pow2_neg(int sexp) {   // sexp in [-127, 119]: a normal float
  return __int_as_float((127 - sexp) << 23);
}

// One warp per (padded) row.  Lane l holds values 4l..4l+3 of each 128 of the
// row (coalesced loads and stores); the 8 lanes of a group of 8 hold one block
// of 32, whose amax is a 3-step shuffle.  Loads go out kQuantUnroll steps at a
// time.  With `normalize` a first pass over the row sums the squares (no
// block-wide barrier: the warp owns the row) and the second pass re-reads the
// row from cache.
template <typename T>
__global__ void __launch_bounds__(32 * kQuantWarps)
    quant_mxfp8_kernel(const QuantSrc<T> src, int rows, int rows_pad, int K, int row_blocks,
                       int normalize, float norm_eps, uint8_t* __restrict__ codes,
                       uint8_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
  if (r >= rows_pad) return;                      // warp-uniform
  const T* row = r < rows ? source_row(src, r, K) : nullptr;
  float inv = 1.f;
  if (normalize && row) {
    float ss = 0.f;
    for (int base = 0; base < K; base += 128 * kQuantUnroll) {
      float v[kQuantUnroll][4];
#pragma unroll
      for (int u = 0; u < kQuantUnroll; ++u) {
        const int k0 = base + u * 128 + lane * 4;
        if (k0 < K) load4(row + k0, v[u]);
        else v[u][0] = v[u][1] = v[u][2] = v[u][3] = 0.f;
      }
#pragma unroll
      for (int u = 0; u < kQuantUnroll; ++u)
        ss = fmaf(v[u][0], v[u][0], fmaf(v[u][1], v[u][1], fmaf(v[u][2], v[u][2], fmaf(v[u][3], v[u][3], ss))));
    }
    inv = rsqrtf(fmaxf(warp_sum(ss), norm_eps));
  }
  const int rb = r / 128, rr = r % 128;
  uint8_t* srow = scales + static_cast<size_t>(rb) * 512 + (rr % 32) * 16 + (rr / 32) * 4;
  for (int base = 0; base < K; base += 128 * kQuantUnroll) {
    float v[kQuantUnroll][4];
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int k0 = base + u * 128 + lane * 4;
      if (row && k0 < K) load4(row + k0, v[u]);
      else v[u][0] = v[u][1] = v[u][2] = v[u][3] = 0.f;
    }
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      if (base + u * 128 >= K) break;             // warp-uniform (K is a multiple of 128)
      const int k0 = base + u * 128 + lane * 4;
      float amax = fmaxf(fmaxf(fabsf(v[u][0]), fabsf(v[u][1])), fmaxf(fabsf(v[u][2]), fabsf(v[u][3])));
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
      // the normalised values' amax (a uniform positive scale commutes with max)
      const int sexp = block_exponent(amax * inv);
      const int q32 = k0 / 32;
      if ((lane & 7) == 0)
        srow[static_cast<size_t>(q32 / 4) * row_blocks * 512 + (q32 % 4)] =
            static_cast<uint8_t>(row ? sexp + 127 : 127);
      if (!row) continue;
      const float f = inv * pow2_neg(sexp);
      const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
          make_float2(v[u][0] * f, v[u][1] * f), __NV_SATFINITE, __NV_E4M3);
      const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
          make_float2(v[u][2] * f, v[u][3] * f), __NV_SATFINITE, __NV_E4M3);
      *reinterpret_cast<uint32_t*>(codes + static_cast<size_t>(r) * K + k0) =
          static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
    }
  }
}

template <typename T>
cudaError_t launch_quant(const QuantSrc<T>& src, int rows, int row_align, int K, int normalize,
                         float norm_eps, uint8_t* codes, uint8_t* scales, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (K % 128 != 0 || (row_align != 128 && row_align != 256)) return cudaErrorInvalidValue;
  const int rows_pad = (rows + row_align - 1) / row_align * row_align;
  const int row_blocks = rows_pad / 128;
  quant_mxfp8_kernel<T><<<(rows_pad + kQuantWarps - 1) / kQuantWarps, 32 * kQuantWarps, 0, s>>>(
      src, rows, rows_pad, K, row_blocks, normalize, norm_eps, codes, scales);
  return cudaGetLastError();
}

}  // namespace

size_t mxfp8_scale_bytes(int rows, int K, int row_align) {
  return static_cast<size_t>((rows + row_align - 1) / row_align * (row_align / 128)) * (K / 128) * 512;
}

cudaError_t launch_quant_mxfp8_bf16(const __nv_bfloat16* const* segs, const int* seg_rows,
                                    int n_seg, int group, int rows, int row_align, int K,
                                    int normalize, float norm_eps, uint8_t* codes, uint8_t* scales,
                                    cudaStream_t s) {
  if (n_seg < 1 || n_seg > 4 || (group > 0 && n_seg != 2)) return cudaErrorInvalidValue;
  QuantSrc<__nv_bfloat16> q;
  memset(&q, 0, sizeof(q));
  for (int i = 0; i < n_seg; ++i) {
    q.seg[i] = segs[i];
    q.seg_row[i] = seg_rows ? seg_rows[i] : 0;
  }
  q.seg_row[n_seg] = rows;
  q.n_seg = n_seg;
  q.group = group;
  return launch_quant(q, rows, row_align, K, normalize, norm_eps, codes, scales, s);
}

cudaError_t launch_quant_mxfp8_f32(const float* src, int rows, int K, int normalize, float norm_eps,
                                   uint8_t* codes, uint8_t* scales, cudaStream_t s) {
  QuantSrc<float> q;
  memset(&q, 0, sizeof(q));
  q.seg[0] = src;
  q.seg_row[1] = rows;
  q.n_seg = 1;
  return launch_quant(q, rows, 128, K, normalize, norm_eps, codes, scales, s);
}

}  // namespace dory
