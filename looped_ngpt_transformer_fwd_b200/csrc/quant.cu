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
//
// NVFP4 (same page, the NVFP4 release): blocks of 16 consecutive values along
// K share an E4M3 scale s = E4M3(amax_block / (6 g)) under a per-tensor fp32
// scale g; each value becomes the E2M1 code nearest to x / (s g) (ties to
// even, saturating at 6).  Both decisions are those of the exact rational
// rounding (blockscale.cuh): taken from the hardware conversions of a tight
// fp32 bracket of the quotient, and where the bracket straddles a decision
// point from a float64 quotient (scale) or the exact sign of |x| minus each
// E2M1 midpoint times s g (element).  Codes are packed two per byte
// (element 2i in the low nibble); scales go in 2048-byte chunks, one per (128
// rows, 256 K): chunk (kc, rb) at ((kc * row_blocks) + rb) * 2048, and inside
// it the scale of row r = rb*128 + 32*j + i and 16-block b (0..15) at byte
// (b / 4) * 512 + i*16 + j*4 + b % 4, i.e. four 512-byte pieces, one per
// 64-K MMA, each laid out like an MXFP8 chunk with the four bytes of a word
// being the word's four 16-blocks.
#include <cuda_fp8.h>
#include <string.h>

#include <algorithm>

#include "blockscale.cuh"
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


// One warp per (padded) row.  Lane l holds values 4l..4l+3 of each 128 of the
// row (coalesced loads and stores); the 8 lanes of a group of 8 hold one block
// of 32, whose amax is a 3-step shuffle.  Loads go out kQuantUnroll steps at a
// time.  With `normalize` a first pass over the row sums the squares (no
// block-wide barrier: the warp owns the row) and the second pass re-reads the
// row from cache.
template <typename T>
__global__ void __launch_bounds__(32 * kQuantWarps)
    quant_mxfp8_kernel(const __grid_constant__ QuantSrc<T> src, int rows, int rows_pad, int K, int row_blocks,
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
      const int sexp = mx_block_exponent(amax * inv);
      const int q32 = k0 / 32;
      if ((lane & 7) == 0)
        srow[static_cast<size_t>(q32 / 4) * row_blocks * 512 + (q32 % 4)] =
            static_cast<uint8_t>(row ? sexp + 127 : 127);
      if (!row) continue;
      const float f = inv * mx_pow2_neg(sexp);
      *reinterpret_cast<uint32_t*>(codes + static_cast<size_t>(r) * K + k0) =
          mx_codes4(v[u][0], v[u][1], v[u][2], v[u][3], f);
    }
  }
}

// ------------------------------------------------------------------ one CTA per row
//
// The row kernel of both formats: a CTA quantises one (padded) row, its
// threads holding the whole row in registers as loaded (chunks of 8 values:
// chunk c in thread c % blockDim, slot c / blockDim), so the normalising
// variant reads the row once and sums its squares with one block reduction.
// Many small CTAs (one per row) keep the last wave short; the warp-per-row
// kernels remain for rows too long to hold.

template <typename T> struct Chunk8;
template <> struct Chunk8<__nv_bfloat16> {
  uint4 u;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) {
    u = *reinterpret_cast<const uint4*>(p);
  }
  __device__ __forceinline__ void zero() { u = make_uint4(0u, 0u, 0u, 0u); }
  __device__ __forceinline__ void get(float (&v)[8]) const {
    v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z); v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
  }
};
template <> struct Chunk8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = reinterpret_cast<const float4*>(p)[0];
    b = reinterpret_cast<const float4*>(p)[1];
  }
  __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ void get(float (&v)[8]) const {
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
};

// chunks of 8 a thread holds: 36 registers of bf16 or 32 of fp32
template <typename T> constexpr int kRowQuantChunks = sizeof(T) == 2 ? 9 : 4;

__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  for (int i = 0; i < nw; ++i) t += red[i];
  return t;
}

template <int FMT, typename T>
__global__ void __launch_bounds__(1024)
    quant_rows_kernel(const __grid_constant__ QuantSrc<T> src, int rows, int K, int row_blocks,
                      int normalize, float norm_eps, const float* __restrict__ d_g, float g_host,
                      uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  constexpr int NC = kRowQuantChunks<T>;
  __shared__ float red[32];
  const int r = blockIdx.x;                  // one CTA per row: exits are uniform
  const int nch = K / 8, t = threadIdx.x, nt = blockDim.x;
  const T* row = r < rows ? source_row(src, r, K) : nullptr;
  Chunk8<T> x[NC];
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < NC; ++j) {
    const int c = t + j * nt;
    if (row && c < nch) x[j].load(row + static_cast<size_t>(c) * 8);
    else x[j].zero();
  }
  float inv = 1.f;
  if (normalize && row) {                     // uniform
#pragma unroll
    for (int j = 0; j < NC; ++j) {
      float v[8];
      x[j].get(v);
#pragma unroll
      for (int i = 0; i < 8; ++i) ss = fmaf(v[i], v[i], ss);
    }
    inv = rsqrtf(fmaxf(block_sum(ss, red), norm_eps));
  }
  const int rb = r / 128, rr = r % 128;
  if constexpr (FMT == kOperandsNvfp4) {
    const float g = d_g ? *d_g : g_host;
    const float r6 = nv_scale_factor(g);
    uint8_t* srow = scales + static_cast<size_t>(rb) * 2048 + (rr % 32) * 16 + (rr / 32) * 4;
#pragma unroll
    for (int j = 0; j < NC; ++j) {
      const int c = t + j * nt;
      if (j * nt >= nch) break;               // uniform
      float v[8];
      x[j].get(v);
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[i] *= inv;
        amax = fmaxf(amax, fabsf(v[i]));
      }
      // lanes 2b, 2b+1 hold 16-block c / 2 (every lane shuffles: chunks past
      // the row are zeros and store nothing)
      amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
      if (c >= nch) continue;
      const NvScale sc = nv_block_scale_fast(amax, g, r6);
      if ((c & 1) == 0)
        srow[static_cast<size_t>(c / 32) * row_blocks * 2048 + ((c % 32) / 8) * 512 +
             ((c % 32) / 2) % 4] = static_cast<uint8_t>(row ? sc.code : 0x38u);
      if (!row) continue;
      const uint32_t word = nv_codes8(v, sc, g);
      *reinterpret_cast<uint32_t*>(codes + static_cast<size_t>(r) * (K / 2) + c * 4) = word;
    }
  } else {
    uint8_t* srow = scales + static_cast<size_t>(rb) * 512 + (rr % 32) * 16 + (rr / 32) * 4;
#pragma unroll
    for (int j = 0; j < NC; ++j) {
      const int c = t + j * nt;
      if (j * nt >= nch) break;               // uniform
      float v[8];
      x[j].get(v);
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
      // lanes 4q..4q+3 hold 32-block c / 4
      amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
      if (c >= nch) continue;
      // the normalised values' amax (a uniform positive scale commutes with max)
      const int sexp = mx_block_exponent(amax * inv);
      const int q32 = c / 4;
      if ((c & 3) == 0)
        srow[static_cast<size_t>(q32 / 4) * row_blocks * 512 + (q32 % 4)] =
            static_cast<uint8_t>(row ? sexp + 127 : 127);
      if (!row) continue;
      const float f = inv * mx_pow2_neg(sexp);
      *reinterpret_cast<uint2*>(codes + static_cast<size_t>(r) * K + c * 8) =
          make_uint2(mx_codes4(v[0], v[1], v[2], v[3], f), mx_codes4(v[4], v[5], v[6], v[7], f));
    }
  }
}

// Threads per row for the CTA-per-row kernel (0: the row is too long to hold):
// 128 when the rows fill the GPU, else up to one chunk per thread.
template <typename T>
int row_quant_threads(int rows_pad, int K) {
  const int nch = K / 8;
  int t = rows_pad >= 1024 ? 128 : 1024;
  t = std::min(t, (nch + 31) / 32 * 32);
  const int need = (nch + kRowQuantChunks<T> - 1) / kRowQuantChunks<T>;
  t = std::max(t, (need + 31) / 32 * 32);
  return t <= 1024 ? t : 0;
}

// ------------------------------------------------------------------ NVFP4: a block per thread
// The NVFP4 quantiser with one CTA per (padded) row and each thread owning
// whole 16-value blocks (block b = thread + j * blockDim, two adjacent 16-byte
// loads): the block scale is formed once per block and no shuffles are
// needed.  A normalising row folds 1 / ||row|| into the bracket factor of
// the element decisions: x * fl(fl(inv * (1 / (s g))) * (1 -+ 2^-20)) carries
// one rounding more than without the norm, still inside the 2^-20 margin;
// the block scale uses fl(amax * inv), which is the largest fl(x * inv)
// (rounding is monotone), and the exact fallback takes the normalised
// values fl(x * inv) themselves: the codes are those of quant_rows_kernel.
template <typename T> constexpr int kNvBlocks = sizeof(T) == 2 ? 5 : 3;   // blocks per thread
constexpr int kNvBlockThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kNvBlockThreads)
    quant_nv_blocks_kernel(const __grid_constant__ QuantSrc<T> src, int rows, int K,
                           int row_blocks, int normalize, float norm_eps,
                           const float* __restrict__ d_g, float g_host,
                           uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  constexpr int NB = kNvBlocks<T>;
  __shared__ float red[32];
  const int r = blockIdx.x;                  // one CTA per row: exits are uniform
  const int nb = K / 16, t = threadIdx.x, nt = blockDim.x;
  const T* row = r < rows ? source_row(src, r, K) : nullptr;
  Chunk8<T> x[NB][2];
#pragma unroll
  for (int j = 0; j < NB; ++j) {
    const int b = t + j * nt;
    if (row && b < nb) {
      x[j][0].load(row + static_cast<size_t>(b) * 16);
      x[j][1].load(row + static_cast<size_t>(b) * 16 + 8);
    } else {
      x[j][0].zero();
      x[j][1].zero();
    }
  }
  float inv = 1.f;
  if (normalize && row) {                     // uniform
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < NB; ++j)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float v[8];
        x[j][h].get(v);
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = fmaf(v[i], v[i], ss);
      }
    inv = rsqrtf(fmaxf(block_sum(ss, red), norm_eps));
  }
  const float g = d_g ? *d_g : g_host;
  const float r6 = nv_scale_factor(g);
  const int rb = r / 128, rr = r % 128;
  uint8_t* srow = scales + static_cast<size_t>(rb) * 2048 + (rr % 32) * 16 + (rr / 32) * 4;
#pragma unroll
  for (int j = 0; j < NB; ++j) {
    const int b = t + j * nt;
    if (b >= nb) break;
    float v[8], w[8];
    x[j][0].get(v);
    x[j][1].get(w);
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fmaxf(fabsf(v[i]), fabsf(w[i])));
    const NvScale sc = nv_block_scale_fast(amax * inv, g, r6);
    srow[static_cast<size_t>(b / 16) * row_blocks * 2048 + ((b % 16) / 4) * 512 + (b % 4)] =
        static_cast<uint8_t>(row ? sc.code : 0x38u);
    if (!row) continue;
    uint32_t c0 = 0u, c1 = 0u;
    if (sc.s > 0.f) {
      float rs;
      bool done = false;
      if (nv_fast_scale(sc, g, rs)) {
        const float f = inv * rs;
        const float flo = f * kNvBracketLo, fhi = f * kNvBracketHi;
        const uint32_t l0 = e2m1_codes8(v, flo), l1 = e2m1_codes8(w, flo);
        if (l0 == e2m1_codes8(v, fhi) && l1 == e2m1_codes8(w, fhi)) {
          c0 = l0;
          c1 = l1;
          done = true;
        }
      }
      if (!done) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          v[i] *= inv;
          w[i] *= inv;
        }
        c0 = nv_codes4_exact(v[0], v[1], v[2], v[3], sc.s, g) |
             (nv_codes4_exact(v[4], v[5], v[6], v[7], sc.s, g) << 16);
        c1 = nv_codes4_exact(w[0], w[1], w[2], w[3], sc.s, g) |
             (nv_codes4_exact(w[4], w[5], w[6], w[7], sc.s, g) << 16);
      }
    }
    *reinterpret_cast<uint2*>(codes + static_cast<size_t>(r) * (K / 2) + static_cast<size_t>(b) * 8) =
        make_uint2(c0, c1);
  }
}

// Threads per row for quant_nv_blocks_kernel (0: the row has too many blocks)
template <typename T>
int nv_block_threads(int rows_pad, int K) {
  const int nb = K / 16;
  int t = rows_pad >= 1024 ? 128 : kNvBlockThreads;
  t = std::min(t, (nb + 31) / 32 * 32);
  const int need = (nb + kNvBlocks<T> - 1) / kNvBlocks<T>;
  t = std::max(t, (need + 31) / 32 * 32);
  return t <= kNvBlockThreads ? t : 0;
}

template <typename T>
cudaError_t launch_quant(const QuantSrc<T>& src, int rows, int row_align, int K, int normalize,
                         float norm_eps, uint8_t* codes, uint8_t* scales, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (K % 128 != 0 || (row_align != 128 && row_align != 256)) return cudaErrorInvalidValue;
  const int rows_pad = (rows + row_align - 1) / row_align * row_align;
  const int row_blocks = rows_pad / 128;
  if (const int nt = row_quant_threads<T>(rows_pad, K)) {
    quant_rows_kernel<kOperandsMxfp8, T><<<rows_pad, nt, 0, s>>>(
        src, rows, K, row_blocks, normalize, norm_eps, nullptr, 0.f, codes, scales);
    return cudaGetLastError();
  }
  quant_mxfp8_kernel<T><<<(rows_pad + kQuantWarps - 1) / kQuantWarps, 32 * kQuantWarps, 0, s>>>(
      src, rows, rows_pad, K, row_blocks, normalize, norm_eps, codes, scales);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ NVFP4

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
  v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z); v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
}
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0];
  const float4 b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

constexpr int kNvUnroll = 4;   // 256-value steps whose loads are in flight together

// One warp per (padded) row.  Lane l holds values 8l..8l+7 of each 256 of the
// row; lanes 2b and 2b+1 share 16-block b (amax by one shuffle).
template <typename T>
__global__ void __launch_bounds__(32 * kQuantWarps)
    quant_nvfp4_kernel(const __grid_constant__ QuantSrc<T> src, int rows, int rows_pad, int K, int row_blocks,
                       int normalize, float norm_eps, const float* __restrict__ d_g, float g_host,
                       uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
  if (r >= rows_pad) return;                      // warp-uniform
  const T* row = r < rows ? source_row(src, r, K) : nullptr;
  const float g = d_g ? *d_g : g_host;
  const float r6 = nv_scale_factor(g);
  float inv = 1.f;
  if (normalize && row) {
    float ss = 0.f;
    for (int base = 0; base < K; base += 256 * kNvUnroll) {
      float v[kNvUnroll][8];
#pragma unroll
      for (int u = 0; u < kNvUnroll; ++u) {
        const int k0 = base + u * 256 + lane * 8;
        if (k0 < K) load8(row + k0, v[u]);
        else
#pragma unroll
          for (int i = 0; i < 8; ++i) v[u][i] = 0.f;
      }
#pragma unroll
      for (int u = 0; u < kNvUnroll; ++u)
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = fmaf(v[u][i], v[u][i], ss);
    }
    inv = rsqrtf(fmaxf(warp_sum(ss), norm_eps));
  }
  const int rb = r / 128, rr = r % 128;
  uint8_t* srow = scales + static_cast<size_t>(rb) * 2048 + (rr % 32) * 16 + (rr / 32) * 4;
  for (int base = 0; base < K; base += 256 * kNvUnroll) {
    float v[kNvUnroll][8];
#pragma unroll
    for (int u = 0; u < kNvUnroll; ++u) {
      const int k0 = base + u * 256 + lane * 8;
      if (row && k0 < K) load8(row + k0, v[u]);
      else
#pragma unroll
        for (int i = 0; i < 8; ++i) v[u][i] = 0.f;
    }
#pragma unroll
    for (int u = 0; u < kNvUnroll; ++u) {
      if (base + u * 256 >= K) break;             // warp-uniform (K is a multiple of 256)
      const int k0 = base + u * 256 + lane * 8;
#pragma unroll
      for (int i = 0; i < 8; ++i) v[u][i] *= inv;
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[u][i]));
      amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
      const NvScale sc = nv_block_scale_fast(amax, g, r6);
      const int b = (k0 % 256) / 16;              // 16-block within the 256
      if ((lane & 1) == 0)
        srow[static_cast<size_t>(k0 / 256) * row_blocks * 2048 + (b / 4) * 512 + (b % 4)] =
            static_cast<uint8_t>(row ? sc.code : 0x38u);
      if (!row) continue;
      const uint32_t word = nv_codes8(v[u], sc, g);
      *reinterpret_cast<uint32_t*>(codes + static_cast<size_t>(r) * (K / 2) + k0 / 2) = word;
    }
  }
}

template <typename T>
cudaError_t launch_quant_nv(const QuantSrc<T>& src, int rows, int row_align, int K, int normalize,
                            float norm_eps, const float* d_g, float g, uint8_t* codes,
                            uint8_t* scales, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (K % 256 != 0 || (row_align != 128 && row_align != 256)) return cudaErrorInvalidValue;
  if (!d_g && !(g > 0.f)) return cudaErrorInvalidValue;
  const int rows_pad = (rows + row_align - 1) / row_align * row_align;
  const int row_blocks = rows_pad / 128;
  if (const int nt = nv_block_threads<T>(rows_pad, K)) {
    quant_nv_blocks_kernel<T><<<rows_pad, nt, 0, s>>>(src, rows, K, row_blocks, normalize,
                                                      norm_eps, d_g, g, codes, scales);
    return cudaGetLastError();
  }
  if (const int nt = row_quant_threads<T>(rows_pad, K)) {
    quant_rows_kernel<kOperandsNvfp4, T><<<rows_pad, nt, 0, s>>>(
        src, rows, K, row_blocks, normalize, norm_eps, d_g, g, codes, scales);
    return cudaGetLastError();
  }
  quant_nvfp4_kernel<T><<<(rows_pad + kQuantWarps - 1) / kQuantWarps, 32 * kQuantWarps, 0, s>>>(
      src, rows, rows_pad, K, row_blocks, normalize, norm_eps, d_g, g, codes, scales);
  return cudaGetLastError();
}

// amax of |x| over n bf16 values, as the bits of a non-negative float (their
// order as unsigned integers is the order of the values)
__global__ void amax_bf16_kernel(const __nv_bfloat16* __restrict__ x, size_t n,
                                 uint32_t* __restrict__ amax) {
  float m = 0.f;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    m = fmaxf(m, fabsf(__bfloat162float(x[i])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax, __float_as_uint(m));
}

// g = amax / (6 * 448): the quotient rounded to float64, then to fp32
__global__ void tensor_scale_kernel(const uint32_t* amax, float* g) {
  const float a = __uint_as_float(*amax);
  *g = a > 0.f ? static_cast<float>(static_cast<double>(a) / 2688.0) : 1.f;
}

}  // namespace

size_t nvfp4_scale_bytes(int rows, int K, int row_align) {
  return static_cast<size_t>((rows + row_align - 1) / row_align * (row_align / 128)) * (K / 256) *
         2048;
}

cudaError_t launch_quant_nvfp4_bf16(const __nv_bfloat16* const* segs, const int* seg_rows,
                                    int n_seg, int group, int rows, int row_align, int K,
                                    int normalize, float norm_eps, const float* d_g, float g,
                                    uint8_t* codes, uint8_t* scales, cudaStream_t s) {
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
  return launch_quant_nv(q, rows, row_align, K, normalize, norm_eps, d_g, g, codes, scales, s);
}

cudaError_t launch_quant_nvfp4_f32(const float* src, int rows, int K, int normalize, float norm_eps,
                                   const float* d_g, float g, uint8_t* codes, uint8_t* scales,
                                   cudaStream_t s) {
  QuantSrc<float> q;
  memset(&q, 0, sizeof(q));
  q.seg[0] = src;
  q.seg_row[1] = rows;
  q.n_seg = 1;
  return launch_quant_nv(q, rows, 128, K, normalize, norm_eps, d_g, g, codes, scales, s);
}

cudaError_t launch_nvfp4_tensor_scale(const __nv_bfloat16* const* mats, const size_t* counts, int n,
                                      uint32_t* d_amax, float* d_g, cudaStream_t s) {
  if (n < 1 || !d_amax || !d_g) return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(d_amax, 0, sizeof(uint32_t), s);
  for (int i = 0; i < n && e == cudaSuccess; ++i) {
    if (counts[i] == 0) continue;
    const size_t blocks = std::min<size_t>((counts[i] + 255) / 256, 4096);
    amax_bf16_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(mats[i], counts[i], d_amax);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;
  tensor_scale_kernel<<<1, 1, 0, s>>>(d_amax, d_g);
  return cudaGetLastError();
}

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
