// Embedding lookup, LM-head scaling and sampling around the looped stack.
// The pages describe the model between its first and last hidden states only;
// these follow the nGPT backbone the model card cites ("NVIDIA Nemotron Labs
// Dory 1.0 4B ...", Key ideas): the input is the token's embedding row scaled to
// unit L2 norm, the logits are s_z[v] * (E_out[v] . h) (the projection runs on
// the tensor-core GEMM, the scale here), and a token is drawn greedily
// (temperature 0: argmax, lowest index on a tie) or by the Gumbel-max rule
// argmax_v z_v / T - log(-log U_v), U_v from the counter-based hash lowbias32
// (C. Wellons, "Prospecting for Hash Functions", 2018) of (seed, the row's
// step counter, v), computed in double precision.
#include "common.cuh"
#include "kernels.h"

namespace dory {

namespace {

// one warp per token row: gather, L2 norm, bf16 out
__global__ void embed_kernel(const __nv_bfloat16* __restrict__ table, int vocab, int d,
                             const int32_t* __restrict__ tokens, int n,
                             __nv_bfloat16* __restrict__ out, uint32_t* status) {
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= n) return;
  const int t = tokens[r];
  uint4* dst = reinterpret_cast<uint4*>(out + static_cast<size_t>(r) * d);
  if (t < 0 || t >= vocab) {
    if (lane == 0) report_status(status, kStatusBounds);
    for (int c = lane; c < d / 8; c += 32) dst[c] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(table + static_cast<size_t>(t) * d);
  float ss = 0.f;
  for (int c = lane; c < d / 8; c += 32) {
    const uint4 u = src[c];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) ss += bf16_lo(w[i]) * bf16_lo(w[i]) + bf16_hi(w[i]) * bf16_hi(w[i]);
  }
  const float inv = rsqrtf(fmaxf(warp_sum(ss), 1e-20f));
  for (int c = lane; c < d / 8; c += 32) {
    const uint4 u = src[c];
    dst[c] = make_uint4(pack_bf16x2(bf16_lo(u.x) * inv, bf16_hi(u.x) * inv),
                        pack_bf16x2(bf16_lo(u.y) * inv, bf16_hi(u.y) * inv),
                        pack_bf16x2(bf16_lo(u.z) * inv, bf16_hi(u.z) * inv),
                        pack_bf16x2(bf16_lo(u.w) * inv, bf16_hi(u.w) * inv));
  }
}

__global__ void scale_columns_kernel(float* __restrict__ z, const float* __restrict__ s,
                                     size_t n4, int v4) {
  const size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  if (i >= n4) return;
  float4 a = reinterpret_cast<float4*>(z)[i];
  const float4 b = reinterpret_cast<const float4*>(s)[i % v4];
  a.x *= b.x; a.y *= b.y; a.z *= b.z; a.w *= b.w;
  reinterpret_cast<float4*>(z)[i] = a;
}

__device__ __forceinline__ uint32_t lowbias32(uint32_t x) {
  x ^= x >> 16;
  x *= 0x7FEB352Du;
  x ^= x >> 15;
  x *= 0x846CA68Bu;
  x ^= x >> 16;
  return x;
}

constexpr int kSampleThreads = 512;

// one CTA per row: the best (key, index) over the vocabulary, ties to the
// lower index
__global__ void __launch_bounds__(kSampleThreads)
    sample_kernel(const float* __restrict__ logits, int vocab, double temperature, uint32_t seed,
                  const int32_t* __restrict__ steps, int32_t* __restrict__ tokens) {
  __shared__ double best_key[kSampleThreads / 32];
  __shared__ int best_idx[kSampleThreads / 32];
  const int r = blockIdx.x;
  const float* z = logits + static_cast<size_t>(r) * vocab;
  const uint32_t base = temperature > 0.0 ? lowbias32(lowbias32(seed) ^ static_cast<uint32_t>(steps[r])) : 0u;
  double bk = -INFINITY;
  int bi = 0x7FFFFFFF;
  for (int v = threadIdx.x; v < vocab; v += kSampleThreads) {
    double key = static_cast<double>(z[v]);
    if (temperature > 0.0) {
      const double u = (static_cast<double>(lowbias32(base ^ static_cast<uint32_t>(v))) + 0.5) *
                       (1.0 / 4294967296.0);
      key = key / temperature - log(-log(u));
    }
    if (key > bk) {          // v increases within a thread: the first maximum stays
      bk = key;
      bi = v;
    }
  }
  // warp then block arg-max; equal keys keep the lower index
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double ok = __shfl_xor_sync(0xFFFFFFFFu, bk, o);
    const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
    if (ok > bk || (ok == bk && oi < bi)) {
      bk = ok;
      bi = oi;
    }
  }
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    best_key[w] = bk;
    best_idx[w] = bi;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double k = best_key[0];
    int i = best_idx[0];
    for (int j = 1; j < kSampleThreads / 32; ++j)
      if (best_key[j] > k || (best_key[j] == k && best_idx[j] < i)) {
        k = best_key[j];
        i = best_idx[j];
      }
    tokens[r] = i;
  }
}

}  // namespace

cudaError_t launch_embed(const __nv_bfloat16* table, int vocab, int d, const int32_t* tokens,
                         int n, __nv_bfloat16* out, uint32_t* status, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  if (d % 8 != 0) return cudaErrorInvalidValue;
  embed_kernel<<<(n + 7) / 8, 256, 0, s>>>(table, vocab, d, tokens, n, out, status);
  return cudaGetLastError();
}

cudaError_t launch_scale_columns(float* z, const float* scale, int rows, int cols, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (cols % 4 != 0) return cudaErrorInvalidValue;
  const size_t n4 = static_cast<size_t>(rows) * cols / 4;
  scale_columns_kernel<<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, s>>>(z, scale, n4, cols / 4);
  return cudaGetLastError();
}

cudaError_t launch_sample(const float* logits, int n, int vocab, float temperature, uint32_t seed,
                          const int32_t* steps, int32_t* tokens, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  sample_kernel<<<n, kSampleThreads, 0, s>>>(logits, vocab, static_cast<double>(temperature), seed,
                                             steps, tokens);
  return cudaGetLastError();
}

}  // namespace dory
