// Row and gather kernels of the attention sublayer's backward on a training
// sequence (positions 0..T-1, every key one of the sequence's own): the
// building block, with the MLP sublayer's, of the step that truncated
// depth-one back-propagation runs over the final recurrent invocation
// ("Dory1.0-4B: A Looped Normalized-GPT", Methodology in Plain English).
//
// The products run on the tcgen05 GEMM per KV head, the G query heads of the
// head's group stacked into one [G*T, hd] operand (so the group's sums of dK
// and dV come out of the contraction):
//   S = Q_s K^T,  P = softmax(scale S) masked,  O_s = P V,
//   dP = dO_s V^T,  dS = scale P (dP - rowsum(P dP)),
//   dV = P^T dO_s,  dQ_s = dS K,  dK = dS^T Q_s.
// Softmax rows use their exact maximum (the backward has the whole row).
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace dory {

namespace {

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// dst[(g * T + t) * hd + e] = src[(t * src_heads + head0 + g) * hd + e]
__global__ void gather_heads_kernel(const __nv_bfloat16* __restrict__ src, int T, int src_heads,
                                    int head0, int G, int hd, __nv_bfloat16* __restrict__ dst) {
  const size_t id = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;   // one uint4
  const int per_row = hd / 8;
  const size_t total = static_cast<size_t>(G) * T * per_row;
  if (id >= total) return;
  const int c = static_cast<int>(id % per_row);
  const size_t gt = id / per_row;
  const int t = static_cast<int>(gt % T), g = static_cast<int>(gt / T);
  reinterpret_cast<uint4*>(dst + gt * hd)[c] =
      reinterpret_cast<const uint4*>(src + (static_cast<size_t>(t) * src_heads + head0 + g) * hd)[c];
}

// Eight consecutive fp32 values and eight bf16 values (16-byte accesses; row
// pitches are multiples of 8 elements).
__device__ __forceinline__ void ld8f(const float* p, float (&v)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0];
  const float4 b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void ld8h(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
  v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z); v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
}
__device__ __forceinline__ void st8h(__nv_bfloat16* p, const float (&v)[8]) {
  *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                            pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
}

__device__ __forceinline__ float block_reduce(float v, float* red, bool is_max) {
  v = is_max ? warp_max_f(v) : warp_sum(v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = is_max ? -INFINITY : 0.f;
  for (int w = 0; w < static_cast<int>((blockDim.x + 31) >> 5); ++w)
    r = is_max ? fmaxf(r, red[w]) : r + red[w];
  __syncthreads();   // red is reused by the next reduction
  return r;
}

// One CTA per row r of S [rows, ld] (row r is query t = r % T): P = masked
// softmax(scale S) over keys j in [lo(t), t] (lo = max(0, t - W + 1) for a
// window W, else 0), bf16, zeros elsewhere up to ld.  Eight keys per access.
__global__ void softmax_rows_kernel(const float* __restrict__ S, int T, int ld, int window,
                                    float scale, __nv_bfloat16* __restrict__ P) {
  __shared__ float red[32];
  const int r = blockIdx.x;
  const int t = r % T;
  const int lo = window > 0 ? max(0, t - window + 1) : 0;
  const float* s = S + static_cast<size_t>(r) * ld;
  __nv_bfloat16* p = P + static_cast<size_t>(r) * ld;
  const int c0 = lo / 8, c1 = t / 8;   // chunks holding visible keys
  float m = -INFINITY;
  for (int c = c0 + threadIdx.x; c <= c1; c += blockDim.x) {
    float v[8];
    ld8f(s + 8 * c, v);
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (8 * c + u >= lo && 8 * c + u <= t) m = fmaxf(m, v[u]);
  }
  m = block_reduce(m, red, true);
  float l = 0.f;
  for (int c = c0 + threadIdx.x; c <= c1; c += blockDim.x) {
    float v[8];
    ld8f(s + 8 * c, v);
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (8 * c + u >= lo && 8 * c + u <= t) l += __expf(scale * (v[u] - m));
  }
  const float inv = 1.f / block_reduce(l, red, false);
  for (int c = threadIdx.x; c < ld / 8; c += blockDim.x) {
    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (c >= c0 && c <= c1) {
      float x[8];
      ld8f(s + 8 * c, x);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        v[u] = (8 * c + u >= lo && 8 * c + u <= t) ? __expf(scale * (x[u] - m)) * inv : 0.f;
    }
    st8h(p + 8 * c, v);
  }
}

// dS = scale * P * (dP - D), D = sum_j P dP over the row's visible keys (one
// CTA per row, query t = row % T); entries outside [lo(t), t] are zero and
// their dP is not read (the dP GEMM skips tiles above the diagonal).
__global__ void softmax_bwd_rows_kernel(const __nv_bfloat16* __restrict__ P,
                                        const float* __restrict__ dP, int T, int ld, int window,
                                        float scale, __nv_bfloat16* __restrict__ dS) {
  __shared__ float red[32];
  const size_t off = static_cast<size_t>(blockIdx.x) * ld;
  const int t = blockIdx.x % T;
  const int lo = window > 0 ? max(0, t - window + 1) : 0;
  const int c0 = lo / 8, c1 = t / 8;
  float acc = 0.f;
  for (int c = c0 + threadIdx.x; c <= c1; c += blockDim.x) {
    float pv[8], dv[8];
    ld8h(P + off + 8 * c, pv);
    ld8f(dP + off + 8 * c, dv);
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (8 * c + u >= lo && 8 * c + u <= t) acc += pv[u] * dv[u];
  }
  const float D = block_reduce(acc, red, false);
  for (int c = threadIdx.x; c < ld / 8; c += blockDim.x) {
    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (c >= c0 && c <= c1) {
      float pv[8], dv[8];
      ld8h(P + off + 8 * c, pv);
      ld8f(dP + off + 8 * c, dv);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        v[u] = (8 * c + u >= lo && 8 * c + u <= t) ? scale * pv[u] * (dv[u] - D) : 0.f;
    }
    st8h(dS + off + 8 * c, v);
  }
}

// o[t][q][e] = gate[t][q] * O_s(kv = q / G)[(q % G) * T + t][e]  (bf16)
__global__ void gated_output_kernel(const float* __restrict__ Os, const float* __restrict__ gate,
                                    int T, int hq, int G, int hd, __nv_bfloat16* __restrict__ o) {
  const size_t id = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;   // 4 values
  const size_t total = static_cast<size_t>(T) * hq * hd / 4;
  if (id >= total) return;
  const int e = static_cast<int>(id % (hd / 4)) * 4;
  const size_t tq = id / (hd / 4);
  const int q = static_cast<int>(tq % hq), t = static_cast<int>(tq / hq);
  const size_t srow = (static_cast<size_t>(q / G) * G * T + static_cast<size_t>(q % G) * T + t) * hd;
  const float4 v = *reinterpret_cast<const float4*>(Os + srow + e);
  const float gv = gate[static_cast<size_t>(t) * hq + q];
  *reinterpret_cast<uint2*>(o + tq * hd + e) =
      make_uint2(pack_bf16x2(v.x * gv, v.y * gv), pack_bf16x2(v.z * gv, v.w * gv));
}

// Per (t, query head q), one warp: dgate = <do, O>, the gate logit's gradient
// dgate * gate * (1 - gate) into d_raw[t][gate_col0 + q], and dO_s = gate * do
// (bf16, stacked like O_s).
__global__ void gate_bwd_kernel(const float* __restrict__ dout, const float* __restrict__ Os,
                                const float* __restrict__ gate, int T, int hq, int G, int hd,
                                __nv_bfloat16* __restrict__ dOs, __nv_bfloat16* __restrict__ d_raw,
                                int ld_raw, int gate_col0) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= T * hq) return;
  const int q = warp % hq, t = warp / hq;
  const size_t srow = (static_cast<size_t>(q / G) * G * T + static_cast<size_t>(q % G) * T + t) * hd;
  const float* dv = dout + (static_cast<size_t>(t) * hq + q) * hd;
  const float gv = gate[static_cast<size_t>(t) * hq + q];
  float acc = 0.f;
  for (int e = lane; e < hd; e += 32) {
    const float x = dv[e];
    acc += x * Os[srow + e];
    dOs[srow + e] = __float2bfloat16_rn(gv * x);
  }
  acc = warp_sum(acc);
  if (lane == 0)
    d_raw[static_cast<size_t>(t) * ld_raw + gate_col0 + q] = __float2bfloat16_rn(acc * gv * (1.f - gv));
}

// dst[(t * dst_heads + head0 + g) * hd + e] = src[(g * T + t) * hd + e]  (fp32)
__global__ void scatter_heads_kernel(const float* __restrict__ src, int T, int G, int hd,
                                     int dst_heads, int head0, float* __restrict__ dst) {
  const size_t id = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;   // 4 values
  const size_t total = static_cast<size_t>(G) * T * hd / 4;
  if (id >= total) return;
  const int e = static_cast<int>(id % (hd / 4)) * 4;
  const size_t gt = id / (hd / 4);
  const int t = static_cast<int>(gt % T), g = static_cast<int>(gt / T);
  *reinterpret_cast<float4*>(dst + (static_cast<size_t>(t) * dst_heads + head0 + g) * hd + e) =
      *reinterpret_cast<const float4*>(src + gt * hd + e);
}

// Backward of q_hat = s_qk * u, u = r / |r|, r = RoPE(raw) for one head row per
// warp (heads 0..hq-1 query, hq..hq+hkv-1 key): d_raw = RoPE^-1((s dq_hat -
// u <u, s dq_hat>) / |r|) into the row's columns of d_raw (bf16).  The s_qk
// gradient sum dq_hat * u: each lane adds its pairs' terms over the warp's
// rows in order, the warps' sums are added in warp order into one row of
// partials per CTA (deterministic).  rope: pair-major (cos, sin) [hd/2][T].
constexpr int kQkMaxPairsPerLane = 2;   // head_dim <= 128
__global__ void qk_bwd_kernel(const float* __restrict__ raw, int ld_raw_f,
                              const float* __restrict__ dq_hat, const float* __restrict__ dk_hat,
                              const float* __restrict__ s_qk, const float2* __restrict__ rope,
                              int T, int hq, int hkv, int hd, float norm_eps,
                              __nv_bfloat16* __restrict__ d_raw, int ld_raw,
                              float* __restrict__ ds_part) {
  extern __shared__ float ds_sm[];   // [warps][hd]
  const int warps = blockDim.x >> 5;
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = hd / 2;
  float acc[2 * kQkMaxPairsPerLane];
#pragma unroll
  for (int k = 0; k < 2 * kQkMaxPairsPerLane; ++k) acc[k] = 0.f;
  for (int w = blockIdx.x * warps + wid; w < T * (hq + hkv); w += gridDim.x * warps) {
    const int t = w / (hq + hkv), hh = w % (hq + hkv);
    const bool is_q = hh < hq;
    const int col0 = is_q ? hh * hd : hq * hd + (hh - hq) * hd;   // raw / d_raw columns
    const float* x = raw + static_cast<size_t>(t) * ld_raw_f + col0;
    const float* dh = is_q ? dq_hat + (static_cast<size_t>(t) * hq + hh) * hd
                           : dk_hat + (static_cast<size_t>(t) * hkv + (hh - hq)) * hd;
    float ua[kQkMaxPairsPerLane], ub[kQkMaxPairsPerLane], cs_c[kQkMaxPairsPerLane],
        cs_s[kQkMaxPairsPerLane];
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < kQkMaxPairsPerLane; ++k) {
      const int i = lane + 32 * k;
      ua[k] = ub[k] = cs_c[k] = cs_s[k] = 0.f;
      if (i < half) {
        const float2 cs = rope[static_cast<size_t>(i) * T + t];
        const float a = x[i], b = x[i + half];
        cs_c[k] = cs.x;
        cs_s[k] = cs.y;
        ua[k] = a * cs.x - b * cs.y;   // r, normalised below
        ub[k] = b * cs.x + a * cs.y;
        ss += ua[k] * ua[k] + ub[k] * ub[k];
      }
    }
    const float inv = rsqrtf(fmaxf(warp_sum(ss), norm_eps));
    float c = 0.f;
#pragma unroll
    for (int k = 0; k < kQkMaxPairsPerLane; ++k) {
      const int i = lane + 32 * k;
      if (i < half) {
        ua[k] *= inv;
        ub[k] *= inv;
        c += ua[k] * s_qk[i] * dh[i] + ub[k] * s_qk[i + half] * dh[i + half];
        acc[2 * k] += dh[i] * ua[k];
        acc[2 * k + 1] += dh[i + half] * ub[k];
      }
    }
    c = warp_sum(c);
    __nv_bfloat16* out = d_raw + static_cast<size_t>(t) * ld_raw + col0;
#pragma unroll
    for (int k = 0; k < kQkMaxPairsPerLane; ++k) {
      const int i = lane + 32 * k;
      if (i < half) {
        const float da = (s_qk[i] * dh[i] - ua[k] * c) * inv;
        const float db = (s_qk[i + half] * dh[i + half] - ub[k] * c) * inv;
        // the inverse rotation
        out[i] = __float2bfloat16_rn(da * cs_c[k] + db * cs_s[k]);
        out[i + half] = __float2bfloat16_rn(db * cs_c[k] - da * cs_s[k]);
      }
    }
  }
#pragma unroll
  for (int k = 0; k < kQkMaxPairsPerLane; ++k) {
    const int i = lane + 32 * k;
    if (i < half) {
      ds_sm[wid * hd + i] = acc[2 * k];
      ds_sm[wid * hd + i + half] = acc[2 * k + 1];
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < hd; e += blockDim.x) {
    float sum = 0.f;
    for (int w = 0; w < warps; ++w) sum += ds_sm[w * hd + e];
    ds_part[static_cast<size_t>(blockIdx.x) * hd + e] = sum;
  }
}

// fp32 [T][hkv][hd] head rows into bf16 columns col0 + head * hd of d_raw
__global__ void v_grad_kernel(const float* __restrict__ dv, int T, int hkv, int hd,
                              __nv_bfloat16* __restrict__ d_raw, int ld_raw, int col0) {
  const size_t id = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  const size_t total = static_cast<size_t>(T) * hkv * hd;
  if (id >= total) return;
  const int t = static_cast<int>(id / (static_cast<size_t>(hkv) * hd));
  const int c = static_cast<int>(id % (static_cast<size_t>(hkv) * hd));
  d_raw[static_cast<size_t>(t) * ld_raw + col0 + c] = __float2bfloat16_rn(dv[id]);
}

}  // namespace

cudaError_t launch_gather_heads(const __nv_bfloat16* src, int T, int src_heads, int head0, int G,
                                int hd, __nv_bfloat16* dst, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  if (hd % 8) return cudaErrorInvalidValue;
  const size_t n = static_cast<size_t>(G) * T * (hd / 8);
  gather_heads_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(src, T, src_heads, head0,
                                                                             G, hd, dst);
  return cudaGetLastError();
}

cudaError_t launch_softmax_rows(const float* S, int rows, int T, int ld, int window, float scale,
                                __nv_bfloat16* P, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (ld % 8) return cudaErrorInvalidValue;
  softmax_rows_kernel<<<rows, 256, 0, s>>>(S, T, ld, window, scale, P);
  return cudaGetLastError();
}

cudaError_t launch_softmax_bwd_rows(const __nv_bfloat16* P, const float* dP, int rows, int T,
                                    int ld, int window, float scale, __nv_bfloat16* dS,
                                    cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (ld % 8) return cudaErrorInvalidValue;
  softmax_bwd_rows_kernel<<<rows, 256, 0, s>>>(P, dP, T, ld, window, scale, dS);
  return cudaGetLastError();
}

cudaError_t launch_gated_output(const float* Os, const float* gate, int T, int hq, int G, int hd,
                                __nv_bfloat16* o, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  if (hd % 4) return cudaErrorInvalidValue;
  const size_t n = static_cast<size_t>(T) * hq * hd / 4;
  gated_output_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(Os, gate, T, hq, G, hd, o);
  return cudaGetLastError();
}

cudaError_t launch_gate_bwd(const float* dout, const float* Os, const float* gate, int T, int hq,
                            int G, int hd, __nv_bfloat16* dOs, __nv_bfloat16* d_raw, int ld_raw,
                            int gate_col0, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const size_t warps = static_cast<size_t>(T) * hq;
  gate_bwd_kernel<<<static_cast<unsigned>((warps * 32 + 255) / 256), 256, 0, s>>>(
      dout, Os, gate, T, hq, G, hd, dOs, d_raw, ld_raw, gate_col0);
  return cudaGetLastError();
}

cudaError_t launch_scatter_heads(const float* src, int T, int G, int hd, int dst_heads, int head0,
                                 float* dst, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  if (hd % 4) return cudaErrorInvalidValue;
  const size_t n = static_cast<size_t>(G) * T * hd / 4;
  scatter_heads_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(src, T, G, hd, dst_heads,
                                                                              head0, dst);
  return cudaGetLastError();
}

int qk_bwd_grid(int num_sms) { return 2 * num_sms; }

cudaError_t launch_qk_bwd(const float* raw, int ld_raw_f, const float* dq_hat, const float* dk_hat,
                          const float* s_qk, const float2* rope, int T, int hq, int hkv, int hd,
                          float norm_eps, __nv_bfloat16* d_raw, int ld_raw, float* ds_part,
                          int grid, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  if (hd > 64 * kQkMaxPairsPerLane || hd % 2) return cudaErrorInvalidValue;
  qk_bwd_kernel<<<grid, 256, 8 * hd * sizeof(float), s>>>(raw, ld_raw_f, dq_hat, dk_hat, s_qk, rope,
                                                          T, hq, hkv, hd, norm_eps, d_raw, ld_raw,
                                                          ds_part);
  return cudaGetLastError();
}

cudaError_t launch_v_grad(const float* dv, int T, int hkv, int hd, __nv_bfloat16* d_raw, int ld_raw,
                          int col0, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const size_t n = static_cast<size_t>(T) * hkv * hd;
  v_grad_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(dv, T, hkv, hd, d_raw, ld_raw,
                                                                       col0);
  return cudaGetLastError();
}

}  // namespace dory
