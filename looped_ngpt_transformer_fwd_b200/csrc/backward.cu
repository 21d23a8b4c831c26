// Backward of the MLP sublayer: the building block of the training step that
// truncated depth-one back-propagation runs over the final recurrent
// invocation ("Dory1.0-4B: A Looped Normalized-GPT", Methodology in Plain
// English: only the final recurrent invocation is trained).
//
// Forward (as the inference path computes it, bf16 GEMM operands):
//   [g | u] = h_b W_gu^T,  a = SiLU(s g) * u  (bf16),  y = a W_d^T,
//   y_hat = y / |y|,  z = h + alpha * (y_hat - h),  h_out = z / |z|
// (the norm of a before the down projection is folded away exactly: y_hat
// does not depend on the length of a, so neither do the gradients).
// Backward, given dL/dh_out, with n(x) the row norm and P_x the projection
// v -> v - x_hat <x_hat, v>:
//   dz = P_hout(dh_out) / |z|,  dh = (1 - alpha) dz (+ the GEMM term below),
//   dalpha = sum_rows dz * (y_hat - h),  dy = P_yhat(alpha dz) / |y|,
//   da = dy W_d,  dW_d = dy^T a,
//   du = da SiLU(s g),  dg = da u s sigma(s g) (1 + s g (1 - sigma(s g))),
//   dh += dg W_g + du W_u,  dW_g = dg^T h_b,  dW_u = du^T h_b.
// The products run on the tcgen05 GEMM, the transposed operands read
// MN-major straight from their row-major buffers (no transposes in memory).
#include "common.cuh"
#include "kernels.h"

namespace dory {

namespace {

constexpr int kBwdChunks = 3;   // float4 chunks per thread (256 threads at d = 3072)

__device__ __forceinline__ float block_sum_bwd(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();   // red may still be read from a previous reduction
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  const int nw = (blockDim.x + 31) >> 5;
  for (int i = 0; i < nw; ++i) t += red[i];
  return t;
}

__device__ __forceinline__ float dot4(const float4& a, const float4& b) {
  return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
}

// The nGPT update's backward for rows blockIdx.x, blockIdx.x + gridDim.x, ...
// Writes dh (its direct part), dy in bf16 (the dgrad / wgrad operand) and this
// CTA's sum of dz * (y_hat - h) over its rows into dalpha_part[blockIdx.x].
__global__ void mlp_bwd_row_kernel(const float* __restrict__ y, const float* __restrict__ h,
                                   const float* __restrict__ alpha,
                                   const float* __restrict__ dh_out, int rows, int d,
                                   float norm_eps, float* __restrict__ dh,
                                   __nv_bfloat16* __restrict__ dy_b,
                                   float* __restrict__ dalpha_part) {
  __shared__ float red[32];
  const int nch = d >> 2;
  float4 acc[kBwdChunks];
#pragma unroll
  for (int j = 0; j < kBwdChunks; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int r = blockIdx.x; r < rows; r += gridDim.x) {   // uniform across the CTA
    const size_t off = static_cast<size_t>(r) * d;
    float4 yv[kBwdChunks], hv[kBwdChunks], gv[kBwdChunks];
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < kBwdChunks; ++j) {
      const int c = threadIdx.x + j * blockDim.x;
      yv[j] = hv[j] = gv[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c < nch) {
        yv[j] = reinterpret_cast<const float4*>(y + off)[c];
        hv[j] = reinterpret_cast<const float4*>(h + off)[c];
        gv[j] = reinterpret_cast<const float4*>(dh_out + off)[c];
        ss += dot4(yv[j], yv[j]);
      }
    }
    const float inv_y = rsqrtf(fmaxf(block_sum_bwd(ss, red), norm_eps));
    // y_hat (over y) and z (over h)
    ss = 0.f;
#pragma unroll
    for (int j = 0; j < kBwdChunks; ++j) {
      const int c = threadIdx.x + j * blockDim.x;
      if (c < nch) {
        const float4 a = reinterpret_cast<const float4*>(alpha)[c];
        yv[j].x *= inv_y; yv[j].y *= inv_y; yv[j].z *= inv_y; yv[j].w *= inv_y;
        hv[j] = make_float4(hv[j].x + a.x * (yv[j].x - hv[j].x), hv[j].y + a.y * (yv[j].y - hv[j].y),
                            hv[j].z + a.z * (yv[j].z - hv[j].z), hv[j].w + a.w * (yv[j].w - hv[j].w));
        ss += dot4(hv[j], hv[j]);
      }
    }
    const float inv_z = rsqrtf(fmaxf(block_sum_bwd(ss, red), norm_eps));
    // <h_out, dh_out> with h_out = z / |z|
    ss = 0.f;
#pragma unroll
    for (int j = 0; j < kBwdChunks; ++j) ss += dot4(hv[j], gv[j]);
    const float c1 = block_sum_bwd(ss, red) * inv_z;
    // dz = (dh_out - h_out c1) / |z|; h (the input) is z - alpha (y_hat - h),
    // re-read for dalpha
    ss = 0.f;
#pragma unroll
    for (int j = 0; j < kBwdChunks; ++j) {
      const int c = threadIdx.x + j * blockDim.x;
      if (c < nch) {
        const float4 a = reinterpret_cast<const float4*>(alpha)[c];
        const float4 hin = reinterpret_cast<const float4*>(h + off)[c];
        float4 dz;
        dz.x = (gv[j].x - hv[j].x * inv_z * c1) * inv_z;
        dz.y = (gv[j].y - hv[j].y * inv_z * c1) * inv_z;
        dz.z = (gv[j].z - hv[j].z * inv_z * c1) * inv_z;
        dz.w = (gv[j].w - hv[j].w * inv_z * c1) * inv_z;
        acc[j].x += dz.x * (yv[j].x - hin.x);
        acc[j].y += dz.y * (yv[j].y - hin.y);
        acc[j].z += dz.z * (yv[j].z - hin.z);
        acc[j].w += dz.w * (yv[j].w - hin.w);
        reinterpret_cast<float4*>(dh + off)[c] =
            make_float4((1.f - a.x) * dz.x, (1.f - a.y) * dz.y, (1.f - a.z) * dz.z, (1.f - a.w) * dz.w);
        gv[j] = make_float4(a.x * dz.x, a.y * dz.y, a.z * dz.z, a.w * dz.w);   // d y_hat
        ss += dot4(yv[j], gv[j]);
      }
    }
    const float c2 = block_sum_bwd(ss, red);
#pragma unroll
    for (int j = 0; j < kBwdChunks; ++j) {
      const int c = threadIdx.x + j * blockDim.x;
      if (c < nch) {
        const float4 dyv = make_float4((gv[j].x - yv[j].x * c2) * inv_y, (gv[j].y - yv[j].y * c2) * inv_y,
                                       (gv[j].z - yv[j].z * c2) * inv_y, (gv[j].w - yv[j].w * c2) * inv_y);
        reinterpret_cast<uint2*>(dy_b + off)[c] =
            make_uint2(pack_bf16x2(dyv.x, dyv.y), pack_bf16x2(dyv.z, dyv.w));
      }
    }
  }
#pragma unroll
  for (int j = 0; j < kBwdChunks; ++j) {
    const int c = threadIdx.x + j * blockDim.x;
    if (c < nch) reinterpret_cast<float4*>(dalpha_part + static_cast<size_t>(blockIdx.x) * d)[c] = acc[j];
  }
}

// out[c] = sum over g of part[g][c]: 32 columns per CTA, 8 row lanes each
// summing every 8th group in order, then the 8 partial sums in lane order (a
// fixed order: deterministic)
__global__ void colsum_kernel(const float* __restrict__ part, int groups, int d,
                              float* __restrict__ out) {
  __shared__ float sm[8][33];
  const int cx = threadIdx.x & 31, gy = threadIdx.x >> 5;
  const int c = blockIdx.x * 32 + cx;
  float s = 0.f;
  if (c < d)
    for (int g = gy; g < groups; g += 8) s += part[static_cast<size_t>(g) * d + c];
  sm[gy][cx] = s;
  __syncthreads();
  if (gy == 0 && c < d) {
    float t = 0.f;
#pragma unroll
    for (int y = 0; y < 8; ++y) t += sm[y][cx];
    out[c] = t;
  }
}

// SwiGLU backward over [rows, ff]: g, u from the fp32 products laid out like
// the packed gate / up weights (gate and up columns alternating in groups of
// `group`), da [rows, ff].  Writes d[g | u] in the same packed layout (the
// dgrad operand) and dg, du as separate [rows, ff] matrices (the wgrad
// operands).  Four consecutive columns per thread.
__global__ void swiglu_bwd_kernel(const float* __restrict__ gu, const float* __restrict__ da,
                                  int rows, int ff, int group, float gate_scale,
                                  __nv_bfloat16* __restrict__ dgu_packed,
                                  __nv_bfloat16* __restrict__ dg_sep,
                                  __nv_bfloat16* __restrict__ du_sep) {
  const size_t id = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  const size_t per_row = static_cast<size_t>(ff) / 4;
  if (id >= per_row * rows) return;
  const int r = static_cast<int>(id / per_row);
  const int j = static_cast<int>(id % per_row) * 4;
  const size_t pg = static_cast<size_t>(r) * 2 * ff + static_cast<size_t>(j / group) * 2 * group + j % group;
  const float4 g = *reinterpret_cast<const float4*>(gu + pg);
  const float4 u = *reinterpret_cast<const float4*>(gu + pg + group);
  const float4 a = *reinterpret_cast<const float4*>(da + static_cast<size_t>(r) * ff + j);
  const float gv[4] = {g.x, g.y, g.z, g.w}, uv[4] = {u.x, u.y, u.z, u.w}, av[4] = {a.x, a.y, a.z, a.w};
  float dg[4], du[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float x = gate_scale * gv[i];
    const float sg = sigmoidf_(x);
    du[i] = av[i] * x * sg;
    dg[i] = av[i] * uv[i] * gate_scale * sg * (1.f + x * (1.f - sg));
  }
  const uint2 pdg = make_uint2(pack_bf16x2(dg[0], dg[1]), pack_bf16x2(dg[2], dg[3]));
  const uint2 pdu = make_uint2(pack_bf16x2(du[0], du[1]), pack_bf16x2(du[2], du[3]));
  *reinterpret_cast<uint2*>(dgu_packed + pg) = pdg;
  *reinterpret_cast<uint2*>(dgu_packed + pg + group) = pdu;
  *reinterpret_cast<uint2*>(dg_sep + static_cast<size_t>(r) * ff + j) = pdg;
  *reinterpret_cast<uint2*>(du_sep + static_cast<size_t>(r) * ff + j) = pdu;
}

__global__ void add_inplace_kernel(float* __restrict__ x, const float* __restrict__ y, size_t n4) {
  const size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  if (i >= n4) return;
  float4 a = reinterpret_cast<float4*>(x)[i];
  const float4 b = reinterpret_cast<const float4*>(y)[i];
  a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
  reinterpret_cast<float4*>(x)[i] = a;
}

}  // namespace

int mlp_bwd_row_grid(int rows, int num_sms) { return rows < 4 * num_sms ? rows : 4 * num_sms; }

cudaError_t launch_mlp_bwd_row(const float* y, const float* h, const float* alpha,
                               const float* dh_out, int rows, int d, float norm_eps, float* dh,
                               __nv_bfloat16* dy_b, float* dalpha_part, int grid, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (d % 4 != 0 || grid <= 0) return cudaErrorInvalidValue;
  int threads = (d / 4 + kBwdChunks - 1) / kBwdChunks;
  threads = ((threads + 31) / 32) * 32;
  if (threads > 1024) return cudaErrorInvalidValue;
  mlp_bwd_row_kernel<<<grid, threads, 0, s>>>(y, h, alpha, dh_out, rows, d, norm_eps, dh, dy_b,
                                              dalpha_part);
  return cudaGetLastError();
}

cudaError_t launch_colsum(const float* part, int groups, int d, float* out, cudaStream_t s) {
  if (d <= 0) return cudaSuccess;
  colsum_kernel<<<(d + 31) / 32, 256, 0, s>>>(part, groups, d, out);
  return cudaGetLastError();
}

cudaError_t launch_swiglu_bwd(const float* gu, const float* da, int rows, int ff, int group,
                              float gate_scale, __nv_bfloat16* dgu_packed, __nv_bfloat16* dg_sep,
                              __nv_bfloat16* du_sep, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (ff % 4 != 0 || group % 4 != 0 || ff % group != 0) return cudaErrorInvalidValue;
  const size_t n = static_cast<size_t>(rows) * (ff / 4);
  swiglu_bwd_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(
      gu, da, rows, ff, group, gate_scale, dgu_packed, dg_sep, du_sep);
  return cudaGetLastError();
}

cudaError_t launch_add_inplace(float* x, const float* y, size_t n, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  if (n % 4 != 0) return cudaErrorInvalidValue;
  const size_t n4 = n / 4;
  add_inplace_kernel<<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, s>>>(x, y, n4);
  return cudaGetLastError();
}

}  // namespace dory
