// Row-wise kernels of the looped nGPT pass (HBM-bound; one CTA per row):
//   - the nGPT hypersphere update h <- Norm(h + alpha * (Norm(y) - h)) that
//     closes every sublayer ("Dory1.0-4B: A Looped Normalized-GPT",
//     Methodology in Plain English), summing K-split partial products of the
//     projection first, and optionally saving the input block's output e and
//     re-injecting it, x <- Norm(x + e), before a pass of the recurrent block
//     (same page, Methodology);
//   - input staging (bf16 -> fp32 stream + bf16 GEMM operand);
//   - KV-cache commits of fresh keys/values into their slots (ring slots
//     pos % window for sliding-window layers, pos for full layers).
#include <algorithm>

#include "blockscale.cuh"
#include "common.cuh"
#include "kernels.h"

namespace dory {

namespace {

constexpr int kRowMaxChunks = 3;   // float4 chunks per thread (256 threads for d = 3072)

// Sum over the block with one barrier: `red` must not have been read since
// the block's previous barrier (the row kernel alternates two buffers: a
// thread reads a buffer's sums right after that reduction's barrier, so two
// reductions later every thread is done with it).
__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float t = 0.f;
  const int nw = (blockDim.x + 31) >> 5;
  for (int i = 0; i < nw; ++i) t += red[i];
  return t;
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

__device__ __forceinline__ float dot4(const float4& a, const float4& b) {
  return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
}

// Quantise float4 chunk c (values 4c..4c+3) of row r for the next projection.
// The chunks of one scale block sit in consecutive lanes of one warp (4 for
// an NVFP4 block of 16, 8 for an MXFP8 block of 32), and every lane of the
// warp holds a valid chunk or none does, so the block amax is a few shuffles.
__device__ __forceinline__ void quant_chunk(const RowUpdateParams& p, int r, int c,
                                            const float4& v) {
  const int rb = r / 128, rr = r % 128;
  float amax = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
  if (p.q_fmt == kOperandsNvfp4) {
    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
    const NvScale sc = nv_block_scale_fast(amax, p.q_g, p.q_r6);
    const uint32_t word = nv_codes4(v.x, v.y, v.z, v.w, sc, p.q_g);
    reinterpret_cast<uint16_t*>(p.q_codes + static_cast<size_t>(r) * (p.d / 2))[c] =
        static_cast<uint16_t>(word);
    if ((c & 3) == 0) {
      const int b16 = c / 4, kc = b16 / 16, b = b16 % 16;
      p.q_scales[(static_cast<size_t>(kc) * p.q_row_blocks + rb) * 2048 + (b / 4) * 512 +
                 (rr % 32) * 16 + (rr / 32) * 4 + (b % 4)] = static_cast<uint8_t>(sc.code);
    }
  } else {
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    const int sexp = mx_block_exponent(amax);
    reinterpret_cast<uint32_t*>(p.q_codes + static_cast<size_t>(r) * p.d)[c] =
        mx_codes4(v.x, v.y, v.z, v.w, mx_pow2_neg(sexp));
    if ((c & 7) == 0) {
      const int q32 = c / 8;
      p.q_scales[static_cast<size_t>(rb) * 512 + (rr % 32) * 16 + (rr / 32) * 4 +
                 static_cast<size_t>(q32 / 4) * p.q_row_blocks * 512 + (q32 % 4)] =
          static_cast<uint8_t>(sexp + 127);
    }
  }
}

// Three block reductions per row (||y||, ||h'||, ||h_new + e||), with y and h
// held in registers between them.  The kernel is bound by how many rows are in
// flight per SM: variants that need more live registers (all three norms from
// one pass of seven row sums, or two rows per CTA) measured slower on B200,
// and capping the registers at 40 (six resident CTAs instead of four, a
// 12-byte spill) measured 10 % faster than the uncapped 52.
// alpha (and the re-injected row e) go to shared memory by cp.async as the
// kernel starts, so their latency passes under the y / h loads and the first
// reduction; each thread reads back only its own chunks (no barrier).
template <int kThreads, int kMinBlocks>
__global__ void __launch_bounds__(kThreads, kMinBlocks) row_update_kernel(const RowUpdateParams p) {
  __shared__ float red[2][32];
  // alpha | e: d / 4 chunks (d_model is at most 4096)
  constexpr int kPre = kRowMaxChunks * kThreads < 1024 ? kRowMaxChunks * kThreads : 1024;
  __shared__ float4 pre[2][kPre];
  const int r = blockIdx.x;
  // one CTA per row: these exits are uniform across the block
  if (p.row_k) {
    const int kr = p.row_k[r];
    if (kr < 1 || kr > p.k_hi) {
      if (threadIdx.x == 0 && p.loop == 1) report_status(p.status, kStatusBounds);
      return;
    }
    if (p.loop > kr) return;        // this row's loops are done
  }
  // re-injecting the row just saved as e would give Norm(2 h_new) = h_new
  const bool reinject =
      p.e != nullptr && p.e != p.e_save && (!p.row_k || p.loop < p.row_k[r]);
  const int nch = p.d >> 2;
  const size_t row_off = static_cast<size_t>(r) * p.d;
#pragma unroll
  for (int j = 0; j < kRowMaxChunks; ++j) {
    const int c = threadIdx.x + j * blockDim.x;
    if (c < nch) {
      cp_async16(&pre[0][c], p.alpha + 4 * c);
      if (reinject) cp_async16(&pre[1][c], p.e + row_off + 4 * c);
    }
  }
  float4 y[kRowMaxChunks], h[kRowMaxChunks];
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < kRowMaxChunks; ++j) {
    const int c = threadIdx.x + j * blockDim.x;
    y[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    h[j] = y[j];
    if (c < nch) {
      for (int s = 0; s < p.splits; ++s) {
        const float4 t = reinterpret_cast<const float4*>(p.y + s * p.split_stride + row_off)[c];
        y[j].x += t.x; y[j].y += t.y; y[j].z += t.z; y[j].w += t.w;
      }
      h[j] = reinterpret_cast<const float4*>(p.h + row_off)[c];
      ss += dot4(y[j], y[j]);
    }
  }
  const float inv_y = rsqrtf(fmaxf(block_sum(ss, red[0]), p.norm_eps));
  ss = 0.f;
  cp_async_wait_all();
#pragma unroll
  for (int j = 0; j < kRowMaxChunks; ++j) {
    const int c = threadIdx.x + j * blockDim.x;
    if (c < nch) {
      const float4 a = pre[0][c];
      h[j].x += a.x * (y[j].x * inv_y - h[j].x);
      h[j].y += a.y * (y[j].y * inv_y - h[j].y);
      h[j].z += a.z * (y[j].z * inv_y - h[j].z);
      h[j].w += a.w * (y[j].w * inv_y - h[j].w);
      ss += dot4(h[j], h[j]);
    }
  }
  const float inv_h = rsqrtf(fmaxf(block_sum(ss, red[1]), p.norm_eps));
  ss = 0.f;
#pragma unroll
  for (int j = 0; j < kRowMaxChunks; ++j) {
    const int c = threadIdx.x + j * blockDim.x;
    if (c < nch) {
      h[j].x *= inv_h; h[j].y *= inv_h; h[j].z *= inv_h; h[j].w *= inv_h;
      if (p.e_save) reinterpret_cast<float4*>(p.e_save + row_off)[c] = h[j];
      if (reinject) {
        const float4 e = pre[1][c];
        h[j].x += e.x; h[j].y += e.y; h[j].z += e.z; h[j].w += e.w;
        ss += dot4(h[j], h[j]);
      }
    }
  }
  if (reinject) {
    // block_sum is reached by every thread (reinject is uniform)
    const float inv_x = rsqrtf(fmaxf(block_sum(ss, red[0]), p.norm_eps));
#pragma unroll
    for (int j = 0; j < kRowMaxChunks; ++j) {
      h[j].x *= inv_x; h[j].y *= inv_x; h[j].z *= inv_x; h[j].w *= inv_x;
    }
  }
#pragma unroll
  for (int j = 0; j < kRowMaxChunks; ++j) {
    const int c = threadIdx.x + j * blockDim.x;
    if (c < nch) {
      reinterpret_cast<float4*>(p.h + row_off)[c] = h[j];
      const uint2 b = make_uint2(pack_bf16x2(h[j].x, h[j].y), pack_bf16x2(h[j].z, h[j].w));
      if (p.hb) reinterpret_cast<uint2*>(p.hb + row_off)[c] = b;
      if (p.out) reinterpret_cast<uint2*>(p.out + row_off)[c] = b;
      if (p.q_fmt) quant_chunk(p, r, c, h[j]);   // warp-uniform (c < nch is)
    }
  }
}

// ------------------------------------------------------------------ pipelined row update
// The same update for many rows of one K slice without per-row loop counts
// or a fused quantiser (bf16 prefill; 33.4 against 38.0 us per 4096-row
// update of d_model 3072 on B200, cold L2): a persistent CTA streams its rows (r = blockIdx.x, + gridDim.x,
// ...) through a ring of shared-memory stages that one producer lane fills
// with bulk copies (y, h, and e when re-injecting: one d-float vector each),
// so loads stay in flight while the eight consumer warps reduce.  A consumer
// warp frees a stage as soon as its values are in registers.  Consumer
// thread t holds the same chunks as thread t of row_update_kernel and the
// block sums add the same warp sums in the same order: the results are
// bit-identical to that kernel's.
constexpr int kPipeConsumers = 256;
constexpr int kPipeThreads = 32 + kPipeConsumers;
constexpr int kPipeChunks = 4;          // d_model <= 4096
constexpr int kPipeStageBudget = 110 * 1024;   // two CTAs per SM

__device__ __forceinline__ void bulk_load_1d(void* dst, const void* src, uint32_t bytes,
                                             uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void consumer_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(kPipeConsumers) : "memory");
}
// (a, b) summed over the consumer warps with one named barrier; `red` holds
// two buffers of 16 floats used alternately (count n).
__device__ __forceinline__ float2 consumer_sum2(float a, float b, float* red, int& n) {
  a = warp_sum(a);
  b = warp_sum(b);
  float* rb = red + (n & 1) * 16;
  ++n;
  const int w = (threadIdx.x >> 5) - 1;
  if ((threadIdx.x & 31) == 0) {
    rb[w] = a;
    rb[8 + w] = b;
  }
  consumer_bar();
  float2 t = make_float2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < kPipeConsumers / 32; ++i) {
    t.x += rb[i];
    t.y += rb[8 + i];
  }
  return t;
}

__global__ void __launch_bounds__(kPipeThreads, 2)
    row_update_pipe_kernel(const RowUpdateParams p, int stages) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int d = p.d, nch = d >> 2;
  const bool reinject = p.e != nullptr && p.e != p.e_save;
  const int nv = reinject ? 3 : 2;                 // vectors per stage: y | h | e
  const uint32_t vec_bytes = static_cast<uint32_t>(d) * 4;
  float* buf = reinterpret_cast<float*>(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(stages) * nv * vec_bytes);
  uint64_t* empty = full + stages;
  float* red = reinterpret_cast<float*>(empty + stages);    // [2][16]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(red + 32);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kPipeConsumers / 32);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------ producer
    if (lane == 0) {
      uint32_t issued = 0, parity = 0;
      int k = 0;
      for (int r = blockIdx.x; r < p.rows; r += gridDim.x, ++k) {
        const int s = k % stages;
        const uint32_t ph = (k / stages) & 1u;
        if (!mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, p.status)) break;
        float* dst = buf + static_cast<size_t>(s) * nv * d;
        const size_t off = static_cast<size_t>(r) * d;
        mbar_arrive_expect_tx(&full[s], nv * vec_bytes);
        bulk_load_1d(dst, p.y + off, vec_bytes, &full[s]);
        bulk_load_1d(dst + d, p.h + off, vec_bytes, &full[s]);
        if (reinject) bulk_load_1d(dst + 2 * d, p.e + off, vec_bytes, &full[s]);
        issued |= 1u << s;
        parity = (parity & ~(1u << s)) | (ph << s);
      }
      if (*abort_flag) {
        // let the copies in flight land before the CTA exits
        for (int s = 0; s < stages; ++s)
          if (issued & (1u << s)) drain_wait(&full[s], (parity >> s) & 1u);
      }
    }
    return;
  }

  // -------------------------------------------------- consumers
  const int t = threadIdx.x - 32;
  int nred = 0, k = 0;
  for (int r = blockIdx.x; r < p.rows; r += gridDim.x, ++k) {
    const int s = k % stages;
    const uint32_t ph = (k / stages) & 1u;
    const bool ok =
        __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[s], ph, abort_flag, p.status));
    const float4* sy = reinterpret_cast<const float4*>(buf + static_cast<size_t>(s) * nv * d);
    const float4* sh = sy + nch;
    const float4* se = sh + nch;
    float4 y[kPipeChunks], h[kPipeChunks], e[kPipeChunks];
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < kPipeChunks; ++j) {
      const int c = t + j * kPipeConsumers;
      y[j] = h[j] = e[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c < nch) {
        y[j] = sy[c];
        h[j] = sh[c];
        if (reinject) e[j] = se[c];
        ss += dot4(y[j], y[j]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);       // the stage may take a later row
    // a consumer warp whose wait gave up makes every consumer stop here
    const float2 s1 = consumer_sum2(ss, ok ? 0.f : 1.f, red, nred);
    if (s1.y > 0.f) break;
    const float inv_y = rsqrtf(fmaxf(s1.x, p.norm_eps));
    const size_t row_off = static_cast<size_t>(r) * d;
    ss = 0.f;
#pragma unroll
    for (int j = 0; j < kPipeChunks; ++j) {
      const int c = t + j * kPipeConsumers;
      if (c < nch) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(p.alpha) + c);
        h[j].x += a.x * (y[j].x * inv_y - h[j].x);
        h[j].y += a.y * (y[j].y * inv_y - h[j].y);
        h[j].z += a.z * (y[j].z * inv_y - h[j].z);
        h[j].w += a.w * (y[j].w * inv_y - h[j].w);
        ss += dot4(h[j], h[j]);
      }
    }
    const float inv_h = rsqrtf(fmaxf(consumer_sum2(ss, 0.f, red, nred).x, p.norm_eps));
    ss = 0.f;
#pragma unroll
    for (int j = 0; j < kPipeChunks; ++j) {
      const int c = t + j * kPipeConsumers;
      if (c < nch) {
        h[j].x *= inv_h; h[j].y *= inv_h; h[j].z *= inv_h; h[j].w *= inv_h;
        if (p.e_save) reinterpret_cast<float4*>(p.e_save + row_off)[c] = h[j];
        if (reinject) {
          h[j].x += e[j].x; h[j].y += e[j].y; h[j].z += e[j].z; h[j].w += e[j].w;
          ss += dot4(h[j], h[j]);
        }
      }
    }
    if (reinject) {
      const float inv_x = rsqrtf(fmaxf(consumer_sum2(ss, 0.f, red, nred).x, p.norm_eps));
#pragma unroll
      for (int j = 0; j < kPipeChunks; ++j) {
        h[j].x *= inv_x; h[j].y *= inv_x; h[j].z *= inv_x; h[j].w *= inv_x;
      }
    }
#pragma unroll
    for (int j = 0; j < kPipeChunks; ++j) {
      const int c = t + j * kPipeConsumers;
      if (c < nch) {
        reinterpret_cast<float4*>(p.h + row_off)[c] = h[j];
        const uint2 b = make_uint2(pack_bf16x2(h[j].x, h[j].y), pack_bf16x2(h[j].z, h[j].w));
        if (p.hb) reinterpret_cast<uint2*>(p.hb + row_off)[c] = b;
        if (p.out) reinterpret_cast<uint2*>(p.out + row_off)[c] = b;
        if (p.q_fmt) quant_chunk(p, r, c, h[j]);   // warp-uniform (c < nch is)
      }
    }
  }
}

__global__ void load_rows_kernel(const __nv_bfloat16* __restrict__ src, float* __restrict__ h,
                                 __nv_bfloat16* __restrict__ hb, size_t n4) {
  const size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  if (i >= n4) return;
  const uint2 v = reinterpret_cast<const uint2*>(src)[i];
  reinterpret_cast<float4*>(h)[i] = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
  reinterpret_cast<uint2*>(hb)[i] = v;
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                                   size_t n4) {
  const size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  if (i >= n4) return;
  const float4 v = reinterpret_cast<const float4*>(src)[i];
  reinterpret_cast<uint2*>(dst)[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
}

__global__ void kv_commit_kernel(const KvLayerView kv, const __nv_bfloat16* __restrict__ k_new,
                                 const __nv_bfloat16* __restrict__ v_new, int rows, int first_row,
                                 int seq, int pos0, const int32_t* __restrict__ d_seq,
                                 const int32_t* __restrict__ d_pos, uint32_t* status,
                                 const int32_t* __restrict__ row_k, int loop) {
  const int per_row = kv.n_kv * (kv.hd / 8);
  const size_t id = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  const size_t total = static_cast<size_t>(rows - first_row) * per_row;
  if (id >= total) return;
  const int r = first_row + static_cast<int>(id / per_row);
  if (row_k && loop > row_k[r]) return;   // this row's loops are done
  const int rem = static_cast<int>(id % per_row);
  const int head = rem / (kv.hd / 8);
  const int c8 = rem % (kv.hd / 8);
  const int s = d_seq ? d_seq[r] : seq;
  const int pos = d_pos ? d_pos[r] : pos0 + r;
  if (s < 0 || s >= kv.max_seqs || pos < 0 || pos >= kv.max_ctx) {
    report_status(status, kStatusBounds);
    return;
  }
  const int slot = pos % kv.cap;
  const size_t src = (static_cast<size_t>(r) * kv.n_kv + head) * kv.hd + c8 * 8;
  const size_t dst = s * kv.seq_stride + (static_cast<size_t>(head) * kv.cap + slot) * kv.hd + c8 * 8;
  reinterpret_cast<uint4*>(kv.k_base + dst)[0] = reinterpret_cast<const uint4*>(k_new + src)[0];
  reinterpret_cast<uint4*>(kv.v_base + dst)[0] = reinterpret_cast<const uint4*>(v_new + src)[0];
}

constexpr double kTwoPi = 6.283185307179586476925286766559;

__global__ void rope_table_kernel(const double* __restrict__ inv_freq, int half, int rows,
                                  int pos0, const int32_t* __restrict__ d_pos,
                                  float2* __restrict__ out) {
  // pair-major: entry (pair i, row r) at i * rows + r
  const int id = blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= rows * half) return;
  const int i = id / rows, r = id % rows;
  const int pos = d_pos ? d_pos[r] : pos0 + r;
  const double ang = static_cast<double>(pos) * inv_freq[i];
  const double turns = rint(ang * (1.0 / kTwoPi));
  const float red = static_cast<float>(fma(-turns, kTwoPi, ang));
  float sn, cs;
  sincosf(red, &sn, &cs);
  out[id] = make_float2(cs, sn);
}

// one CTA per (row, head group); thread i owns dimensions i and i + hd/2
__global__ void qkvg_post_kernel(const QkvgPostParams p) {
  __shared__ float red[32];
  const int r = blockIdx.x, g = blockIdx.y, i = threadIdx.x;
  const int hd = p.hd, half = hd / 2;
  const float* row = p.part + static_cast<size_t>(r) * p.ld;
  const int n_heads = p.n_q_heads + 2 * p.n_kv_heads;
  if (g == n_heads) {
    // gate logits
    for (int j = i; j < p.n_q_heads; j += blockDim.x) {
      float v = 0.f;
      for (int s = 0; s < p.splits; ++s) v += row[s * p.split_stride + n_heads * hd + j];
      p.gate_out[static_cast<size_t>(r) * p.n_q_heads + j] = sigmoidf_(v);
    }
    return;
  }
  float a = 0.f, b = 0.f;
  for (int s = 0; s < p.splits; ++s) {
    a += row[s * p.split_stride + g * hd + i];
    b += row[s * p.split_stride + g * hd + i + half];
  }
  const bool is_v = g >= p.n_q_heads + p.n_kv_heads;
  if (!is_v) {
    const float2 cs = p.rope[static_cast<size_t>(i) * p.rows + r];
    const float a2 = a * cs.x - b * cs.y;
    const float b2 = b * cs.x + a * cs.y;
    const float inv = rsqrtf(fmaxf(block_sum(a2 * a2 + b2 * b2, red), p.norm_eps));
    a = a2 * inv * p.s_qk[i];
    b = b2 * inv * p.s_qk[i + half];
  }
  __nv_bfloat16* dst;
  if (g < p.n_q_heads)
    dst = p.q_out + (static_cast<size_t>(r) * p.n_q_heads + g) * hd;
  else if (!is_v)
    dst = p.k_out + (static_cast<size_t>(r) * p.n_kv_heads + (g - p.n_q_heads)) * hd;
  else
    dst = p.v_out + (static_cast<size_t>(r) * p.n_kv_heads + (g - p.n_q_heads - p.n_kv_heads)) * hd;
  dst[i] = __float2bfloat16_rn(a);
  dst[i + half] = __float2bfloat16_rn(b);
  if (p.commit && g >= p.n_q_heads && !(p.row_k && p.loop > p.row_k[r])) {
    // this row's k or v head straight into its cache slot
    const int sq = p.d_seq[r], pos = p.d_pos[r];
    if (sq < 0 || sq >= p.kv.max_seqs || pos < 0 || pos >= p.kv.max_ctx) {
      if (i == 0) report_status(p.status, kStatusBounds);
    } else {
      const int head = is_v ? g - p.n_q_heads - p.n_kv_heads : g - p.n_q_heads;
      __nv_bfloat16* cache = (is_v ? p.kv.v_base : p.kv.k_base) + sq * p.kv.seq_stride +
                             (static_cast<size_t>(head) * p.kv.cap + pos % p.kv.cap) * hd;
      cache[i] = __float2bfloat16_rn(a);
      cache[i + half] = __float2bfloat16_rn(b);
    }
  }
}

__global__ void swiglu_post_kernel(const float* __restrict__ part, int splits, size_t split_stride,
                                   int rows, int d_ff, float gate_scale, int group,
                                   __nv_bfloat16* __restrict__ out) {
  const size_t id = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  if (id >= static_cast<size_t>(rows) * d_ff) return;
  const int r = static_cast<int>(id / d_ff), c = static_cast<int>(id % d_ff);
  const size_t gcol = static_cast<size_t>(c / group) * 2 * group + (c % group);
  const float* row = part + static_cast<size_t>(r) * 2 * d_ff;
  float g = 0.f, u = 0.f;
  for (int s = 0; s < splits; ++s) {
    g += row[s * split_stride + gcol];
    u += row[s * split_stride + gcol + group];
  }
  g *= gate_scale;
  out[id] = __float2bfloat16_rn(g * sigmoidf_(g) * u);
}

}  // namespace

cudaError_t launch_rope_table(const double* inv_freq, int hd, int rows, int pos0,
                              const int32_t* d_pos, float2* out, cudaStream_t s) {
  const int n = rows * (hd / 2);
  if (n <= 0) return cudaSuccess;
  rope_table_kernel<<<(n + 255) / 256, 256, 0, s>>>(inv_freq, hd / 2, rows, pos0, d_pos, out);
  return cudaGetLastError();
}

cudaError_t launch_qkvg_post(const QkvgPostParams& p, cudaStream_t s) {
  if (p.rows <= 0) return cudaSuccess;
  dim3 grid(p.rows, p.n_q_heads + 2 * p.n_kv_heads + 1);
  qkvg_post_kernel<<<grid, p.hd / 2, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_swiglu_post(const float* part, int splits, size_t split_stride, int rows,
                               int d_ff, float gate_scale, int group, __nv_bfloat16* out,
                               cudaStream_t s) {
  const size_t n = static_cast<size_t>(rows) * d_ff;
  if (n == 0) return cudaSuccess;
  if (group <= 0 || d_ff % group != 0) return cudaErrorInvalidValue;
  swiglu_post_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(
      part, splits, split_stride, rows, d_ff, gate_scale, group, out);
  return cudaGetLastError();
}

cudaError_t launch_row_update(const RowUpdateParams& p, cudaStream_t s) {
  if (p.d % 4 != 0 || p.rows < 0) return cudaErrorInvalidValue;
  if (p.q_fmt && (p.row_k || !p.q_codes || !p.q_scales || p.d % 128 != 0 ||
                  (p.q_fmt == kOperandsNvfp4 && (p.d % 256 != 0 || !(p.q_g > 0.f))) ||
                  p.q_row_blocks < (p.rows + 127) / 128))
    return cudaErrorInvalidValue;
  if (p.rows == 0) return cudaSuccess;
  int threads = (p.d / 4 + kRowMaxChunks - 1) / kRowMaxChunks;
  threads = ((threads + 31) / 32) * 32;
  if (threads < 32) threads = 32;
  if (p.d > 4096) return cudaErrorInvalidValue;   // the prefetch buffer's size
  RowUpdateParams q = p;
  if (q.q_fmt == kOperandsNvfp4) q.q_r6 = 1.f / (6.f * q.q_g);
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (p.splits == 1 && !p.row_k && !p.q_fmt && p.rows >= sms) {
    // many rows of one K slice: the pipelined kernel, two CTAs per SM (with
    // the stream quantiser fused in, the update is compute-heavier and the
    // one-row CTAs, 48 warps per SM against 16 consumer warps, measured
    // faster: 8.35 against 9.06 ms per NVFP4 prefill step)
    const bool reinject = p.e != nullptr && p.e != p.e_save;
    const size_t stage = static_cast<size_t>(reinject ? 3 : 2) * p.d * 4;
    const int stages = static_cast<int>(std::min<size_t>(8, std::max<size_t>(2, kPipeStageBudget / stage)));
    const size_t bytes = stages * stage + stages * 16 + 32 * 4 + 16;
    static uint32_t attr_done = 0;   // one bit per device ordinal < 32
    if (dev >= 32 || !(attr_done & (1u << dev))) {
      e = cudaFuncSetAttribute(row_update_pipe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(std::min<size_t>(227 * 1024, 2 * kPipeStageBudget + 4096)));
      if (e != cudaSuccess) return e;
      if (dev < 32) attr_done |= 1u << dev;
    }
    const int grid = std::min(p.rows, 2 * sms);
    row_update_pipe_kernel<<<grid, kPipeThreads, bytes, s>>>(q, stages);
    return cudaGetLastError();
  }
  if (threads <= 256)
    row_update_kernel<256, 6><<<p.rows, threads, 0, s>>>(q);
  else if (threads <= 512)   // d_model above 3072
    row_update_kernel<512, 2><<<p.rows, threads, 0, s>>>(q);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_load_rows(const __nv_bfloat16* src, float* h, __nv_bfloat16* hb, int rows,
                             int d, cudaStream_t s) {
  const size_t n4 = static_cast<size_t>(rows) * d / 4;
  if (n4 == 0) return cudaSuccess;
  load_rows_kernel<<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, s>>>(src, h, hb, n4);
  return cudaGetLastError();
}

cudaError_t launch_f32_to_bf16(const float* src, __nv_bfloat16* dst, size_t n, cudaStream_t s) {
  const size_t n4 = n / 4;
  if (n4 == 0) return cudaSuccess;
  f32_to_bf16_kernel<<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, s>>>(src, dst, n4);
  return cudaGetLastError();
}

cudaError_t launch_kv_commit(const KvLayerView& kv, const __nv_bfloat16* k_new,
                             const __nv_bfloat16* v_new, int rows, int first_row, int seq,
                             int pos0, const int32_t* d_seq, const int32_t* d_pos,
                             uint32_t* status, cudaStream_t s, const int32_t* row_k, int loop) {
  if (first_row >= rows) return cudaSuccess;
  const size_t total = static_cast<size_t>(rows - first_row) * kv.n_kv * (kv.hd / 8);
  kv_commit_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, s>>>(
      kv, k_new, v_new, rows, first_row, seq, pos0, d_seq, d_pos, status, row_k, loop);
  return cudaGetLastError();
}

}  // namespace dory
