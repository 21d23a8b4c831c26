// Decode attention (one new query per sequence) over the KV cache of one
// layer, split over the keys so that a batch of long contexts fills all SMs,
// followed by a combine step that merges the splits and applies the per-head
// sigmoid output gate ("Dory1.0-4B: A Looped Normalized-GPT", Methodology in
// Plain English: GQA with sigmoid output gates, sliding-window and full
// layers).  The new token's key and value are already in their cache slot
// (committed before this kernel), so every key comes from the cache: slots
// pos % capacity of a sliding-window ring, or pos of a full layer.
//
// One CTA = one (split, KV head, sequence); the query heads of the KV head's
// group form the rows of a 16-row bf16 mma.sync tile (rows beyond the group are
// zero), so K and V stream through once per group.  K/V tiles of 64 keys are
// staged in shared memory with 16-byte cp.async in a 3-deep pipeline; each of
// the 4 warps owns 16 keys of every tile and its own online-softmax state,
// merged at the end of the split.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace dory {

namespace {

constexpr int kDecTile = 64;
constexpr int kDecStages = 3;
constexpr int kDecThreads = 128;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
template <int CH>
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return static_cast<uint32_t>((r * CH + (c ^ (r & 7))) * 16);
}

// kProbe: also record the keys the softmax included (mask probe, diagnostics)
template <int HD, bool kProbe>
__global__ void __launch_bounds__(kDecThreads) decode_attn_kernel(const DecodeAttnParams p) {
  constexpr int CH = HD / 8;
  constexpr int KSTEPS = HD / 16;
  constexpr int ONT = HD / 8;
  constexpr int kTileBytes = kDecTile * HD * 2;
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);   // stage s: K at s*2*tile, V after it

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int n_splits = gridDim.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int group = p.n_q_heads / p.kv.n_kv;

  const int seq = p.d_seq[b];
  const int pos = p.d_pos[b];
  const bool bad = seq < 0 || seq >= p.kv.max_seqs || pos < 0 || pos >= p.kv.max_ctx ||
                   pos > p.max_pos;
  if (bad && tid == 0 && split == 0 && kvh == 0) report_status(p.status, kStatusBounds);
  const int lo = bad ? 0 : (p.window > 0 ? max(0, pos - p.window + 1) : 0);
  const int k_begin = lo + split * p.split_keys;
  const int k_end = bad ? k_begin : min(pos + 1, k_begin + p.split_keys);   // exclusive
  const int n_tiles = k_end > k_begin ? (k_end - k_begin + kDecTile - 1) / kDecTile : 0;

  const __nv_bfloat16* kbase = p.kv.k_base + static_cast<size_t>(bad ? 0 : seq) * p.kv.seq_stride +
                               static_cast<size_t>(kvh) * p.kv.cap * HD;
  const __nv_bfloat16* vbase = p.kv.v_base + static_cast<size_t>(bad ? 0 : seq) * p.kv.seq_stride +
                               static_cast<size_t>(kvh) * p.kv.cap * HD;

  auto load_tile = [&](int t, int stage) {
    const uint32_t dk = sbase + stage * 2 * kTileBytes, dv = dk + kTileBytes;
    const int t0 = k_begin + t * kDecTile;
    for (int i = tid; i < kDecTile * CH; i += kDecThreads) {
      const int r = i / CH, c = i % CH;
      const int kp = t0 + r;
      const bool ok = kp < k_end;
      const size_t off = static_cast<size_t>(ok ? kp % p.kv.cap : 0) * HD + c * 8;
      cp_async16(dk + swz<CH>(r, c), kbase + off, ok);
      cp_async16(dv + swz<CH>(r, c), vbase + off, ok);
    }
  };

  // prologue: up to kDecStages-1 tiles in flight
#pragma unroll
  for (int s = 0; s < kDecStages - 1; ++s) {
    if (s < n_tiles) load_tile(s, s);
    cp_async_commit();
  }

  // Q fragments: rows = query heads of this group (row g < group), zero elsewhere
  uint32_t qa[KSTEPS][4];
  {
    const bool live = g < group;
    const __nv_bfloat16* q =
        p.q + (static_cast<size_t>(b) * p.n_q_heads + kvh * group + (live ? g : 0)) * HD;
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
      qa[ks][0] = live ? *reinterpret_cast<const uint32_t*>(q + ks * 16 + t4 * 2) : 0u;
      qa[ks][2] = live ? *reinterpret_cast<const uint32_t*>(q + ks * 16 + 8 + t4 * 2) : 0u;
      qa[ks][1] = 0u;
      qa[ks][3] = 0u;
    }
  }

  float o[ONT][4];
#pragma unroll
  for (int j = 0; j < ONT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;   // row g only (rows g+8 are padding)
  ProbeAcc pacc;
  probe_reset(pacc);

  for (int t = 0; t < n_tiles; ++t) {
    const int nxt = t + kDecStages - 1;
    if (nxt < n_tiles) load_tile(nxt, nxt % kDecStages);
    cp_async_commit();
    cp_async_wait<kDecStages - 1>();
    __syncthreads();
    const uint32_t kb = sbase + (t % kDecStages) * 2 * kTileBytes, vb = kb + kTileBytes;
    const int key0 = warp * 16;   // this warp's 16 keys of the tile

    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
      const int mtx = lane >> 3;
      const int r = key0 + (lane & 7) + (mtx >> 1) * 8;
      const int c = 2 * ks + (mtx & 1);
      uint32_t b0, b1, b2, b3;
      ldsm_x4(kb + swz<CH>(r, c), b0, b1, b2, b3);
      mma_bf16(s[0], qa[ks], b0, b1);
      mma_bf16(s[1], qa[ks], b2, b3);
    }
    const int kp0 = k_begin + t * kDecTile + key0;
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int kp = kp0 + j * 8 + t4 * 2 + e;
        const float v = kp < k_end ? s[j][e] * p.scale_log2 : -INFINITY;
        s[j][e] = v;
        mx = fmaxf(mx, v);
        if constexpr (kProbe) {
          if (v != -INFINITY) probe_add(pacc, kp);
        }
      }
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
    const float corr = exp2f(m_run - m_use);
    m_run = m_new;
    const float p00 = exp2f(s[0][0] - m_use), p01 = exp2f(s[0][1] - m_use);
    const float p10 = exp2f(s[1][0] - m_use), p11 = exp2f(s[1][1] - m_use);
    l_run = l_run * corr + (p00 + p01 + p10 + p11);
    uint32_t pa[4] = {pack_bf16x2(p00, p01), 0u, pack_bf16x2(p10, p11), 0u};
#pragma unroll
    for (int j = 0; j < ONT; ++j) {
      o[j][0] *= corr;
      o[j][1] *= corr;
    }
#pragma unroll
    for (int jp = 0; jp < ONT / 2; ++jp) {
      const int mtx = lane >> 3;
      const int r = key0 + (lane & 7) + (mtx & 1) * 8;
      const int c = 2 * jp + (mtx >> 1);
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(vb + swz<CH>(r, c), b0, b1, b2, b3);
      mma_bf16(o[2 * jp], pa, b0, b1);
      mma_bf16(o[2 * jp + 1], pa, b2, b3);
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  if constexpr (kProbe) {
    if (g < group)
      probe_flush(p.probe + (static_cast<size_t>(b) * p.n_q_heads + kvh * group + g) * 4, pacc);
  }

  // merge the 4 warps: shared scratch reuses the pipeline buffers
  __syncthreads();
  float* red_ml = reinterpret_cast<float*>(smem);            // [4 warps][4 rows][2]
  float* red_o = red_ml + 4 * 4 * 2;                          // [4 warps][4 rows][HD]
  l_run += __shfl_xor_sync(0xFFFFFFFFu, l_run, 1);
  l_run += __shfl_xor_sync(0xFFFFFFFFu, l_run, 2);
  if (g < group) {
    if (t4 == 0) {
      red_ml[(warp * 4 + g) * 2 + 0] = m_run;
      red_ml[(warp * 4 + g) * 2 + 1] = l_run;
    }
#pragma unroll
    for (int j = 0; j < ONT; ++j) {
      red_o[(warp * 4 + g) * HD + j * 8 + t4 * 2] = o[j][0];
      red_o[(warp * 4 + g) * HD + j * 8 + t4 * 2 + 1] = o[j][1];
    }
  }
  __syncthreads();
  for (int i = tid; i < group * HD; i += kDecThreads) {
    const int r = i / HD, d = i % HD;
    float mm = -INFINITY;
    for (int w = 0; w < 4; ++w) mm = fmaxf(mm, red_ml[(w * 4 + r) * 2]);
    const float mu = (mm == -INFINITY) ? 0.f : mm;
    float l = 0.f, acc = 0.f;
    for (int w = 0; w < 4; ++w) {
      const float f = exp2f(red_ml[(w * 4 + r) * 2] - mu);
      l += red_ml[(w * 4 + r) * 2 + 1] * f;
      acc += red_o[(w * 4 + r) * HD + d] * f;
    }
    const int head = kvh * group + r;
    const size_t pidx = (static_cast<size_t>(b) * p.n_q_heads + head) * n_splits + split;
    p.part_acc[pidx * HD + d] = acc;
    if (d == 0) {
      p.part_ml[pidx * 2 + 0] = mm;
      p.part_ml[pidx * 2 + 1] = l;
    }
  }
}

// merge the splits of one (sequence, query head), normalise, gate, store bf16
template <int HD>
__global__ void __launch_bounds__(HD) decode_combine_kernel(const DecodeAttnParams p, int n_splits) {
  const int head = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const size_t base = (static_cast<size_t>(b) * p.n_q_heads + head) * n_splits;
  float mm = -INFINITY;
  for (int s = 0; s < n_splits; ++s) mm = fmaxf(mm, p.part_ml[(base + s) * 2]);
  const float mu = (mm == -INFINITY) ? 0.f : mm;
  float l = 0.f, acc = 0.f;
  for (int s = 0; s < n_splits; ++s) {
    const float f = exp2f(p.part_ml[(base + s) * 2] - mu);
    l += p.part_ml[(base + s) * 2 + 1] * f;
    acc += p.part_acc[(base + s) * HD + d] * f;
  }
  const float gate = p.gate[static_cast<size_t>(b) * p.n_q_heads + head];
  const float v = l > 0.f ? acc / l * gate : 0.f;
  p.out[(static_cast<size_t>(b) * p.n_q_heads + head) * HD + d] = __float2bfloat16_rn(v);
}

template <int HD>
cudaError_t launch_decode_impl(const DecodeAttnParams& p, cudaStream_t s) {
  const int smem = kDecStages * 2 * kDecTile * HD * 2;
  auto kern = p.probe ? decode_attn_kernel<HD, true> : decode_attn_kernel<HD, false>;
  static uint32_t attr_done[2] = {0, 0};   // per instantiation, one bit per device < 32
  uint32_t& done = attr_done[p.probe ? 1 : 0];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 32 || !(done & (1u << dev))) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    if (dev < 32) done |= 1u << dev;
  }
  const int n_splits = decode_attention_splits(p.max_pos, p.window, p.split_keys);
  dim3 grid(n_splits, p.kv.n_kv, p.batch);
  kern<<<grid, kDecThreads, smem, s>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_decode_combine(p, n_splits, s);
}

}  // namespace

cudaError_t launch_decode_combine(const DecodeAttnParams& p, int n_splits, cudaStream_t s) {
  if (p.kv.hd == 128)
    decode_combine_kernel<128><<<dim3(p.n_q_heads, p.batch), 128, 0, s>>>(p, n_splits);
  else if (p.kv.hd == 64)
    decode_combine_kernel<64><<<dim3(p.n_q_heads, p.batch), 64, 0, s>>>(p, n_splits);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

int decode_attention_splits(int max_pos, int window, int split_keys) {
  const int max_keys = window > 0 ? (max_pos + 1 < window ? max_pos + 1 : window) : max_pos + 1;
  return (max_keys + split_keys - 1) / split_keys;
}

cudaError_t launch_decode_attention(const DecodeAttnParams& p, cudaStream_t s) {
  if (p.batch <= 0) return cudaSuccess;
  if (p.n_q_heads / p.kv.n_kv > 4 || p.split_keys % kDecTile != 0 || p.split_keys <= 0)
    return cudaErrorInvalidValue;
  if (p.kv.hd == 128) return launch_decode_impl<128>(p, s);
  if (p.kv.hd == 64) return launch_decode_impl<64>(p, s);
  return cudaErrorInvalidValue;
}

}  // namespace dory
