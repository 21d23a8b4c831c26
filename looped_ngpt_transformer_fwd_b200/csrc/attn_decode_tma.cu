// Decode attention v2 (head_dim 128; sliding windows a multiple of 64): the
// KV stream of one (split, KV head, sequence) is fed by TMA into a 3-stage
// ring of 64-key tiles (128-byte swizzle, K and V), one producer warp and four
// compute warps synchronised by mbarriers only.  Same maths as the split-KV
// kernel in attn_decode.cu ("Dory1.0-4B: A Looped Normalized-GPT",
// Methodology in Plain English: GQA with sigmoid output gates, sliding-window
// and full layers), reorganised for bandwidth:
//   * static softmax maximum: |logit| <= softmax_scale * max s_qk^2 (the
//     keys and queries are normalised and scaled by s_qk), so P = exp2(s*log2e
//     - m_log2) needs no running maximum and the splits merge by plain sums;
//   * S = Q K^T with the query heads of the KV head's group as the 16 MMA rows
//     (rows beyond the group are zero), then O^T = V^T P^T with 16 dims per MMA
//     and the group's heads as the 8 MMA columns, so the S accumulators feed
//     the second MMA directly and O needs only 32 registers per thread.
// Tiles are aligned to multiples of 64 positions so that no tile crosses the
// end of a sliding-window ring; V rows past the query position (slots that may
// never have been written) are zeroed in shared memory before use.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace dory {

namespace {

constexpr int kTile = 64;
constexpr int kStages = 3;
constexpr int kCompute = 4;                         // compute warps (16 keys each per tile)
constexpr int kThreads = 32 * (kCompute + 1);
constexpr int kHalf = kTile * 128;                  // 8 KB: 64 keys x 64 dims (one TMA box)
constexpr int kStageBytes = 4 * kHalf;              // K dims 0-63 | K 64-127 | V 0-63 | V 64-127
constexpr int kOffBar = kStages * kStageBytes;
constexpr int kSmemBytes = kOffBar + 128 + 1024;

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
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// byte offset of (key row r, 16-byte chunk c of 0..15) in a [64 keys x 128 dims]
// tile stored as two swizzled 64-dim halves
__device__ __forceinline__ uint32_t kv_off(int r, int c) {
  return static_cast<uint32_t>((c >> 3) * kHalf + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// kProbe: also record the keys given a nonzero weight (mask probe, diagnostics)
template <bool kProbe>
__global__ void __launch_bounds__(kThreads, 2)
    decode_attn_tma_kernel(const __grid_constant__ CUtensorMap tmCache, const DecodeAttnParams p,
                           int split_tiles, float m_log2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* empty = full + kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kStages);

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int n_splits = gridDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int group = p.n_q_heads / p.kv.n_kv;
  const int cap = p.kv.cap;

  const int seq = p.d_seq[b];
  const int pos = p.d_pos[b];
  const bool bad = seq < 0 || seq >= p.kv.max_seqs || pos < 0 || pos >= p.kv.max_ctx ||
                   pos > p.max_pos;
  if (bad && threadIdx.x == 0 && split == 0 && kvh == 0) report_status(p.status, kStatusBounds);
  const int lo = bad ? 0 : (p.window > 0 ? max(0, pos - p.window + 1) : 0);
  const int last_tile = bad ? -1 : pos / kTile;
  const int t_begin = lo / kTile + split * split_tiles;
  const int t_end = min(last_tile, t_begin + split_tiles - 1);
  const int n_tiles = max(0, t_end - t_begin + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCompute);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
    fence_proxy_async_smem();
  }
  __syncthreads();

  float o[8][4];   // O^T: 8 tiles of 16 dims; rows dims (g, g+8), columns heads (2*t4, 2*t4+1)
  float l = 0.f;   // this thread's partial row sum for head g
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

  if (warp == kCompute) {
    if (lane == 0 && n_tiles > 0) {
      // ----------------------------------------------------- TMA producer
      prefetch_tmap(&tmCache);
      const int krow0 = (seq * 2 * p.kv.n_kv + kvh) * cap;
      const int vrow0 = krow0 + p.kv.n_kv * cap;
      int stage = 0;
      uint32_t phase = 0, issued = 0, parity_bits = 0;
      bool ok = true;
      for (int j = 0; j < n_tiles; ++j) {
        if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.status)) {
          ok = false;
          break;
        }
        const int slot = ((t_begin + j) * kTile) % cap;
        uint8_t* st = smem + stage * kStageBytes;
        mbar_arrive_expect_tx(&full[stage], kStageBytes);
        tma_load_2d(st, &tmCache, &full[stage], 0, krow0 + slot);
        tma_load_2d(st + kHalf, &tmCache, &full[stage], 64, krow0 + slot);
        tma_load_2d(st + 2 * kHalf, &tmCache, &full[stage], 0, vrow0 + slot);
        tma_load_2d(st + 3 * kHalf, &tmCache, &full[stage], 64, vrow0 + slot);
        issued |= 1u << stage;
        parity_bits = (parity_bits & ~(1u << stage)) | (phase << stage);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {
        for (int s = 0; s < kStages; ++s)
          if (issued & (1u << s)) drain_wait(&full[s], (parity_bits >> s) & 1u);
      }
    }
  } else {
    // ------------------------------------------------------- compute warps
    // Q fragments (A operand of S = Q K^T): rows = heads of the group
    uint32_t qa[8][2];
    {
      const bool live = g < group;
      const __nv_bfloat16* q =
          p.q + (static_cast<size_t>(b) * p.n_q_heads + kvh * group + (live ? g : 0)) * 128;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        qa[ks][0] = live ? *reinterpret_cast<const uint32_t*>(q + ks * 16 + t4 * 2) : 0u;
        qa[ks][1] = live ? *reinterpret_cast<const uint32_t*>(q + ks * 16 + 8 + t4 * 2) : 0u;
      }
    }
    const int key0 = warp * 16;
    int stage = 0;
    uint32_t phase = 0;
    ProbeAcc pacc;
    probe_reset(pacc);
    for (int j = 0; j < n_tiles; ++j) {
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[stage], phase, abort_flag, p.status)))
        break;
      const uint32_t kb = smem_u32(smem + stage * kStageBytes);
      const uint32_t vb = kb + 2 * kHalf;
      const int kp0 = (t_begin + j) * kTile + key0;   // position of this warp's first key
      if (kp0 + 15 > pos) {
        // keys past the query: their V rows may never have been written
        uint8_t* vrow = smem + stage * kStageBytes + 2 * kHalf;
        for (int i = lane; i < 16 * 16; i += 32) {
          const int r = key0 + (i >> 4), c = i & 15;
          if ((t_begin + j) * kTile + r > pos)
            *reinterpret_cast<uint4*>(vrow + kv_off(r, c)) = make_uint4(0u, 0u, 0u, 0u);
        }
        __syncwarp();
        // order these generic-proxy writes before the next TMA refill of the stage
        fence_proxy_async_smem();
      }
      // S = Q K^T for this warp's 16 keys (two n-tiles of 8 keys)
      float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int mtx = lane >> 3;
        const int r = key0 + (lane & 7) + (mtx >> 1) * 8;
        const int c = 2 * ks + (mtx & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + kv_off(r, c), b0, b1, b2, b3);
        mma_bf16(s[0], qa[ks][0], 0u, qa[ks][1], 0u, b0, b1);
        mma_bf16(s[1], qa[ks][0], 0u, qa[ks][1], 0u, b2, b3);
      }
      // P = exp2(S * scale - m) on the valid keys (row g = head g of the group)
      float pv[2][2];
#pragma unroll
      for (int n = 0; n < 2; ++n) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int kp = kp0 + n * 8 + t4 * 2 + e;
          const bool ok = kp >= lo && kp <= pos;
          pv[n][e] = ok ? ex2(fmaf(s[n][e], p.scale_log2, -m_log2)) : 0.f;
          l += pv[n][e];
          if constexpr (kProbe) {
            if (pv[n][e] > 0.f) probe_add(pacc, kp);
          }
        }
      }
      const uint32_t pb0 = pack_bf16x2(pv[0][0], pv[0][1]);
      const uint32_t pb1 = pack_bf16x2(pv[1][0], pv[1][1]);
      // O^T += V^T P^T: 8 tiles of 16 dims; A = V^T from the V tile (transposed loads)
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const int mtx = lane >> 3;
        const int r = key0 + (lane & 7) + (mtx >> 1) * 8;
        const int c = 2 * mt + (mtx & 1);
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(vb + kv_off(r, c), a0, a1, a2, a3);
        mma_bf16(o[mt], a0, a1, a2, a3, pb0, pb1);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
      if (++stage == kStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if constexpr (kProbe) {
      if (g < group)
        probe_flush(p.probe + (static_cast<size_t>(b) * p.n_q_heads + kvh * group + g) * 4, pacc);
    }
  }

  // merge the compute warps (plain sums: every split and warp shares m_log2)
  __syncthreads();
  float* red_l = reinterpret_cast<float*>(smem);                 // [warps][8 heads]
  float* red_o = red_l + kCompute * 8;                            // [warps][8 heads][128]
  if (warp < kCompute) {
    l += __shfl_xor_sync(0xFFFFFFFFu, l, 1);
    l += __shfl_xor_sync(0xFFFFFFFFu, l, 2);
    if (t4 == 0 && g < 8) red_l[warp * 8 + g] = l;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int head = t4 * 2 + (e & 1);
        const int dim = mt * 16 + g + (e >> 1) * 8;
        if (head < group) red_o[(warp * 8 + head) * 128 + dim] = o[mt][e];
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < group * 128; i += kThreads) {
    const int hh = i >> 7, dim = i & 127;
    float acc = 0.f, ls = 0.f;
#pragma unroll
    for (int w = 0; w < kCompute; ++w) {
      acc += red_o[(w * 8 + hh) * 128 + dim];
      ls += red_l[w * 8 + hh];
    }
    const size_t pidx = (static_cast<size_t>(b) * p.n_q_heads + kvh * group + hh) * n_splits + split;
    p.part_acc[pidx * 128 + dim] = acc;
    if (dim == 0) {
      p.part_ml[pidx * 2 + 0] = m_log2;
      p.part_ml[pidx * 2 + 1] = ls;
    }
  }
}

}  // namespace

bool decode_attention_tma_supported(int head_dim, int window, int group) {
  return head_dim == 128 && (window <= 0 || window % kTile == 0) && group <= 8;
}

int decode_attention_tma_splits(int max_pos, int window, int* split_tiles) {
  const int max_keys = window > 0 ? (max_pos + 1 < window ? max_pos + 1 : window) : max_pos + 1;
  const int tiles = (max_keys + kTile - 1) / kTile + 1;   // +1: alignment to 64 positions
  int st = (tiles + 63) / 64;
  if (st < 8) st = 8;
  *split_tiles = st;
  return (tiles + st - 1) / st;
}

cudaError_t launch_decode_attention_tma(const DecodeAttnParams& p, float m_log2,
                                        cudaStream_t s) {
  if (p.batch <= 0) return cudaSuccess;
  CUtensorMap tc;
  if (!make_tmap_bf16(&tc, p.kv.k_base,
                      static_cast<uint64_t>(p.kv.max_seqs) * 2 * p.kv.n_kv * p.kv.cap, 128, kTile))
    return cudaErrorInvalidValue;
  static uint32_t attr_done = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 32 || !(attr_done & (1u << dev))) {
    e = cudaFuncSetAttribute(decode_attn_tma_kernel<false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(decode_attn_tma_kernel<true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    if (dev < 32) attr_done |= 1u << dev;
  }
  int split_tiles = 0;
  const int n_splits = decode_attention_tma_splits(p.max_pos, p.window, &split_tiles);
  dim3 grid(n_splits, p.kv.n_kv, p.batch);
  if (p.probe)
    decode_attn_tma_kernel<true><<<grid, kThreads, kSmemBytes, s>>>(tc, p, split_tiles, m_log2);
  else
    decode_attn_tma_kernel<false><<<grid, kThreads, kSmemBytes, s>>>(tc, p, split_tiles, m_log2);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_decode_combine(p, n_splits, s);
}

}  // namespace dory
