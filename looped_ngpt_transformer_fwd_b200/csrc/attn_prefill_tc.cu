// Prefill attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA)
// for head_dim 128: causal grouped-query attention, sliding-window or full,
// with the per-head sigmoid output gate ("Dory1.0-4B: A Looped
// Normalized-GPT", Methodology in Plain English).
//
// Softmax with a static maximum.  Queries and keys are L2-normalised per head
// and scaled by s_qk (the nGPT QK normalisation), so every logit obeys
//   |softmax_scale * q_hat . k_hat| <= softmax_scale * max_i s_qk[i]^2 =: B.
// softmax(x) = exp(x - c) / sum exp(x - c) holds for any constant c; with
// c = B every exponent lies in [-2B, 0], so no running maximum, no rescaling
// of the accumulator and no per-tile corrections are needed: P = exp2(x*log2e
// - B*log2e) is written as bf16 and O += P V accumulates in TMEM across all
// key tiles.  The host uses this kernel only when 2B*log2e < 120 (no
// underflow of the smallest weight in fp32/bf16); otherwise it keeps the
// online-softmax kernel.
//
// One CTA = 128 queries of one query head.  Warp 0 issues TMA loads (Q once,
// then 64-key K/V tiles through a 3-stage ring, from the layer's cache for
// positions below pos0 and from this call's fresh K/V otherwise), warp 1 owns
// TMEM and issues the MMAs (S = Q K^T into one of two 64-column TMEM buffers;
// O += P V into 128 columns), warps 2-5 turn S into P (one query row per
// thread: mask, exp2, row sum, bf16 store to shared memory) and finally write
// gate * O / l.  Every wait is bounded.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace dory {

namespace {

constexpr int kQ = 128;           // queries per CTA
constexpr int kKT = 64;           // keys per tile
constexpr int kHD = 128;
constexpr int kStages = 3;
constexpr int kThreads = 192;
constexpr int kQBytes = kQ * kHD * 2;                 // 32 KB (two 64-dim sub-tiles)
constexpr int kSubKV = kKT * 64 * 2;                  // 8 KB: 64 keys x 64 dims
constexpr int kStageBytes = 4 * kSubKV;               // K (2 sub-tiles) + V (2 sub-tiles)
constexpr int kPBytes = kQ * kKT * 2;                 // 16 KB
constexpr int kOffKV = kQBytes;
constexpr int kOffP = kOffKV + kStages * kStageBytes;
constexpr int kOffBar = kOffP + 2 * kPBytes;
constexpr int kSmemBytes = kOffBar + 256 + 1024;
constexpr uint32_t kTmemCols = 256;                   // S0 | S1 | O

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// K-major descriptor variant for the MN-major B operand (V, dims contiguous):
// SW128 atoms of 64 dims x 8 keys; LBO = distance between the two 64-dim
// sub-tiles, SBO = 1024 B between groups of 8 keys.
__device__ __forceinline__ uint64_t umma_desc_sw128_mn(uint32_t smem_addr, uint32_t lbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) return;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    prefill_attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                           const __grid_constant__ CUtensorMap tmKnew,
                           const __grid_constant__ CUtensorMap tmVnew,
                           const __grid_constant__ CUtensorMap tmCache,
                           const PrefillAttnTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;               // [kStages]
  uint64_t* kv_empty = kv_full + kStages;     // [kStages]
  uint64_t* s_full = kv_empty + kStages;      // [2]
  uint64_t* s_empty = s_full + 2;             // [2]
  uint64_t* p_full = s_empty + 2;             // [2]
  uint64_t* p_empty = p_full + 2;             // [2]
  uint64_t* o_full = p_empty + 2;
  uint64_t* drain = o_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.y;
  const int group = p.n_q_heads / p.n_kv;
  const int kvh = head / group;
  const int mblk = gridDim.x - 1 - blockIdx.x;        // heaviest query blocks first
  const int m0 = mblk * kQ;
  const int rows = min(kQ, p.n - m0);
  const int q_lo = p.pos0 + m0, q_hi = q_lo + rows - 1;
  const int key_lo = p.window > 0 ? max(0, q_lo - p.window + 1) : 0;
  const int kt_begin = key_lo / kKT, kt_end = q_hi / kKT;   // inclusive
  const int n_tiles = kt_end - kt_begin + 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_empty[b], 128);
      mbar_init(&p_full[b], 128);
      mbar_init(&p_empty[b], 1);
    }
    mbar_init(o_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmKnew);
    prefetch_tmap(&tmVnew);
    prefetch_tmap(&tmCache);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------- TMA producer
      bool ok = true;
      mbar_arrive_expect_tx(q_full, kQBytes);
      tma_load_3d(smem, &tmQ, q_full, 0, head, m0);
      tma_load_3d(smem + kQBytes / 2, &tmQ, q_full, 64, head, m0);
      int stage = 0;
      uint32_t phase = 0, issued = 0, parity_bits = 0;
      for (int j = 0; j < n_tiles; ++j) {
        if (!mbar_wait_bounded(&kv_empty[stage], phase ^ 1u, abort_flag, p.status)) {
          ok = false;
          break;
        }
        uint8_t* st = smem + kOffKV + stage * kStageBytes;
        const int kp0 = (kt_begin + j) * kKT;
        mbar_arrive_expect_tx(&kv_full[stage], kStageBytes);
        if (kp0 < p.pos0) {
          // cached positions: slot rows of this sequence's K and V planes
          const int slot = kp0 % p.cap;
          const int krow = (p.seq * 2 * p.n_kv + kvh) * p.cap + slot;
          const int vrow = krow + p.n_kv * p.cap;
          tma_load_2d(st, &tmCache, &kv_full[stage], 0, krow);
          tma_load_2d(st + kSubKV, &tmCache, &kv_full[stage], 64, krow);
          tma_load_2d(st + 2 * kSubKV, &tmCache, &kv_full[stage], 0, vrow);
          tma_load_2d(st + 3 * kSubKV, &tmCache, &kv_full[stage], 64, vrow);
        } else {
          const int t0 = kp0 - p.pos0;
          tma_load_3d(st, &tmKnew, &kv_full[stage], 0, kvh, t0);
          tma_load_3d(st + kSubKV, &tmKnew, &kv_full[stage], 64, kvh, t0);
          tma_load_3d(st + 2 * kSubKV, &tmVnew, &kv_full[stage], 0, kvh, t0);
          tma_load_3d(st + 3 * kSubKV, &tmVnew, &kv_full[stage], 64, kvh, t0);
        }
        issued |= 1u << stage;
        parity_bits = (parity_bits & ~(1u << stage)) | (phase << stage);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {
        drain_wait(q_full, 0);
        for (int s = 0; s < kStages; ++s)
          if (issued & (1u << s)) drain_wait(&kv_full[s], (parity_bits >> s) & 1u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc_s = umma_idesc_bf16(kQ, kKT);
      constexpr uint32_t idesc_o = umma_idesc_bf16(kQ, kHD) | (1u << 16);   // B (V) MN-major
      const uint32_t q_addr = smem_u32(smem);
      const uint32_t p_addr = smem_u32(smem + kOffP);
      bool ok = mbar_wait_bounded(q_full, 0, abort_flag, p.status);
      bool issued = false;
      int stage = 0;
      uint32_t phase = 0;
      int prev_stage = 0;
      for (int j = 0; ok && j <= n_tiles; ++j) {
        if (j < n_tiles) {
          const int buf = j & 1;
          const uint32_t use = j >> 1;
          if (!mbar_wait_bounded(&kv_full[stage], phase, abort_flag, p.status) ||
              !mbar_wait_bounded(&s_empty[buf], (use & 1u) ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(smem + kOffKV + stage * kStageBytes);
#pragma unroll
          for (int kk = 0; kk < kHD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * (kQBytes / 2) + (kk & 3) * 32;
            const uint32_t koff = (kk >> 2) * kSubKV + (kk & 3) * 32;
            umma_bf16(tmem + buf * kKT, umma_desc_sw128(q_addr + off),
                      umma_desc_sw128(k_addr + koff), idesc_s, kk > 0 ? 1u : 0u);
          }
          issued = true;
          umma_commit(&s_full[buf]);
        }
        if (j > 0) {
          // O += P_{j-1} V_{j-1}
          const int pj = j - 1;
          const int pbuf = pj & 1;
          const uint32_t puse = pj >> 1;
          if (!mbar_wait_bounded(&p_full[pbuf], puse & 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t v_addr = smem_u32(smem + kOffKV + prev_stage * kStageBytes) + 2 * kSubKV;
#pragma unroll
          for (int kk = 0; kk < kKT / 16; ++kk) {
            umma_bf16(tmem + 2 * kKT, umma_desc_sw128(p_addr + pbuf * kPBytes + kk * 32),
                      umma_desc_sw128_mn(v_addr + kk * 2048, kSubKV), idesc_o,
                      (pj > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&p_empty[pbuf]);
          umma_commit(&kv_empty[prev_stage]);
        }
        prev_stage = stage;
        if (j < n_tiles && ++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok) {
        umma_commit(o_full);
      } else if (issued) {
        umma_commit(drain);
        drain_wait(drain, 0);
      }
    }
  } else {
    // ----------------------------------------------------- softmax / output
    const int quad = warp & 3;
    const int r = quad * 32 + lane;                 // query row of this thread
    const int qp = q_lo + r;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    uint8_t* prow = smem + kOffP + r * 128;
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int buf = j & 1;
      const uint32_t use = j >> 1;
      // warp-uniform: the TMEM loads below are warp-collective
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(&s_full[buf], use & 1u, abort_flag, p.status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[kKT];
      {
        float t[32];
        tmem_ld32(tmem + lane_base + buf * kKT, t);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[i] = t[i];
        tmem_ld32(tmem + lane_base + buf * kKT + 32, t);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[32 + i] = t[i];
      }
      tc_fence_before();
      mbar_arrive(&s_empty[buf]);
      const int kp0 = (kt_begin + j) * kKT;
      const bool need_mask = (kp0 < key_lo) || (kp0 + kKT - 1 > q_lo) ||
                             (p.window > 0 && q_hi - kp0 >= p.window) || (kp0 + kKT - 1 > p.last_pos);
      uint32_t packed[kKT / 2];
#pragma unroll
      for (int i = 0; i < kKT; i += 2) {
        float e0 = ex2(fmaf(s[i], p.scale_log2, -p.m_log2));
        float e1 = ex2(fmaf(s[i + 1], p.scale_log2, -p.m_log2));
        if (need_mask) {
          const int k0 = kp0 + i, k1 = k0 + 1;
          const bool ok0 = k0 <= qp && (p.window <= 0 || qp - k0 < p.window);
          const bool ok1 = k1 <= qp && (p.window <= 0 || qp - k1 < p.window);
          e0 = ok0 ? e0 : 0.f;
          e1 = ok1 ? e1 : 0.f;
        }
        const uint32_t pk = pack_bf16x2(e0, e1);
        // the row sum uses the rounded weights, matching what the MMA multiplies
        l += bf16_lo(pk) + bf16_hi(pk);
        packed[i / 2] = pk;
      }
      if (j >= 2 && !__all_sync(0xFFFFFFFFu,
                                mbar_wait_bounded(&p_empty[buf], (use & 1u) ^ 1u, abort_flag, p.status))) {
        ok = false;
        break;
      }
      uint8_t* pb = prow + buf * kPBytes;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        *reinterpret_cast<uint4*>(pb + ((c ^ (r & 7)) << 4)) =
            make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&p_full[buf]);
    }
    if (ok && __all_sync(0xFFFFFFFFu, mbar_wait_bounded(o_full, 0, abort_flag, p.status))) {
      tc_fence_after();
      const bool row_ok = r < rows;
      const int t = m0 + r;
      const float scale = row_ok ? p.gate[static_cast<size_t>(t) * p.n_q_heads + head] / l : 0.f;
      __nv_bfloat16* dst = p.out + (static_cast<size_t>(t) * p.n_q_heads + head) * kHD;
#pragma unroll 1
      for (int c = 0; c < kHD; c += 32) {
        float o[32];
        tmem_ld32(tmem + lane_base + 2 * kKT + c, o);
        if (row_ok) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            d4[i] = make_uint4(pack_bf16x2(o[8 * i] * scale, o[8 * i + 1] * scale),
                               pack_bf16x2(o[8 * i + 2] * scale, o[8 * i + 3] * scale),
                               pack_bf16x2(o[8 * i + 4] * scale, o[8 * i + 5] * scale),
                               pack_bf16x2(o[8 * i + 6] * scale, o[8 * i + 7] * scale));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

bool make_tmap_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                  uint32_t box0, uint32_t box1, uint32_t box2) {
  using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
  static EncodeFn encode = nullptr;
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return false;
    encode = reinterpret_cast<EncodeFn>(fn);
  }
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {box0, box1, box2};
  cuuint32_t estr[3] = {1, 1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace

bool prefill_attention_tc_supported(int head_dim, int pos0, int window, float m_log2) {
  if (head_dim != kHD || pos0 % kKT != 0) return false;
  if (window > 0 && window % kKT != 0) return false;
  return 2.f * m_log2 < 120.f;
}

cudaError_t launch_prefill_attention_tc(const PrefillAttnTcParams& p, const __nv_bfloat16* q,
                                        const __nv_bfloat16* k_new, const __nv_bfloat16* v_new,
                                        const KvLayerView& kv, cudaStream_t s) {
  if (p.n <= 0) return cudaSuccess;
  CUtensorMap tq, tk, tv, tc;
  if (!make_tmap_3d(&tq, q, kHD, p.n_q_heads, p.n, 64, 1, kQ) ||
      !make_tmap_3d(&tk, k_new, kHD, p.n_kv, p.n, 64, 1, kKT) ||
      !make_tmap_3d(&tv, v_new, kHD, p.n_kv, p.n, 64, 1, kKT) ||
      !make_tmap_bf16(&tc, kv.k_base, static_cast<uint64_t>(kv.max_seqs) * 2 * kv.n_kv * kv.cap,
                      kHD, kKT))
    return cudaErrorInvalidValue;
  static uint32_t attr_done = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 32 || !(attr_done & (1u << dev))) {
    e = cudaFuncSetAttribute(prefill_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemBytes);
    if (e != cudaSuccess) return e;
    if (dev < 32) attr_done |= 1u << dev;
  }
  dim3 grid((p.n + kQ - 1) / kQ, p.n_q_heads);
  prefill_attn_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(tq, tk, tv, tc, p);
  return cudaGetLastError();
}

}  // namespace dory
