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
// One CTA = two adjacent 128-query tiles of one query head, sharing every K/V
// tile.  Warp 0 issues TMA loads (both Q tiles once, then 64-key K/V tiles
// through a 3-stage ring, from the layer's cache for positions below pos0 and
// from this call's fresh K/V otherwise), warp 1 owns TMEM and issues the MMAs
// (per query tile: S = Q K^T into one of two 64-column TMEM buffers, O += P V
// into 128 columns), and two softmax warpgroups (warps 2-5 and 6-9, one per
// query tile, so two warps share each SM sub-partition and hide each other's
// latency) turn S into P (one query row per thread: mask, exp2, row sum, bf16
// store to shared memory) and finally write gate * O / l.  Every wait is
// bounded.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace dory {

namespace {

constexpr int kQ = 128;           // queries per query tile
constexpr int kKT = 64;           // keys per tile
constexpr int kHD = 128;
constexpr int kStages = 3;
constexpr int kGroups = 2;        // query tiles (and softmax warpgroups) per CTA
constexpr int kThreads = 64 + kGroups * 128;
constexpr int kQBytes = kQ * kHD * 2;                 // 32 KB per query tile
constexpr int kSubKV = kKT * 64 * 2;                  // 8 KB: 64 keys x 64 dims
constexpr int kStageBytes = 4 * kSubKV;               // K (2 sub-tiles) + V (2 sub-tiles)
constexpr int kPBytes = kQ * kKT * 2;                 // 16 KB
constexpr int kOffKV = kGroups * kQBytes;
constexpr int kOffP = kOffKV + kStages * kStageBytes;
constexpr int kOffBar = kOffP + kGroups * 2 * kPBytes;
constexpr int kSmemBytes = kOffBar + 256 + 1024;
constexpr uint32_t kTmemCols = 512;                   // per group: S0 | S1 | O (256 columns)

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Descriptor of the MN-major B operand (V, dims contiguous): SW128 atoms of
// 64 dims x 8 keys; LBO = distance between the two 64-dim sub-tiles, SBO =
// 1024 B between groups of 8 keys.
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

// Query-tile geometry shared by every role of the CTA.
struct QTile {
  int m0, rows, q_lo, q_hi, kb, ke;   // key tiles kb..ke (inclusive)
  bool active;
};

__device__ __forceinline__ QTile make_qtile(const PrefillAttnTcParams& p, int qblock) {
  QTile t;
  t.m0 = qblock * kQ;
  t.rows = min(kQ, p.n - t.m0);
  t.active = t.rows > 0;
  t.q_lo = p.pos0 + t.m0;
  t.q_hi = t.q_lo + max(t.rows, 1) - 1;
  const int key_lo = p.window > 0 ? max(0, t.q_lo - p.window + 1) : 0;
  t.kb = key_lo / kKT;
  t.ke = t.q_hi / kKT;
  return t;
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
  uint64_t* kv_full = bars + 1;                 // [kStages]
  uint64_t* kv_empty = kv_full + kStages;       // [kStages]
  uint64_t* s_full = kv_empty + kStages;        // [group][2]
  uint64_t* s_empty = s_full + 2 * kGroups;     // [group][2]
  uint64_t* p_full = s_empty + 2 * kGroups;     // [group][2]
  uint64_t* p_empty = p_full + 2 * kGroups;     // [group][2]
  uint64_t* o_full = p_empty + 2 * kGroups;     // [group]
  uint64_t* drain = o_full + kGroups;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.y;
  const int group_size = p.n_q_heads / p.n_kv;
  const int kvh = head / group_size;
  const int pair = gridDim.x - 1 - blockIdx.x;        // heaviest query tiles first
  QTile qt[kGroups];
#pragma unroll
  for (int g = 0; g < kGroups; ++g) qt[g] = make_qtile(p, pair * kGroups + g);
  // key tiles of the CTA: the union of the tiles' ranges (later tiles reach further)
  const int kt_first = qt[0].kb;
  int kt_last = qt[0].ke;
#pragma unroll
  for (int g = 1; g < kGroups; ++g)
    if (qt[g].active) kt_last = max(kt_last, qt[g].ke);
  const int n_tiles = kt_last - kt_first + 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2 * kGroups; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_empty[b], 128);
      mbar_init(&p_full[b], 128);
      mbar_init(&p_empty[b], 1);
    }
    for (int g = 0; g < kGroups; ++g) mbar_init(&o_full[g], 1);
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
      int q_bytes = 0;
#pragma unroll
      for (int g = 0; g < kGroups; ++g) q_bytes += qt[g].active ? kQBytes : 0;
      mbar_arrive_expect_tx(q_full, q_bytes);
#pragma unroll
      for (int g = 0; g < kGroups; ++g) {
        if (!qt[g].active) continue;
        tma_load_3d(smem + g * kQBytes, &tmQ, q_full, 0, head, qt[g].m0);
        tma_load_3d(smem + g * kQBytes + kQBytes / 2, &tmQ, q_full, 64, head, qt[g].m0);
      }
      int stage = 0;
      uint32_t phase = 0, issued = 0, parity_bits = 0;
      for (int j = 0; j < n_tiles; ++j) {
        if (!mbar_wait_bounded(&kv_empty[stage], phase ^ 1u, abort_flag, p.status)) {
          ok = false;
          break;
        }
        uint8_t* st = smem + kOffKV + stage * kStageBytes;
        const int kp0 = (kt_first + j) * kKT;
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
      bool ok = mbar_wait_bounded(q_full, 0, abort_flag, p.status);
      bool issued = false;
      int stage = 0, prev_stage = 0;
      uint32_t phase = 0;
      for (int j = 0; ok && j <= n_tiles; ++j) {
        const int t = kt_first + j;
        if (j < n_tiles) {
          if (!mbar_wait_bounded(&kv_full[stage], phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          const uint32_t k_addr = smem_u32(smem + kOffKV + stage * kStageBytes);
#pragma unroll
          for (int g = 0; g < kGroups; ++g) {
            if (!qt[g].active || t < qt[g].kb || t > qt[g].ke) continue;
            const int i = t - qt[g].kb;                 // the group's own tile index
            const int buf = i & 1;
            if (!mbar_wait_bounded(&s_empty[2 * g + buf], ((i >> 1) & 1u) ^ 1u, abort_flag,
                                   p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t q_addr = smem_u32(smem + g * kQBytes);
#pragma unroll
            for (int kk = 0; kk < kHD / 16; ++kk) {
              const uint32_t off = (kk >> 2) * (kQBytes / 2) + (kk & 3) * 32;
              const uint32_t koff = (kk >> 2) * kSubKV + (kk & 3) * 32;
              umma_bf16(tmem + g * 256 + buf * kKT, umma_desc_sw128(q_addr + off),
                        umma_desc_sw128(k_addr + koff), idesc_s, kk > 0 ? 1u : 0u);
            }
            issued = true;
            umma_commit(&s_full[2 * g + buf]);
          }
          if (!ok) break;
        }
        if (j > 0) {
          // O_g += P_g V for the previous key tile
          const int tp = t - 1;
          const uint32_t v_addr = smem_u32(smem + kOffKV + prev_stage * kStageBytes) + 2 * kSubKV;
#pragma unroll
          for (int g = 0; g < kGroups; ++g) {
            if (!qt[g].active || tp < qt[g].kb || tp > qt[g].ke) continue;
            const int i = tp - qt[g].kb;
            const int buf = i & 1;
            if (!mbar_wait_bounded(&p_full[2 * g + buf], (i >> 1) & 1u, abort_flag, p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t p_addr = smem_u32(smem + kOffP + (2 * g + buf) * kPBytes);
#pragma unroll
            for (int kk = 0; kk < kKT / 16; ++kk) {
              umma_bf16(tmem + g * 256 + 2 * kKT, umma_desc_sw128(p_addr + kk * 32),
                        umma_desc_sw128_mn(v_addr + kk * 2048, kSubKV), idesc_o,
                        (i > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&p_empty[2 * g + buf]);
            if (tp == qt[g].ke) umma_commit(&o_full[g]);
          }
          if (!ok) break;
          umma_commit(&kv_empty[prev_stage]);
        }
        prev_stage = stage;
        if (j < n_tiles && ++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok && issued) {
        umma_commit(drain);
        drain_wait(drain, 0);
      }
    }
  } else {
    // ----------------------------------------------------- softmax / output
    const int g = (warp - 2) >> 2;                 // softmax warpgroup = query tile
    const QTile q = qt[g];
    const int quad = warp & 3;
    const int r = quad * 32 + lane;                // query row of this thread
    const int qp = q.q_lo + r;
    const uint32_t tbase = tmem + (static_cast<uint32_t>(quad * 32) << 16) + g * 256;
    uint8_t* prow = smem + kOffP + (2 * g) * kPBytes + r * 128;
    const float scale = p.scale_log2, moff = p.m_log2;
    float l = 0.f;
    bool ok = q.active;
    const int n_mine = q.active ? q.ke - q.kb + 1 : 0;
    for (int i = 0; ok && i < n_mine; ++i) {
      const int buf = i & 1;
      const uint32_t use = i >> 1;
      // warp-uniform: the TMEM loads below are warp-collective
      if (!__all_sync(0xFFFFFFFFu,
                      mbar_wait_bounded(&s_full[2 * g + buf], use & 1u, abort_flag, p.status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[kKT];
      {
        float t[32];
        tmem_ld32(tbase + buf * kKT, t);
#pragma unroll
        for (int c = 0; c < 32; ++c) s[c] = t[c];
        tmem_ld32(tbase + buf * kKT + 32, t);
#pragma unroll
        for (int c = 0; c < 32; ++c) s[32 + c] = t[c];
      }
      tc_fence_before();
      mbar_arrive(&s_empty[2 * g + buf]);
      const int kp0 = (q.kb + i) * kKT;
      const int key_lo = p.window > 0 ? max(0, q.q_lo - p.window + 1) : 0;
      const bool need_mask = (kp0 < key_lo) || (kp0 + kKT - 1 > q.q_lo) ||
                             (p.window > 0 && q.q_hi - kp0 >= p.window);
      uint32_t packed[kKT / 2];
      if (!need_mask) {
#pragma unroll
        for (int c = 0; c < kKT; c += 2) {
          const float e0 = ex2(fmaf(s[c], scale, -moff));
          const float e1 = ex2(fmaf(s[c + 1], scale, -moff));
          l += e0 + e1;
          packed[c / 2] = pack_bf16x2(e0, e1);
        }
      } else {
#pragma unroll
        for (int c = 0; c < kKT; c += 2) {
          const int k0 = kp0 + c, k1 = k0 + 1;
          const bool ok0 = k0 <= qp && (p.window <= 0 || qp - k0 < p.window);
          const bool ok1 = k1 <= qp && (p.window <= 0 || qp - k1 < p.window);
          const float e0 = ok0 ? ex2(fmaf(s[c], scale, -moff)) : 0.f;
          const float e1 = ok1 ? ex2(fmaf(s[c + 1], scale, -moff)) : 0.f;
          l += e0 + e1;
          packed[c / 2] = pack_bf16x2(e0, e1);
        }
      }
      if (i >= 2 && !__all_sync(0xFFFFFFFFu, mbar_wait_bounded(&p_empty[2 * g + buf],
                                                               (use & 1u) ^ 1u, abort_flag,
                                                               p.status))) {
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
      mbar_arrive(&p_full[2 * g + buf]);
    }
    if (ok && __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&o_full[g], 0, abort_flag, p.status))) {
      tc_fence_after();
      const bool row_ok = r < q.rows;
      const int t = q.m0 + r;
      const float f = row_ok ? p.gate[static_cast<size_t>(t) * p.n_q_heads + head] / l : 0.f;
      __nv_bfloat16* dst = p.out + (static_cast<size_t>(t) * p.n_q_heads + head) * kHD;
#pragma unroll 1
      for (int c = 0; c < kHD; c += 32) {
        float o[32];
        tmem_ld32(tbase + 2 * kKT + c, o);
        if (row_ok) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            d4[k] = make_uint4(pack_bf16x2(o[8 * k] * f, o[8 * k + 1] * f),
                               pack_bf16x2(o[8 * k + 2] * f, o[8 * k + 3] * f),
                               pack_bf16x2(o[8 * k + 4] * f, o[8 * k + 5] * f),
                               pack_bf16x2(o[8 * k + 6] * f, o[8 * k + 7] * f));
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
  dim3 grid((p.n + kGroups * kQ - 1) / (kGroups * kQ), p.n_q_heads);
  prefill_attn_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(tq, tk, tv, tc, p);
  return cudaGetLastError();
}

}  // namespace dory
