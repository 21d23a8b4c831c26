// Prefill attention for one layer of the looped nGPT stack: causal grouped-
// query attention, sliding-window (the last W keys, the query's own position
// included) or full, with the per-head sigmoid output gate applied to the
// result ("Dory1.0-4B: A Looped Normalized-GPT", Methodology in Plain English:
// GQA with input-dependent sigmoid output gates; SWA and full layers).
// Logits are softmax_scale * q_hat . k_hat of the already RoPE-rotated,
// normalised and s_qk-scaled queries and keys.
//
// Keys at positions below pos0 come from the layer's cache (ring slots
// pos % capacity for sliding-window layers); keys of this call come from the
// fresh buffer written by the QKVG projection, so a sliding-window ring can be
// committed after attention without clobbering keys this call still reads.
//
// FlashAttention-style: one CTA = 128 queries of one query head (8 warps x 16
// rows), 64-key K/V tiles double-buffered in shared memory with cp.async
// (XOR-swizzled 16-byte chunks), bf16 mma.sync with fp32 accumulation, online
// softmax in base 2, key tiles outside the window or past the diagonal never
// loaded.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace dory {

namespace {

constexpr int kAttnBM = 128;
constexpr int kAttnBN = 64;
constexpr int kAttnThreads = 256;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;   // 0 bytes read -> 16 zero bytes written
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

// byte offset of 16-byte chunk `c` of row `r` in a tile whose rows hold CH chunks
template <int CH>
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return static_cast<uint32_t>((r * CH + (c ^ (r & 7))) * 16);
}

// kProbe: also record the keys the softmax included (mask probe, diagnostics)
template <int HD, bool kProbe>
__global__ void __launch_bounds__(kAttnThreads, 2) prefill_attn_kernel(const PrefillAttnParams p) {
  constexpr int CH = HD / 8;               // 16-byte chunks per row
  constexpr int KSTEPS = HD / 16;          // mma k-steps over the head dimension
  constexpr int ONT = HD / 8;              // output n-tiles
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sK = sQ + kAttnBM * HD * 2;
  const uint32_t sV = sK + 2 * kAttnBN * HD * 2;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int head = blockIdx.y;
  const int group = p.n_q_heads / p.kv.n_kv;
  const int kvh = head / group;
  const int mblk = gridDim.x - 1 - blockIdx.x;     // heaviest (latest) query blocks first
  const int m0 = mblk * kAttnBM;
  const int rows = min(kAttnBM, p.n - m0);
  const int q_lo = p.pos0 + m0;                   // first query position of the block
  const int q_hi = q_lo + rows - 1;               // last
  const int key_lo = p.window > 0 ? max(0, q_lo - p.window + 1) : 0;
  const int kt_begin = key_lo / kAttnBN;
  const int kt_end = q_hi / kAttnBN;              // inclusive
  const int last_pos = p.pos0 + p.n - 1;

  // ---- async loads
  auto load_q = [&]() {
    for (int i = tid; i < kAttnBM * CH; i += kAttnThreads) {
      const int r = i / CH, c = i % CH;
      const bool ok = r < rows;
      const __nv_bfloat16* src =
          p.q + (static_cast<size_t>(m0 + (ok ? r : 0)) * p.n_q_heads + head) * HD + c * 8;
      cp_async16(sQ + swz<CH>(r, c), src, ok);
    }
  };
  auto load_kv = [&](int kt, int buf) {
    const uint32_t dk = sK + buf * kAttnBN * HD * 2, dv = sV + buf * kAttnBN * HD * 2;
    for (int i = tid; i < kAttnBN * CH; i += kAttnThreads) {
      const int r = i / CH, c = i % CH;
      const int kp = kt * kAttnBN + r;
      const bool ok = kp >= key_lo && kp <= last_pos;
      const __nv_bfloat16 *ks, *vs;
      if (ok && kp < p.pos0) {
        const size_t off = p.seq * p.kv.seq_stride +
                           (static_cast<size_t>(kvh) * p.kv.cap + kp % p.kv.cap) * HD + c * 8;
        ks = p.kv.k_base + off;
        vs = p.kv.v_base + off;
      } else {
        const size_t off =
            (static_cast<size_t>(ok ? kp - p.pos0 : 0) * p.kv.n_kv + kvh) * HD + c * 8;
        ks = p.k_new + off;
        vs = p.v_new + off;
      }
      cp_async16(dk + swz<CH>(r, c), ks, ok);
      cp_async16(dv + swz<CH>(r, c), vs, ok);
    }
  };

  load_q();
  load_kv(kt_begin, 0);
  cp_async_commit();

  float o[ONT][4];
#pragma unroll
  for (int j = 0; j < ONT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};

  const int g = lane >> 2, t4 = lane & 3;
  const int qrow0 = warp * 16 + g;                 // this thread's rows: qrow0, qrow0 + 8
  const int qpos[2] = {q_lo + qrow0, q_lo + qrow0 + 8};
  ProbeAcc pacc[2];
  probe_reset(pacc[0]);
  probe_reset(pacc[1]);

  for (int kt = kt_begin; kt <= kt_end; ++kt) {
    const int buf = (kt - kt_begin) & 1;
    if (kt < kt_end) {
      load_kv(kt + 1, buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t kb = sK + buf * kAttnBN * HD * 2, vb = sV + buf * kAttnBN * HD * 2;

    // S = Q K^T for 64 keys: 8 n-tiles of 8 keys
    float s[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
      uint32_t qa[4];   // Q fragment re-read from shared memory (keeps registers for O)
      {
        const int mtx = lane >> 3;
        const int r = warp * 16 + (lane & 7) + (mtx & 1) * 8;
        const int c = 2 * ks + (mtx >> 1);
        ldsm_x4(sQ + swz<CH>(r, c), qa[0], qa[1], qa[2], qa[3]);
      }
#pragma unroll
      for (int jp = 0; jp < 4; ++jp) {          // pairs of n-tiles (16 keys)
        const int mtx = lane >> 3;
        const int r = jp * 16 + (lane & 7) + (mtx >> 1) * 8;
        const int c = 2 * ks + (mtx & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + swz<CH>(r, c), b0, b1, b2, b3);
        mma_bf16(s[2 * jp], qa, b0, b1);
        mma_bf16(s[2 * jp + 1], qa, b2, b3);
      }
    }

    // scale, mask, online softmax
    const bool need_mask = (kt * kAttnBN < key_lo + 0) || ((kt + 1) * kAttnBN - 1 > q_lo) ||
                           (p.window > 0 && q_hi - kt * kAttnBN >= p.window);
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = s[j][e] * p.scale_log2;
        if (need_mask) {
          const int kp = kt * kAttnBN + j * 8 + t4 * 2 + (e & 1);
          const int qp = qpos[e >> 1];
          const bool ok = kp <= qp && kp >= 0 && (p.window <= 0 || qp - kp < p.window);
          v = ok ? v : -INFINITY;
        }
        s[j][e] = v;
        mx[e >> 1] = fmaxf(mx[e >> 1], v);
        if constexpr (kProbe) {
          if (v != -INFINITY) probe_add(pacc[e >> 1], kt * kAttnBN + j * 8 + t4 * 2 + (e & 1));
        }
      }
    }
    float corr[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xFFFFFFFFu, mx[h], 1));
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xFFFFFFFFu, mx[h], 2));
      const float m_new = fmaxf(m_run[h], mx[h]);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      corr[h] = exp2f(m_run[h] - m_use);
      m_run[h] = m_new;
      mx[h] = m_use;
    }
    float lsum[2] = {0.f, 0.f};
    uint32_t pa[4][4];    // P as bf16 A fragments, one per 16-key k-step
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float p0 = exp2f(s[j][0] - mx[0]), p1 = exp2f(s[j][1] - mx[0]);
      const float p2 = exp2f(s[j][2] - mx[1]), p3 = exp2f(s[j][3] - mx[1]);
      lsum[0] += p0 + p1;
      lsum[1] += p2 + p3;
      pa[j >> 1][(j & 1) * 2 + 0] = pack_bf16x2(p0, p1);
      pa[j >> 1][(j & 1) * 2 + 1] = pack_bf16x2(p2, p3);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) l_run[h] = l_run[h] * corr[h] + lsum[h];
#pragma unroll
    for (int j = 0; j < ONT; ++j) {
      o[j][0] *= corr[0]; o[j][1] *= corr[0];
      o[j][2] *= corr[1]; o[j][3] *= corr[1];
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int jp = 0; jp < ONT / 2; ++jp) {
        const int mtx = lane >> 3;
        const int r = kk * 16 + (lane & 7) + (mtx & 1) * 8;
        const int c = 2 * jp + (mtx >> 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vb + swz<CH>(r, c), b0, b1, b2, b3);
        mma_bf16(o[2 * jp], pa[kk], b0, b1);
        mma_bf16(o[2 * jp + 1], pa[kk], b2, b3);
      }
    }
    __syncthreads();
  }

  // finish: full row sums, normalise, gate, store bf16
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l_run[h] += __shfl_xor_sync(0xFFFFFFFFu, l_run[h], 1);
    l_run[h] += __shfl_xor_sync(0xFFFFFFFFu, l_run[h], 2);
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = qrow0 + h * 8;
    if (r >= rows) continue;
    const int t = m0 + r;
    if constexpr (kProbe)
      probe_flush(p.probe + (static_cast<size_t>(t) * p.n_q_heads + head) * 4, pacc[h]);
    const float scale = p.gate[static_cast<size_t>(t) * p.n_q_heads + head] / l_run[h];
    __nv_bfloat16* dst = p.out + (static_cast<size_t>(t) * p.n_q_heads + head) * HD;
#pragma unroll
    for (int j = 0; j < ONT; ++j) {
      const uint32_t v = pack_bf16x2(o[j][2 * h] * scale, o[j][2 * h + 1] * scale);
      *reinterpret_cast<uint32_t*>(dst + j * 8 + t4 * 2) = v;
    }
  }
}

template <int HD>
cudaError_t launch_prefill_impl(const PrefillAttnParams& p, cudaStream_t s) {
  const int smem = (kAttnBM + 4 * kAttnBN) * HD * 2;
  auto kern = p.probe ? prefill_attn_kernel<HD, true> : prefill_attn_kernel<HD, false>;
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
  dim3 grid((p.n + kAttnBM - 1) / kAttnBM, p.n_q_heads);
  kern<<<grid, kAttnThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_attention(const PrefillAttnParams& p, cudaStream_t s) {
  if (p.n <= 0) return cudaSuccess;
  if (p.kv.hd == 128) return launch_prefill_impl<128>(p, s);
  if (p.kv.hd == 64) return launch_prefill_impl<64>(p, s);
  return cudaErrorInvalidValue;
}

}  // namespace dory
