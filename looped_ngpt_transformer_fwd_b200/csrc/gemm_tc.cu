// Persistent tcgen05 GEMM for sm_100a: C = A * B^T with bf16 operands fed by
// TMA (128-byte swizzle), fp32 accumulators in TMEM (double-buffered so the
// epilogue of one tile overlaps the main loop of the next), and fused
// epilogues for the projections of a looped nGPT block:
//   - kEpiQKVG: the fused QKV + gate projection of the attention sublayer
//     ("Dory1.0-4B: A Looped Normalized-GPT", Methodology in Plain English:
//     GQA with sigmoid output gates, RoPE per layer type), with the nGPT
//     query/key normalisation q_hat = s_qk * Norm(RoPE(q)) per head;
//   - kEpiSwiGLU: the gate/up projection with SiLU(gate) * up (same section);
//   - kEpiStoreF32: plain fp32 output (output and down projections, whose
//     nGPT update needs whole-row norms and runs in the row kernel).
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 owns TMEM and
// issues the MMAs, warps 2..5 run the epilogue (one TMEM lane = one output row
// per thread).  Every wait is bounded (see common.cuh); on expiry the kernel
// records kStatusTimeout, drains its outstanding copies and MMAs, frees TMEM
// and returns.
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"

namespace dory {

namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kGemmThreads = 192;

// MX = kOperandsBf16: bf16 operands, 64 K per stage.  kOperandsMxfp8: E4M3
// codes with one E8M0 scale per 32 along K, 128 K per stage (the same 128
// bytes per row).  kOperandsNvfp4: packed E2M1 codes with one E4M3 scale per
// 16 along K, 256 K per stage (again 128 bytes per row).  The block-scaled
// forms stage the step's scale chunks in shared memory after the tiles and
// copy them to TMEM for the MMAs.
template <int BN, int MX = kOperandsBf16>
struct GemmCfg {
  static constexpr bool kNv = MX == kOperandsNvfp4;
  static constexpr int kStages = MX ? (BN == 256 ? 3 : 5) : ((BN == 256) ? 4 : 6);
  static constexpr int kKStep = kNv ? 256 : (MX ? 128 : kBK);   // K elements per stage
  // the stage's step of the tensor maps' x coordinate, in map elements (bf16
  // values, or bytes of codes: 128 per row and stage in both block-scaled forms)
  static constexpr int kKCoord = MX ? 128 : kBK;
  static constexpr int kABytes = kBM * 128;
  static constexpr int kBBytes = BN * 128;
  // scale bytes per 128 rows and stage: 128 x 4 (MXFP8), 128 x 16 (NVFP4)
  static constexpr int kSfChunk = kNv ? 2048 : (MX ? 512 : 0);
  static constexpr int kSfaBytes = kSfChunk;
  static constexpr int kSfbBytes = kSfChunk * (BN / 128);
  // bytes the TMA and bulk copies of one stage deliver (the mbarrier's
  // transaction count), and the stage's footprint, padded to keep every
  // stage's tiles 1024-byte aligned
  static constexpr int kLoadBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
  static constexpr int kStageBytes = (kLoadBytes + 1023) / 1024 * 1024;
  // accumulators (kAccBufs x BN columns), then per stage the A and B scale
  // columns (MXFP8: one 32-bit word per row holds the stage's four scales;
  // NVFP4: one word per row and 64-K MMA); a 256-column block-scaled tile
  // keeps a single accumulator so that the scale columns fit next to it
  static constexpr int kAccBufs = (MX && BN == 256) ? 1 : 2;
  static constexpr int kSfCols = (kNv ? 16 : 4) * (1 + BN / 128);
  static constexpr int kTmemCols = MX ? 512 : 2 * BN;
  static_assert(!MX || kAccBufs * BN + kStages * kSfCols <= 512, "TMEM columns");
  static_assert(kStageBytes % 1024 == 0, "stages keep the tiles 1024-byte aligned");
  // fp32 output staging for bulk tensor stores: 4 epilogue warps x 2 buffers
  // of 32 rows x 32 columns
  static constexpr int kOutBufBytes = 32 * 32 * 4;
  static constexpr int kOutStageBytes = 4 * 2 * kOutBufBytes;
  static constexpr int kBarBytes = 256;
  static constexpr int kSqkBytes = 512;   // s_qk (head_dim <= 128 floats) for the QKVG epilogue
  static constexpr int kSmemBytes =
      kStages * kStageBytes + kOutStageBytes + kBarBytes + kSqkBytes + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory per block");
};

// Output tensor maps of one launch: fp32 output ([0]), or q / k / v for the
// QKVG epilogue, or the activations ([0]) for SwiGLU.
struct OutMaps {
  CUtensorMap m[3];
};

// Bulk tensor store of one staged box (shared -> global, no multicast) and
// the bulk-group bookkeeping around it.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int32_t c0,
                                             int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int32_t c0,
                                             int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// at most one bulk group may still be reading shared memory
__device__ __forceinline__ void bulk_wait_read_1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// ------------------------------------------------------- MXFP8 (block-scaled) MMA
// Plain bulk copy global -> shared, counted on an mbarrier (16-byte multiples).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// Shared-memory descriptor of one 512-byte scale chunk read by tcgen05.cp as
// 32 rows of 16 bytes: no swizzle, 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t sf_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(128u >> 4) << 16;    // leading byte offset (one core matrix wide)
  d |= static_cast<uint64_t>(128u >> 4) << 32;    // stride byte offset: next 8 rows
  d |= static_cast<uint64_t>(1u) << 46;           // descriptor version
  return d;                                       // layout type 0: no swizzle
}
// 32 TMEM lanes x 128 bits from shared memory, repeated in all four 32-lane groups
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}
// Instruction descriptor of tcgen05.mma kind::mxf8f6f4 with block scaling: E4M3
// A and B (K-major), E8M0 scales, fp32 accumulation, scale byte `sf` of each
// 32-bit scale column for both operands.
__host__ __device__ constexpr uint32_t umma_idesc_mxf8(int M, int N, int sf) {
  return (static_cast<uint32_t>(sf) << 4)          // B scale factor id
         | (0u << 7) | (0u << 10)                  // A, B format: E4M3
         | (static_cast<uint32_t>(N >> 3) << 17)   // N / 8
         | (1u << 23)                              // scale format: E8M0
         | (static_cast<uint32_t>(M >> 4) << 24)   // M / 16
         | (static_cast<uint32_t>(sf) << 29);      // A scale factor id
}
__device__ __forceinline__ void umma_mxf8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// Instruction descriptor of tcgen05.mma kind::mxf4nvf4 with block scaling:
// E2M1 A and B (K-major, packed two per byte), UE4M3 scales, one per 16 along
// K (scale_vec::4X: the four scales of a 64-K step fill a 32-bit word, so the
// scale factor ids stay 0), fp32 accumulation.
__host__ __device__ constexpr uint32_t umma_idesc_nvf4(int M, int N) {
  return (1u << 7) | (1u << 10)                    // A, B format: E2M1
         | (static_cast<uint32_t>(N >> 3) << 17)   // N / 8
         | (0u << 23)                              // scale format: UE4M3
         | (static_cast<uint32_t>(M >> 4) << 24);  // M / 16
}
__device__ __forceinline__ void umma_nvf4(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// --------------------------------------------------------------- epilogues
// Accumulators times the tensor-scale product alpha (NVFP4 operands only).
template <bool kAlpha, int N>
__device__ __forceinline__ void apply_alpha(float (&v)[N], float alpha) {
  if constexpr (kAlpha) {
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] *= alpha;
  }
}

__device__ __forceinline__ void store_f32_chunk(float* dst, const float (&v)[32], int valid) {
  // vector stores only where the row start allows them (any row pitch works)
  if (valid >= 32 && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
    float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int i = 0; i < 8; ++i) d4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  } else {
    const int n = valid < 32 ? valid : 32;
    for (int i = 0; i < n; ++i) dst[i] = v[i];
  }
}

// Accumulators plus the tail's partial (when there is one).
__device__ __forceinline__ void add_partial(float (&v)[32], const float* part, int c) {
  if (part) {
    // from L2 (another SM wrote it)
    const float4* s4 = reinterpret_cast<const float4*>(part + c);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 t = __ldcg(s4 + i);
      v[4 * i] += t.x; v[4 * i + 1] += t.y; v[4 * i + 2] += t.z; v[4 * i + 3] += t.w;
    }
  }
}

// `part`: this lane's row of a stream-K tail partial to add, or nullptr.
template <int BN, bool kAlpha>
__device__ __forceinline__ void epi_store_f32(const GemmParams& p, uint32_t taddr, int row, int nt,
                                              int ks, const float* part) {
  float* out = p.out_f32 + static_cast<size_t>(ks) * p.split_stride;
  const bool row_ok = row < p.M;
#pragma unroll 1
  for (int c = 0; c < BN; c += 32) {
    float v[32];
    tmem_ld32(taddr + c, v);
    add_partial(v, part, c);
    apply_alpha<kAlpha>(v, p.alpha);
    const int col = nt * BN + c;
    if (row_ok && col < p.N)
      store_f32_chunk(out + static_cast<size_t>(row) * p.ld_out + col, v, p.N - col);
  }
}

// fp32 output through shared memory and bulk tensor stores: each warp stages
// its 32 rows x 32 columns with the 128-byte swizzle (16-byte chunk j of row r
// at chunk j ^ (r % 8), conflict-free) and one lane stores the box; the tensor
// map [splits][M][N] clips rows past M and columns past N.  Two buffers per
// warp alternate so staging overlaps the previous store.
template <int BN, bool kAlpha>
__device__ __forceinline__ void epi_store_f32_tma(const GemmParams& p, const CUtensorMap* tmC,
                                                  uint32_t taddr, uint8_t* stage, int lane,
                                                  int row0, int nt, int ks, uint32_t& nbuf,
                                                  const float* part) {
#pragma unroll 1
  for (int c = 0; c < BN; c += 32) {
    float v[32];
    tmem_ld32(taddr + c, v);
    add_partial(v, part, c);
    apply_alpha<kAlpha>(v, p.alpha);
    const int col = nt * BN + c;
    if (col >= p.N) continue;                   // warp-uniform
    uint8_t* buf = stage + (nbuf & 1u) * (32 * 32 * 4);
    if (lane == 0) bulk_wait_read_1();          // the store that last read `buf` is done
    __syncwarp();
    float4* rowp = reinterpret_cast<float4*>(buf + lane * 128);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      rowp[j ^ (lane & 7)] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    fence_proxy_async_smem();                   // generic-proxy writes -> bulk copy
    __syncwarp();
    if (lane == 0) {
      tma_store_3d(tmC, buf, col, row0, ks);
      bulk_commit();
    }
    ++nbuf;
  }
}

// Stage this lane's row of a 32-row x 64-column bf16 box (32 packed words,
// 128-byte swizzle) and store the box at (x, y) through `map`.  The warp's two
// staging buffers alternate; `nbuf` counts the boxes.
__device__ __forceinline__ void store_box_bf16(const CUtensorMap* map, uint8_t* stage, int lane,
                                               uint32_t& nbuf, const uint32_t (&w)[32], int x,
                                               int y) {
  uint8_t* buf = stage + (nbuf & 1u) * (32 * 32 * 4);
  if (lane == 0) bulk_wait_read_1();          // the store that last read `buf` is done
  __syncwarp();
  uint4* rowp = reinterpret_cast<uint4*>(buf + lane * 128);
#pragma unroll
  for (int j = 0; j < 8; ++j)
    rowp[j ^ (lane & 7)] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(map, buf, x, y);
    bulk_commit();
  }
  ++nbuf;
}

// SwiGLU activations in 64-column boxes through bulk tensor stores (rows past
// M are clipped by the tensor map).
template <int BN, bool kAlpha>
__device__ __forceinline__ void epi_swiglu_tma(const GemmParams& p, const CUtensorMap* map,
                                               uint32_t taddr, uint8_t* stage, int lane, int row0,
                                               int nt, uint32_t& nbuf) {
  constexpr int H = BN / 2;
  static_assert(H % 64 == 0, "activation boxes are 64 columns wide");
#pragma unroll 1
  for (int c = 0; c < H; c += 64) {
    uint32_t w[32];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float g[32], u[32];
      tmem_ld32(taddr + c + 32 * half, g);
      tmem_ld32(taddr + H + c + 32 * half, u);
      apply_alpha<kAlpha>(g, p.alpha);
      apply_alpha<kAlpha>(u, p.alpha);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float g0 = p.gate_scale * g[2 * i], g1 = p.gate_scale * g[2 * i + 1];
        const float a0 = g0 * sigmoidf_(g0) * u[2 * i];
        const float a1 = g1 * sigmoidf_(g1) * u[2 * i + 1];
        w[16 * half + i] = pack_bf16x2(a0, a1);
      }
    }
    store_box_bf16(map, stage, lane, nbuf, w, nt * H + c, row0);
  }
}

template <int BN, bool kAlpha>
__device__ __forceinline__ void epi_swiglu(const GemmParams& p, uint32_t taddr, int row, int nt) {
  constexpr int H = BN / 2;
  const bool row_ok = row < p.M;
  __nv_bfloat16* out = p.out_act + static_cast<size_t>(row) * p.ld_act + nt * H;
#pragma unroll 1
  for (int c = 0; c < H; c += 32) {
    float g[32], u[32];
    tmem_ld32(taddr + c, g);
    tmem_ld32(taddr + H + c, u);
    if (!row_ok) continue;
    apply_alpha<kAlpha>(g, p.alpha);
    apply_alpha<kAlpha>(u, p.alpha);
    uint32_t packed[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float g0 = p.gate_scale * g[2 * i], g1 = p.gate_scale * g[2 * i + 1];
      const float a0 = g0 * sigmoidf_(g0) * u[2 * i];
      const float a1 = g1 * sigmoidf_(g1) * u[2 * i + 1];
      packed[i] = pack_bf16x2(a0, a1);
    }
    uint4* d4 = reinterpret_cast<uint4*>(out + c);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      d4[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
  }
}

// 32 fp32 values per lane to TMEM columns taddr..taddr+31 (this warp's lanes),
// then wait until they are written.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]),
      "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]),
      "f"(v[15]), "f"(v[16]), "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]),
      "f"(v[22]), "f"(v[23]), "f"(v[24]), "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]),
      "f"(v[29]), "f"(v[30]), "f"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// One head-sized column group (HD columns starting at global column col0).
// q and k heads get RoPE, the per-head L2 norm and the scale s_qk (`sqk`, in
// shared memory); v heads are stored as computed; gate logits go through the
// sigmoid.  q / k take two passes over the accumulator columns, which this
// warp owns until it releases the buffer: the first rotates 32 pairs (i,
// i + HD/2) at a time, adds their squares and writes them back, the second
// scales by s_qk / ||.|| and stores, so no more than 64 values are live.  The
// RoPE table is pair-major ([HD/2][M]): for one pair the 32 lanes (32
// consecutive rows) read 256 contiguous bytes.  With bulk stores (p.c_tma) the
// warp stages 64-column boxes of q, k or v and every lane takes part, rows past
// M included (the maps clip them).  TMEM accesses are warp-collective: every
// lane runs them, whatever its row.
template <int HD, bool kAlpha>
__device__ __forceinline__ void epi_qkvg_group(const GemmParams& p, const float* sqk,
                                               const OutMaps* om, uint8_t* stage, int lane,
                                               int row0, uint32_t& nbuf, uint32_t taddr, int row,
                                               int col0) {
  const int hq = p.n_q_heads, hkv = p.n_kv_heads;
  const int q_end = hq * HD, k_end = q_end + hkv * HD, v_end = k_end + hkv * HD;
  const bool tma = p.c_tma != 0;
  const bool row_ok = row < p.M;
  if (col0 >= v_end) {
    // attention output gate logits, one per query head (col0 is warp-uniform)
    float* g = p.gate_out + static_cast<size_t>(row) * hq;
#pragma unroll 1
    for (int c = 0; c < HD && col0 - v_end + c < hq; c += 32) {
      float t[32];
      tmem_ld32(taddr + c, t);
      apply_alpha<kAlpha>(t, p.alpha);
      if (!row_ok) continue;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int j = col0 - v_end + c + i;
        if (j < hq) g[j] = sigmoidf_(t[i]);
      }
    }
    return;
  }
  int which, head;
  float inv = 1.f;
  const bool qk = col0 < k_end;
  if (qk) {
    // rows past M read the last valid row's angles (their results are clipped)
    const int trow = row_ok ? row : p.M - 1;
    float ss = 0.f;
#pragma unroll 1
    for (int c = 0; c < HD / 2; c += 32) {
      float a[32], b[32];
      tmem_ld32(taddr + c, a);
      tmem_ld32(taddr + c + HD / 2, b);
      apply_alpha<kAlpha>(a, p.alpha);
      apply_alpha<kAlpha>(b, p.alpha);
      const float2* rt = p.rope + static_cast<size_t>(c) * p.M + trow;
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const float2 cs = rt[static_cast<size_t>(u) * p.M];   // cos_i, sin_i of pair c + u
        const float a2 = a[u] * cs.x - b[u] * cs.y;
        const float b2 = b[u] * cs.x + a[u] * cs.y;
        ss = fmaf(a2, a2, fmaf(b2, b2, ss));
        a[u] = a2;
        b[u] = b2;
      }
      tmem_st32(taddr + c, a);
      tmem_st32(taddr + c + HD / 2, b);
    }
    tmem_wait_st();
    inv = rsqrtf(fmaxf(ss, p.norm_eps));
    which = col0 < q_end ? 0 : 1;
    head = col0 < q_end ? col0 / HD : (col0 - q_end) / HD;
  } else {
    which = 2;
    head = (col0 - k_end) / HD;
  }
  const int nh = which == 0 ? hq : hkv;
  __nv_bfloat16* base = which == 0 ? p.q_out : (which == 1 ? p.k_out : p.v_out);
#pragma unroll 1
  for (int half = 0; half < HD / 64; ++half) {
    uint32_t wb[32];
#pragma unroll
    for (int cc = 0; cc < 64; cc += 32) {
      float t[32];
      tmem_ld32(taddr + 64 * half + cc, t);
      if (qk) {
#pragma unroll
        for (int u = 0; u < 32; ++u) t[u] *= inv * sqk[64 * half + cc + u];
      } else {
        apply_alpha<kAlpha>(t, p.alpha);
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) wb[cc / 2 + u] = pack_bf16x2(t[2 * u], t[2 * u + 1]);
    }
    if (tma) {
      store_box_bf16(&om->m[which], stage, lane, nbuf, wb, head * HD + 64 * half, row0);
    } else if (row_ok) {
      uint4* d4 = reinterpret_cast<uint4*>(base + (static_cast<size_t>(row) * nh + head) * HD +
                                           64 * half);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        d4[i] = make_uint4(wb[4 * i], wb[4 * i + 1], wb[4 * i + 2], wb[4 * i + 3]);
    }
  }
}

// Tile t of the persistent loop: K split outermost; inside it the M tiles
// vary fastest (raster_n = 0: the B panel stays while the A panels stream,
// for a small A) or the N tiles do (raster_n = 1: a wave covers few A panels
// and every B panel, which stay in L2 together when A is the larger operand).
struct TileCoord {
  int mt, nt, ks;
};
__device__ __forceinline__ TileCoord tile_coord(int t, int m_tiles, int n_tiles, int raster_n) {
  TileCoord c;
  if (raster_n) {
    c.nt = t % n_tiles;
    const int rest = t / n_tiles;
    c.mt = rest % m_tiles;
    c.ks = rest / m_tiles;
  } else {
    c.mt = t % m_tiles;
    const int rest = t / m_tiles;
    c.nt = rest % n_tiles;
    c.ks = rest / n_tiles;
  }
  return c;
}

// Causal skipping (GemmParams.causal): the largest query position among
// stacked rows [r0, r0 + rows) (T - 1 when they wrap into the next head).
__device__ __forceinline__ int stack_tmax(int r0, int rows, int T) {
  const int t0 = r0 % T;
  return t0 + rows - 1 >= T ? T - 1 : t0 + rows - 1;
}
__device__ __forceinline__ bool tile_live(const GemmParams& p, int mt, int nt, int bn) {
  return p.causal != kCausalTiles || nt * bn <= stack_tmax(mt * kBM, kBM, p.causal_T);
}
__device__ __forceinline__ int kb_limit(const GemmParams& p, int mt, int kb1) {
  return p.causal == kCausalKeysK ? min(kb1, stack_tmax(mt * kBM, kBM, p.causal_T) / kBK + 1) : kb1;
}
__device__ __forceinline__ bool kb_live(const GemmParams& p, int mt, int kb) {
  return p.causal != kCausalRowsK || stack_tmax(kb * kBK, kBK, p.causal_T) >= mt * kBM;
}

// ------------------------------------------------------------ work units
// A CTA's work: with the stream-K tail (GemmParams.sk), first its range of
// the tile-major k blocks of tiles [0, sk_tiles), then whole tiles
// sk_tiles + c, + grid, ...; otherwise whole tiles c, c + grid, ...  Every
// role walks the same sequence.
enum { kUnitWhole = 0, kUnitTail = 1, kUnitHead = 2 };
struct Unit {
  int t;          // tile index (tile_coord)
  int kb0, kb1;   // stream-K: k blocks [kb0, kb1) of the tile; -1: the tile's K split
  int role;       // kUnitTail: partial to this CTA's slot; kUnitHead: adds the next CTA's slot
};
struct Sched {
  int pos, pos_end;       // stream-K k blocks still to do
  int t, t_end, t_step;   // whole tiles still to do
};
__device__ __forceinline__ Sched sched_init(const GemmParams& p, int total, int kb_total) {
  Sched s;
  const int G = gridDim.x, c = blockIdx.x;
  s.pos = s.pos_end = 0;
  s.t = c;
  s.t_step = G;
  s.t_end = total;
  if (p.sk) {
    // launcher: total > G and total % G != 0, so sk_tiles is in (G, 2G) and
    // every range is longer than a tile: a tile meets at most two ranges
    const int sk_tiles = total - (total / G - 1) * G;
    const long long n = static_cast<long long>(sk_tiles) * kb_total;
    s.pos = static_cast<int>(n * c / G);
    s.pos_end = static_cast<int>(n * (c + 1) / G);
    s.t = sk_tiles + c;
  }
  return s;
}
__device__ __forceinline__ bool sched_next(Sched& s, int kb_total, Unit& u) {
  if (s.pos < s.pos_end) {
    u.t = s.pos / kb_total;
    u.kb0 = s.pos % kb_total;
    u.kb1 = min(kb_total, u.kb0 + (s.pos_end - s.pos));
    u.role = u.kb0 > 0 ? kUnitTail : (u.kb1 < kb_total ? kUnitHead : kUnitWhole);
    s.pos += u.kb1 - u.kb0;
    return true;
  }
  if (s.t < s.t_end) {
    u.t = s.t;
    u.kb0 = u.kb1 = -1;
    u.role = kUnitWhole;
    s.t += s.t_step;
    return true;
  }
  return false;
}

// k blocks [kb0, kb1) of a unit: its stream-K range, or its K split's
// (clipped by causal key skipping)
__device__ __forceinline__ void unit_kblocks(const GemmParams& p, const Unit& u, int mt, int ks,
                                             int kb_per_split, int kb_total, int& kb0, int& kb1) {
  if (u.kb0 >= 0) {
    kb0 = u.kb0;
    kb1 = u.kb1;
    return;
  }
  kb0 = ks * kb_per_split;
  kb1 = kb_limit(p, mt, min(kb_total, kb0 + kb_per_split));
}

// sk_sync words: [0] launch counter, [1] CTAs done, [2 + 4 c + w] slot c's
// rows 32w.. published (the counter value + 1 of the launch that wrote them)
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Tail segment: this warp's 32 rows of the partial accumulator to slot
// `slot` (fp32 [128][BN], one row per lane), then publish them.
template <int BN>
__device__ __forceinline__ void epi_sk_tail(const GemmParams& p, uint32_t taddr, int quad,
                                            int lane, int slot, uint32_t tag) {
  float* dst = p.sk_ws + (static_cast<size_t>(slot) * kBM + quad * 32 + lane) * BN;
#pragma unroll 1
  for (int c = 0; c < BN; c += 32) {
    float v[32];
    tmem_ld32(taddr + c, v);
    float4* d4 = reinterpret_cast<float4*>(dst + c);
#pragma unroll
    for (int i = 0; i < 8; ++i) d4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
  __threadfence();
  __syncwarp();
  if (lane == 0) st_release_gpu(p.sk_sync + 2 + 4 * slot + quad, tag);
}

// Head segment: wait (bounded) until slot `slot` holds this warp's rows of
// the tile's tail; returns this lane's row of it, or nullptr when the wait
// gave up (timeout reported; the tile is then stored without it).
template <int BN>
__device__ __forceinline__ const float* sk_head_wait(const GemmParams& p, int quad, int lane,
                                                     int slot, uint32_t tag,
                                                     volatile int* abort_flag) {
  const uint32_t* f = p.sk_sync + 2 + 4 * slot + quad;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (__all_sync(0xFFFFFFFFu, ld_acquire_gpu(f) == tag)) break;
    if ((it & 15u) == 15u) {
      const bool give_up = (abort_flag && *abort_flag) || globaltimer_ns() - t0 > kWaitLimitNs;
      if (__any_sync(0xFFFFFFFFu, give_up)) {
        if (lane == 0) report_status(p.status, kStatusTimeout);
        return nullptr;
      }
    }
  }
  return p.sk_ws + (static_cast<size_t>(slot) * kBM + quad * 32 + lane) * BN;
}


template <int BN, int HD, int EPI, int MX>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ OutMaps om, const GemmParams p) {
  using C = GemmCfg<BN, MX>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* tiles = smem;
  uint8_t* out_stage = smem + S * C::kStageBytes;   // 1024-aligned: stage bytes are multiples of 1 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(out_stage + C::kOutStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* tfull = bars + 2 * S;
  uint64_t* tempty = bars + 2 * S + 2;
  uint64_t* drain = bars + 2 * S + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* sqk = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + C::kBarBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = (p.M + kBM - 1) / kBM;
  const int n_tiles = (p.N + BN - 1) / BN;
  const int kb_total = p.K / C::kKStep;
  const int kb_per_split = (kb_total + p.k_splits - 1) / p.k_splits;
  const int total = m_tiles * n_tiles * p.k_splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);   // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  if constexpr (EPI == kEpiQKVG) {
    if (threadIdx.x < HD) sqk[threadIdx.x] = p.s_qk[threadIdx.x];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      bool ok = true;
      const uint64_t pol_a = l2_policy_evict_first(), pol_b = l2_policy_evict_last();
      Sched sch = sched_init(p, total, kb_total);
      Unit u;
      while (ok && sched_next(sch, kb_total, u)) {
        const TileCoord tc = tile_coord(u.t, m_tiles, n_tiles, p.raster_n);
        const int mt = tc.mt, nt = tc.nt, ks = tc.ks;
        if (!tile_live(p, mt, nt, BN)) continue;   // the same decision in every role
        int kb0, kb1;
        unit_kblocks(p, u, mt, ks, kb_per_split, kb_total, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!kb_live(p, mt, kb)) continue;
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          uint8_t* a_dst = tiles + stage * C::kStageBytes;
          mbar_arrive_expect_tx(&full[stage], C::kLoadBytes);
          if (MX == kOperandsBf16 && p.a_mn) {
            // [K][M] source: 64-element M sub-tiles of 64 K rows (8 KB each)
#pragma unroll
            for (int j = 0; j < kBM / 64; ++j)
              tma_load_2d(a_dst + j * 8192, &tmA, &full[stage], mt * kBM + 64 * j, kb * kBK);
          } else if (p.l2_hint) {
            tma_load_2d_hint(a_dst, &tmA, &full[stage], kb * C::kKCoord, mt * kBM, pol_a);
          } else {
            tma_load_2d(a_dst, &tmA, &full[stage], kb * C::kKCoord, mt * kBM);
          }
          if (MX == kOperandsBf16 && p.b_mn) {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j)
              tma_load_2d(a_dst + C::kABytes + j * 8192, &tmB, &full[stage], nt * BN + 64 * j,
                          kb * kBK);
          } else if (p.l2_hint) {
            tma_load_2d_hint(a_dst + C::kABytes, &tmB, &full[stage], kb * C::kKCoord, nt * BN, pol_b);
          } else {
            tma_load_2d(a_dst + C::kABytes, &tmB, &full[stage], kb * C::kKCoord, nt * BN);
          }
          if constexpr (MX) {
            // this K step's scale chunks: one for A's 128 rows, BN/128 for B's
            bulk_load(a_dst + C::kABytes + C::kBBytes,
                      p.sfa + (static_cast<size_t>(kb) * p.sfa_blocks + mt) * C::kSfChunk,
                      C::kSfaBytes, &full[stage]);
            bulk_load(a_dst + C::kABytes + C::kBBytes + C::kSfaBytes,
                      p.sfb + (static_cast<size_t>(kb) * p.sfb_blocks + nt * (BN / 128)) * C::kSfChunk,
                      C::kSfbBytes, &full[stage]);
          }
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // let every copy this thread started land before the CTA exits
        for (int s = 0; s < S; ++s)
          if (issued_mask & (1u << s)) drain_wait(&full[s], (issued_parity >> s) & 1u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      // MN-major operands (bf16 only): transpose bits 15 (A) and 16 (B), the
      // MN-major swizzled layout (64-element sub-tiles 8 KB apart), and a
      // 16-K step of 16 rows (2048 B) instead of 32 bytes within a row
      const bool a_mn = MX == kOperandsBf16 && p.a_mn, b_mn = MX == kOperandsBf16 && p.b_mn;
      const uint32_t idesc = umma_idesc_bf16(kBM, BN) | (a_mn ? 1u << 15 : 0u) |
                             (b_mn ? 1u << 16 : 0u);
      // descriptors built once; a stage or k-step adds (byte offset >> 4)
      const uint64_t a_desc0 = a_mn ? umma_desc_sw128_mn(smem_u32(tiles), 8192)
                                    : umma_desc_sw128(smem_u32(tiles));
      const uint64_t b_desc0 = b_mn ? umma_desc_sw128_mn(smem_u32(tiles + C::kABytes), 8192)
                                    : umma_desc_sw128(smem_u32(tiles + C::kABytes));
      const uint32_t a_step = a_mn ? 2048 : 32, b_step = b_mn ? 2048 : 32;
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      bool issued = false;
      Sched sch = sched_init(p, total, kb_total);
      Unit u;
      while (ok && sched_next(sch, kb_total, u)) {
        const TileCoord tc = tile_coord(u.t, m_tiles, n_tiles, p.raster_n);
        const int mt = tc.mt, ks = tc.ks;
        if (!tile_live(p, mt, tc.nt, BN)) continue;
        int kb0, kb1;
        unit_kblocks(p, u, mt, ks, kb_per_split, kb_total, kb0, kb1);
        const int acc = it % C::kAccBufs;
        const uint32_t aph = (it / C::kAccBufs) & 1;
        if (!mbar_wait_bounded(&tempty[acc], aph ^ 1u, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        bool first = true;                 // the tile's first live K block overwrites
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!kb_live(p, mt, kb)) continue;
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t soff = static_cast<uint64_t>((stage * C::kStageBytes) >> 4);
          const uint64_t a_desc = a_desc0 + soff, b_desc = b_desc0 + soff;
          if constexpr (C::kNv) {
            // scales to TMEM (this stage's own columns, as for MXFP8): the
            // 512-byte piece kk of each chunk holds 64-K step kk's scales, one
            // 32-bit word per row; A's go to columns 4kk.., B's (BN / 32
            // columns per step) after them; then four K = 64 MMAs
            const uint32_t sf_col = tmem_base + C::kAccBufs * BN + stage * C::kSfCols;
            const uint32_t sfb_col = sf_col + 16;
            const uint32_t sf_smem = smem_u32(tiles + stage * C::kStageBytes + C::kABytes + C::kBBytes);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              tmem_cp_32x128b_x4(sf_col + 4 * kk, sf_desc(sf_smem + 512 * kk));
#pragma unroll
              for (int j = 0; j < BN / 128; ++j)
                tmem_cp_32x128b_x4(sfb_col + kk * (BN / 32) + 4 * j,
                                   sf_desc(sf_smem + C::kSfaBytes + 2048 * j + 512 * kk));
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_nvf4(d_tmem, a_desc + ((kk * 32) >> 4), b_desc + ((kk * 32) >> 4),
                        umma_idesc_nvf4(kBM, BN), sf_col + 4 * kk, sfb_col + kk * (BN / 32),
                        (!first || kk > 0) ? 1u : 0u);
          } else if constexpr (MX) {
            // scales to TMEM (this stage's own columns: the MMAs that read
            // them last time completed before the stage was refilled), then
            // four K = 32 block-scaled MMAs, MMA kk reading scale byte kk
            const uint32_t sf_col = tmem_base + C::kAccBufs * BN + stage * C::kSfCols;
            const uint32_t sf_smem = smem_u32(tiles + stage * C::kStageBytes + C::kABytes + C::kBBytes);
            tmem_cp_32x128b_x4(sf_col, sf_desc(sf_smem));
#pragma unroll
            for (int j = 0; j < BN / 128; ++j)
              tmem_cp_32x128b_x4(sf_col + 4 + 4 * j, sf_desc(sf_smem + C::kSfaBytes + 512 * j));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_mxf8(d_tmem, a_desc + ((kk * 32) >> 4), b_desc + ((kk * 32) >> 4),
                        umma_idesc_mxf8(kBM, BN, kk), sf_col, sf_col + 4,
                        (!first || kk > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              umma_bf16(d_tmem, a_desc + ((kk * a_step) >> 4), b_desc + ((kk * b_step) >> 4),
                        idesc, (!first || kk > 0) ? 1u : 0u);
            }
          }
          issued = true;
          first = false;
          umma_commit(&empty[stage]);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        ++it;
      }
      if (!ok && issued) {
        umma_commit(drain);
        drain_wait(drain, 0);
      }
    }
  } else {
    // ---------------------------------------------------- epilogue warps
    const int quad = warp & 3;
    uint8_t* my_stage = out_stage + (warp - 2) * 2 * C::kOutBufBytes;
    uint32_t nbuf = 0;                 // staged boxes so far (buffer rotation)
    int it = 0;
    // stream-K tag of this launch (the counter only moves after every CTA
    // of the launch has finished)
    const uint32_t tag = p.sk ? *reinterpret_cast<volatile uint32_t*>(p.sk_sync) + 1u : 0u;
    Sched sch = sched_init(p, total, kb_total);
    Unit u;
    while (sched_next(sch, kb_total, u)) {
      const TileCoord tc = tile_coord(u.t, m_tiles, n_tiles, p.raster_n);
      const int mt = tc.mt, nt = tc.nt, ks = tc.ks;
      if (!tile_live(p, mt, nt, BN)) continue;
      const int acc = it % C::kAccBufs;
      const uint32_t aph = (it / C::kAccBufs) & 1;
      // warp-uniform: the TMEM loads below are warp-collective
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(&tfull[acc], aph, abort_flag, p.status))) break;
      tc_fence_after();
      const int row = mt * kBM + quad * 32 + lane;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * BN;
      constexpr bool kAlpha = C::kNv;
      if constexpr (EPI == kEpiStoreF32) {
        if (u.role == kUnitTail) {
          epi_sk_tail<BN>(p, taddr, quad, lane, blockIdx.x, tag);
        } else {
          // a head adds the tail that opens the next CTA's range
          const float* part = u.role == kUnitHead
                                  ? sk_head_wait<BN>(p, quad, lane, blockIdx.x + 1, tag, abort_flag)
                                  : nullptr;
          if (p.c_tma)
            epi_store_f32_tma<BN, kAlpha>(p, &om.m[0], taddr, my_stage, lane, mt * kBM + quad * 32,
                                          nt, ks, nbuf, part);
          else
            epi_store_f32<BN, kAlpha>(p, taddr, row, nt, ks, part);
        }
      } else if constexpr (EPI == kEpiSwiGLU) {
        if (p.c_tma)
          epi_swiglu_tma<BN, kAlpha>(p, &om.m[0], taddr, my_stage, lane, mt * kBM + quad * 32, nt,
                                     nbuf);
        else
          epi_swiglu<BN, kAlpha>(p, taddr, row, nt);
      } else {
#pragma unroll 1
        for (int g = 0; g < BN / HD; ++g)
          epi_qkvg_group<HD, kAlpha>(p, sqk, &om, my_stage, lane, mt * kBM + quad * 32, nbuf,
                             taddr + g * HD, row, nt * BN + g * HD);
      }
      tc_fence_before();
      // one arrival per warp: many arrivals on one mbarrier are serialised
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      ++it;
    }
    // bulk stores read shared memory until they complete: finish before exit
    if (lane == 0 && nbuf > 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
  if (p.sk && threadIdx.x == 0) {
    // the last CTA of the launch resets the done count and moves the counter
    __threadfence();
    if (atomicAdd(p.sk_sync + 1, 1u) == gridDim.x - 1) {
      atomicExch(p.sk_sync + 1, 0u);
      __threadfence();
      atomicAdd(p.sk_sync, 1u);
    }
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn encode = nullptr;
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return nullptr;
    encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  return encode;
}

// [k_splits][M][N] fp32 output viewed as a 3D tensor (N innermost, row pitch
// ld_out, slice pitch split_stride) with 32 x 32 x 1 boxes and the 128-byte
// swizzle.  False when the layout does not allow bulk tensor stores (the
// kernel then stores from registers).
bool make_tmap_out_f32(CUtensorMap* map, const GemmParams& p) {
  EncodeTiledFn encode = encode_tiled();
  if (!encode || !p.out_f32 || p.N <= 0 || p.M <= 0) return false;
  const uint64_t slice = p.k_splits > 1 ? p.split_stride : static_cast<uint64_t>(p.M) * p.ld_out;
  if ((reinterpret_cast<uintptr_t>(p.out_f32) & 15) != 0 || (p.ld_out * 4ull) % 16 != 0 ||
      (slice * 4ull) % 16 != 0 || p.ld_out < p.N || slice < static_cast<uint64_t>(p.M) * p.ld_out)
    return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(p.N), static_cast<cuuint64_t>(p.M),
                        static_cast<cuuint64_t>(p.k_splits)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(p.ld_out) * 4, slice * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, p.out_f32, dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// [M][cols] bf16 output (row pitch ld elements) with 64 x 32 boxes and the
// 128-byte swizzle; false when the layout does not allow bulk tensor stores.
bool make_tmap_out_bf16(CUtensorMap* map, const void* base, int rows, int cols, int ld) {
  EncodeTiledFn encode = encode_tiled();
  if (!encode || !base || rows <= 0 || cols <= 0 || cols % 64 != 0 || ld < cols) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0 || (ld * 2ull) % 16 != 0) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {64, 32};
  cuuint32_t estr[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int HD, int EPI, int MX = kOperandsBf16>
cudaError_t launch_impl(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmParams& p,
                        int num_sms, cudaStream_t s) {
  using C = GemmCfg<BN, MX>;
  auto kern = gemm_tc_kernel<BN, HD, EPI, MX>;
  static uint32_t attr_done = 0;   // one bit per device ordinal < 32
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 32 || !(attr_done & (1u << dev))) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    if (dev < 32) attr_done |= 1u << dev;
  }
  const int m_tiles = (p.M + kBM - 1) / kBM;
  const int n_tiles = (p.N + BN - 1) / BN;
  const int total = m_tiles * n_tiles * p.k_splits;
  const int grid = total < num_sms ? total : num_sms;
  if (grid <= 0) return cudaSuccess;
  GemmParams q = p;
  // stream-K only where a partial last wave exists and its slots fit
  if (q.sk) {
    const bool usable = EPI == kEpiStoreF32 && q.k_splits == 1 && q.causal == kCausalNone &&
                        q.sk_ws && q.sk_sync && total > grid && total % grid != 0;
    if (!usable) q.sk = 0;
  }
  OutMaps om;
  memset(&om, 0, sizeof(om));
  q.c_tma = 0;
  if constexpr (EPI == kEpiStoreF32) q.c_tma = make_tmap_out_f32(&om.m[0], p) ? 1 : 0;
  if constexpr (EPI == kEpiSwiGLU)
    q.c_tma = make_tmap_out_bf16(&om.m[0], p.out_act, p.M, p.N / 2, p.ld_act) ? 1 : 0;
  if constexpr (EPI == kEpiQKVG)
    q.c_tma = (make_tmap_out_bf16(&om.m[0], p.q_out, p.M, p.n_q_heads * HD, p.n_q_heads * HD) &&
               make_tmap_out_bf16(&om.m[1], p.k_out, p.M, p.n_kv_heads * HD, p.n_kv_heads * HD) &&
               make_tmap_out_bf16(&om.m[2], p.v_out, p.M, p.n_kv_heads * HD, p.n_kv_heads * HD))
                  ? 1 : 0;
  kern<<<grid, kGemmThreads, C::kSmemBytes, s>>>(tmA, tmB, om, q);
  return cudaGetLastError();
}

}  // namespace

size_t gemm_sk_workspace_bytes(int grid, int BN) {
  const size_t slots = static_cast<size_t>(grid) * kBM * BN * 4;
  return (slots + 255) / 256 * 256 + (3 + 4 * static_cast<size_t>(grid)) * 4;
}

bool make_tmap_bf16_ld(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                       uint64_t ld, uint32_t box_rows) {
  EncodeTiledFn encode = encode_tiled();
  if (!encode || (ld * 2) % 16 != 0 || ld < cols || (reinterpret_cast<uintptr_t>(base) & 15) != 0)
    return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), box_rows};
  cuuint32_t estr[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows) {
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
  if ((cols * 2) % 16 != 0 || (reinterpret_cast<uintptr_t>(base) & 15) != 0) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_bf16_mn(CUtensorMap* map, const void* base, uint64_t k_rows, uint64_t mn_cols,
                       uint64_t ld) {
  EncodeTiledFn encode = encode_tiled();
  if (ld == 0) ld = mn_cols;
  if (!encode || (ld * 2) % 16 != 0 || ld < mn_cols || (reinterpret_cast<uintptr_t>(base) & 15) != 0)
    return false;
  cuuint64_t dims[2] = {mn_cols, k_rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

bool make_tmap_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                  uint32_t box_rows) {
  EncodeTiledFn encode = encode_tiled();
  if (!encode || cols % 16 != 0 || (reinterpret_cast<uintptr_t>(base) & 15) != 0) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

template <int MX>
cudaError_t dispatch_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmParams& p,
                          int BN, int head_dim, int num_sms, cudaStream_t s) {
  if (BN == 256) {
    switch (p.epi) {
      case kEpiStoreF32: return launch_impl<256, 128, kEpiStoreF32, MX>(tmA, tmB, p, num_sms, s);
      case kEpiSwiGLU: return launch_impl<256, 128, kEpiSwiGLU, MX>(tmA, tmB, p, num_sms, s);
      case kEpiQKVG:
        if (p.k_splits != 1) return cudaErrorInvalidValue;
        if (head_dim == 128) return launch_impl<256, 128, kEpiQKVG, MX>(tmA, tmB, p, num_sms, s);
        if (head_dim == 64) return launch_impl<256, 64, kEpiQKVG, MX>(tmA, tmB, p, num_sms, s);
        return cudaErrorInvalidValue;
    }
  } else if (BN == 128) {
    switch (p.epi) {
      case kEpiStoreF32: return launch_impl<128, 128, kEpiStoreF32, MX>(tmA, tmB, p, num_sms, s);
      case kEpiSwiGLU: return launch_impl<128, 128, kEpiSwiGLU, MX>(tmA, tmB, p, num_sms, s);
      case kEpiQKVG:
        if (p.k_splits != 1) return cudaErrorInvalidValue;
        if (head_dim == 128) return launch_impl<128, 128, kEpiQKVG, MX>(tmA, tmB, p, num_sms, s);
        if (head_dim == 64) return launch_impl<128, 64, kEpiQKVG, MX>(tmA, tmB, p, num_sms, s);
        return cudaErrorInvalidValue;
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmParams& p,
                        int BN, int head_dim, int num_sms, cudaStream_t s) {
  if (p.mx != kOperandsBf16 && p.mx != kOperandsMxfp8 && p.mx != kOperandsNvfp4)
    return cudaErrorInvalidValue;
  const int kstep = p.mx == kOperandsNvfp4 ? 256 : (p.mx ? 128 : kBK);
  if (p.K % kstep != 0 || p.K <= 0 || p.k_splits < 1) return cudaErrorInvalidValue;
  {
    // every K split must own at least one k-block
    const int kb = p.K / kstep, per = (kb + p.k_splits - 1) / p.k_splits;
    if ((p.k_splits - 1) * per >= kb) return cudaErrorInvalidValue;
  }
  // block-scaled operands need their scales (accumulators and scale columns
  // share TMEM); MN-major operands are bf16 only
  if (p.mx && (!p.sfa || !p.sfb)) return cudaErrorInvalidValue;
  if (p.mx && (p.a_mn || p.b_mn)) return cudaErrorInvalidValue;
  // causal skipping: bf16 and whole-K tiles only
  if (p.causal && (p.mx || p.k_splits != 1 || p.causal_T <= 0)) return cudaErrorInvalidValue;
  switch (p.mx) {
    case kOperandsMxfp8: return dispatch_gemm<kOperandsMxfp8>(tmA, tmB, p, BN, head_dim, num_sms, s);
    case kOperandsNvfp4: return dispatch_gemm<kOperandsNvfp4>(tmA, tmB, p, BN, head_dim, num_sms, s);
    default: return dispatch_gemm<kOperandsBf16>(tmA, tmB, p, BN, head_dim, num_sms, s);
  }
}

}  // namespace dory
