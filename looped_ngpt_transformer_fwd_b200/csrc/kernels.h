// Host-side launch interfaces of the sm_100a kernels (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dory {

// ----------------------------------------------------------------- GEMM
enum GemmEpilogue : int {
  kEpiStoreF32 = 0,   // C (fp32), optionally one slice per K split
  kEpiSwiGLU = 1,     // a = SiLU(gate_scale * C[:, gate cols]) * C[:, up cols] -> bf16
  kEpiQKVG = 2,       // RoPE + per-head L2 norm + s_qk on q/k heads, v copy, sigmoid gates
};

struct GemmParams {
  int M = 0, N = 0, K = 0;
  int k_splits = 1;
  int epi = kEpiStoreF32;
  // kEpiStoreF32
  float* out_f32 = nullptr;
  int ld_out = 0;
  size_t split_stride = 0;   // elements between K-split slices
  int c_tma = 0;             // set by the launcher: output written by bulk tensor stores
  // kEpiSwiGLU: tile of BN columns = [BN/2 gate cols | BN/2 up cols]
  __nv_bfloat16* out_act = nullptr;
  int ld_act = 0;
  float gate_scale = 1.f;
  // kEpiQKVG: columns [q heads | k heads | v heads | Hq gate logits | pad]
  __nv_bfloat16* q_out = nullptr;   // [M, Hq, hd]
  __nv_bfloat16* k_out = nullptr;   // [M, Hkv, hd]
  __nv_bfloat16* v_out = nullptr;   // [M, Hkv, hd]
  float* gate_out = nullptr;        // [M, Hq]
  int n_q_heads = 0, n_kv_heads = 0;
  const float* s_qk = nullptr;       // [hd]
  const float2* rope = nullptr;      // [hd/2][M] (cos, sin) of each row's angles (pair-major), this layer's base
  float norm_eps = 1e-20f;
  uint32_t* status = nullptr;
  // Block-scaled operands: mx = kOperandsMxfp8 (A and B tensor maps over E4M3
  // codes, make_tmap_u8; sfa / sfb their E8M0 scales in 512-byte chunks per
  // (128 rows, 128 K)) or kOperandsNvfp4 (maps over packed E2M1 codes, K / 2
  // bytes per row; sfa / sfb their E4M3 scales in 2048-byte chunks per (128
  // rows, 256 K)), with sfa_blocks = ceil(M / 128), sfb_blocks = 128-row
  // blocks of B's scale layout
  int mx = 0;
  const uint8_t* sfa = nullptr;
  const uint8_t* sfb = nullptr;
  int sfa_blocks = 0, sfb_blocks = 0;
  // every accumulator is multiplied by alpha before the epilogue uses it (the
  // product of the two NVFP4 tensor scales; 1 otherwise)
  float alpha = 1.f;
  // order of the persistent tile loop: 0 = M tiles fastest, 1 = N tiles
  // fastest (keeps a wave's A panels and all of B in L2 when A is larger)
  int raster_n = 0;
  // L2 hints on the K-major operand loads: A evict-first (each A panel is
  // read by the N tiles of one wave, then never again) and B evict-last (B is
  // read again by every wave), so B stays in L2 while A streams past
  int l2_hint = 0;
  // bf16 operands stored MN-major: A as [K][M] (a_mn) and / or B as [K][N]
  // (b_mn) row-major, their tensor maps from make_tmap_bf16_mn; the MMAs read
  // them transposed (the backward's dgrad and wgrad products)
  int a_mn = 0, b_mn = 0;
  // causal structure of the attention backward's products (bf16 only): rows
  // r = g * causal_T + t stack the query heads of a KV head's group, keys are
  // positions j; query t sees keys j <= t (kCausal* below)
  int causal = 0, causal_T = 0;
  // stream-K tail (kEpiStoreF32, whole K, no causal skipping): when the
  // tiles leave a partial last wave, the last one-and-a-fraction waves of
  // tiles are cut into contiguous k-block ranges of equal length, one per
  // CTA.  A tile then has at most two segments: the CTA holding its tail
  // writes an fp32 partial to its slot of sk_ws ([grid][128][BN]) and
  // publishes it through sk_sync; the CTA holding its head adds it and
  // stores the tile.  sk_sync ([2 + 4 * grid] words, zero before the first
  // use) keeps a launch counter, so it must not serve two launches at once.
  // Every CTA of the grid must be resident at once (one per SM): only for
  // launches that share the GPU with no concurrent kernel.  The launcher
  // clears sk where the tiles divide evenly into waves.
  int sk = 0;
  float* sk_ws = nullptr;
  uint32_t* sk_sync = nullptr;
};

// Bytes of a stream-K workspace for `grid` CTAs and BN-column tiles: the
// partial slots, then (256-byte aligned) the synchronisation words and a
// spare status word at the end.
size_t gemm_sk_workspace_bytes(int grid, int BN);

enum {
  kCausalNone = 0,
  kCausalTiles = 1,   // C[r][j]: tiles whose keys all follow every query of the tile are skipped (never written)
  kCausalKeysK = 2,   // K runs over keys: a tile's K loop ends after the last key its queries see
  kCausalRowsK = 3    // K runs over stacked rows, output rows are keys: K blocks whose queries all precede the tile's keys are skipped
};

// MLP-sublayer backward pieces (backward.cu): the nGPT update's backward
// (rows spread over `grid` CTAs, each writing its dalpha partial row), the
// column sum of those partials, the SwiGLU backward (packed and separate
// gradient layouts) and an in-place add.
int mlp_bwd_row_grid(int rows, int num_sms);
cudaError_t launch_mlp_bwd_row(const float* y, const float* h, const float* alpha,
                               const float* dh_out, int rows, int d, float norm_eps, float* dh,
                               __nv_bfloat16* dy_b, float* dalpha_part, int grid, cudaStream_t s);
cudaError_t launch_colsum(const float* part, int groups, int d, float* out, cudaStream_t s);
cudaError_t launch_swiglu_bwd(const float* gu, const float* da, int rows, int ff, int group,
                              float gate_scale, __nv_bfloat16* dgu_packed, __nv_bfloat16* dg_sep,
                              __nv_bfloat16* du_sep, cudaStream_t s);
cudaError_t launch_add_inplace(float* x, const float* y, size_t n, cudaStream_t s);

// Attention-sublayer backward pieces (attn_backward.cu), see that file.
cudaError_t launch_gather_heads(const __nv_bfloat16* src, int T, int src_heads, int head0, int G,
                                int hd, __nv_bfloat16* dst, cudaStream_t s);
cudaError_t launch_softmax_rows(const float* S, int rows, int T, int ld, int window, float scale,
                                __nv_bfloat16* P, cudaStream_t s);
cudaError_t launch_softmax_bwd_rows(const __nv_bfloat16* P, const float* dP, int rows, int T,
                                    int ld, int window, float scale, __nv_bfloat16* dS,
                                    cudaStream_t s);
cudaError_t launch_gated_output(const float* Os, const float* gate, int T, int hq, int G, int hd,
                                __nv_bfloat16* o, cudaStream_t s);
cudaError_t launch_gate_bwd(const float* dout, const float* Os, const float* gate, int T, int hq,
                            int G, int hd, __nv_bfloat16* dOs, __nv_bfloat16* d_raw, int ld_raw,
                            int gate_col0, cudaStream_t s);
cudaError_t launch_scatter_heads(const float* src, int T, int G, int hd, int dst_heads, int head0,
                                 float* dst, cudaStream_t s);
int qk_bwd_grid(int num_sms);
cudaError_t launch_qk_bwd(const float* raw, int ld_raw_f, const float* dq_hat, const float* dk_hat,
                          const float* s_qk, const float2* rope, int T, int hq, int hkv, int hd,
                          float norm_eps, __nv_bfloat16* d_raw, int ld_raw, float* ds_part,
                          int grid, cudaStream_t s);
cudaError_t launch_v_grad(const float* dv, int T, int hkv, int hd, __nv_bfloat16* d_raw, int ld_raw,
                          int col0, cudaStream_t s);

// Tensor map of a row-major bf16 matrix [k_rows, mn_cols] (row pitch ld
// elements, 0 = mn_cols) read as an MN-major GEMM operand: 64 x 64 boxes (64
// MN elements = 128 bytes, 64 K rows) with the 128-byte swizzle.
bool make_tmap_bf16_mn(CUtensorMap* map, const void* base, uint64_t k_rows, uint64_t mn_cols,
                       uint64_t ld = 0);
// make_tmap_bf16 with a row pitch of ld elements (>= cols)
bool make_tmap_bf16_ld(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                       uint64_t ld, uint32_t box_rows);

enum { kOperandsBf16 = 0, kOperandsMxfp8 = 1, kOperandsNvfp4 = 2 };

// Encode a 2D tensor map for a row-major uint8 matrix [rows, cols] (MXFP8
// codes) with a (128 x box_rows) box and the 128-byte swizzle.
bool make_tmap_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                  uint32_t box_rows);

// MXFP8 quantisation along K (see quant.cu): codes [rows, K] and scales in
// 512-byte chunks of (128 rows, 128 K).  `normalize` first scales every row to
// unit L2 norm.  bf16 sources come in up to 4 row segments (rows
// [seg_rows[i], seg_rows[i+1]) from segs[i], seg_rows[0] = 0), or with
// group > 0 as two matrices whose rows alternate in groups of `group`.
// Scale chunks cover the rows rounded up to `row_align` (128, or 256 for
// weights read as 256-row tiles); the padding rows get scale code 127.
size_t mxfp8_scale_bytes(int rows, int K, int row_align = 128);
cudaError_t launch_quant_mxfp8_bf16(const __nv_bfloat16* const* segs, const int* seg_rows,
                                    int n_seg, int group, int rows, int row_align, int K,
                                    int normalize, float norm_eps, uint8_t* codes, uint8_t* scales,
                                    cudaStream_t s);
cudaError_t launch_quant_mxfp8_f32(const float* src, int rows, int K, int normalize, float norm_eps,
                                   uint8_t* codes, uint8_t* scales, cudaStream_t s);

// NVFP4 quantisation along K (see quant.cu): packed E2M1 codes [rows, K / 2]
// (element 2i in the low nibble of byte i), E4M3 block scales (blocks of 16)
// in 2048-byte chunks of (128 rows, 256 K), given the fp32 tensor scale g
// (`d_g` on the device when not null, else `g`).  Sources and padding as for
// MXFP8 (padding rows get scale 1.0); K must be a multiple of 256.
size_t nvfp4_scale_bytes(int rows, int K, int row_align = 128);
cudaError_t launch_quant_nvfp4_bf16(const __nv_bfloat16* const* segs, const int* seg_rows,
                                    int n_seg, int group, int rows, int row_align, int K,
                                    int normalize, float norm_eps, const float* d_g, float g,
                                    uint8_t* codes, uint8_t* scales, cudaStream_t s);
cudaError_t launch_quant_nvfp4_f32(const float* src, int rows, int K, int normalize, float norm_eps,
                                   const float* d_g, float g, uint8_t* codes, uint8_t* scales,
                                   cudaStream_t s);
// The NVFP4 tensor scale of a group of bf16 matrices quantised with one scale:
// g = amax / (6 * 448) over all their elements (1 when all are zero), written
// to d_g.  d_amax is a 4-byte scratch word.
cudaError_t launch_nvfp4_tensor_scale(const __nv_bfloat16* const* mats, const size_t* counts, int n,
                                      uint32_t* d_amax, float* d_g, cudaStream_t s);

// Encode a 2D tensor map for a row-major bf16 matrix [rows, cols] with a
// (64 x box_rows) box and the 128-byte swizzle.  Returns false on failure.
bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows);

// C[M, N] = A[M, K] * B[N, K]^T with the chosen epilogue.  BN is 128 or 256;
// head_dim (64 or 128) selects the QKVG epilogue instantiation.
cudaError_t launch_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmParams& p,
                        int BN, int head_dim, int num_sms, cudaStream_t s);

// Output / down projection with the nGPT update fused into the epilogue
// (prefill): a cluster of `cluster` CTAs covers the N = d_model columns of a
// 128-row band; h is updated in place (see gemm_ngpt.cu).
struct NgptGemmParams {
  int M = 0, N = 0, K = 0;
  int cluster = 0;                   // N / ngpt_gemm_cols_per_cta(N)
  float* h = nullptr;                // [M, N] fp32 stream, updated in place
  __nv_bfloat16* hb = nullptr;       // [M, N] bf16 copy for the next GEMM (may be null)
  const float* alpha = nullptr;      // [N]
  float* e_save = nullptr;           // optional: the update result is saved here
  const float* e = nullptr;          // optional: then x <- Norm(x + e)
  __nv_bfloat16* out = nullptr;      // optional final output [M, N] bf16
  float norm_eps = 1e-20f;
  uint32_t* status = nullptr;
};
// Columns per CTA of the fused kernel for this d_model (0: not supported).
int ngpt_gemm_cols_per_cta(int d_model);
cudaError_t launch_gemm_ngpt(const CUtensorMap& tmA, const CUtensorMap& tmB,
                             const NgptGemmParams& p, cudaStream_t s);

// RoPE (cos, sin) table, pair-major [hd/2][rows], for row r at position pos0 + r (or
// d_pos[r]): angle = pos * inv_freq[i] in float64, reduced mod 2*pi, then
// sincosf.
cudaError_t launch_rope_table(const double* inv_freq, int hd, int rows, int pos0,
                              const int32_t* d_pos, float2* out, cudaStream_t s);

// K-split QKVG post-processing (decode): sum the split partial products
// [splits][rows][n_qkvg], then the same per-head RoPE / L2 norm / s_qk / gate
// steps as the fused kEpiQKVG epilogue.
struct KvLayerView {
  __nv_bfloat16* k_base = nullptr;
  __nv_bfloat16* v_base = nullptr;
  size_t seq_stride = 0;   // elements
  int cap = 0;             // slots per (seq, head)
  int n_kv = 0, hd = 0;
  int max_seqs = 0, max_ctx = 0;
};

struct QkvgPostParams {
  const float* part = nullptr;
  int splits = 1;
  size_t split_stride = 0;   // elements
  int ld = 0;                // row pitch of `part` (elements, >= the QKVG column count)
  int rows = 0, n_q_heads = 0, n_kv_heads = 0, hd = 0;
  const float* s_qk = nullptr;
  const float2* rope = nullptr;
  float norm_eps = 1e-20f;
  __nv_bfloat16 *q_out = nullptr, *k_out = nullptr, *v_out = nullptr;
  float* gate_out = nullptr;
  // commit = 1: also write each row's k and v into its cache slot (decode:
  // row r of sequence d_seq[r] at position d_pos[r], slot pos % cap), as a
  // separate kv_commit would: rows with row_k[r] < loop skipped, positions
  // or sequences out of range reported (kStatusBounds) and skipped
  int commit = 0;
  KvLayerView kv;
  const int32_t* d_seq = nullptr;
  const int32_t* d_pos = nullptr;
  const int32_t* row_k = nullptr;
  int loop = 0;
  uint32_t* status = nullptr;
};
cudaError_t launch_qkvg_post(const QkvgPostParams& p, cudaStream_t s);

// K-split gate/up post-processing (decode): columns are the interleaved
// weight rows (`group` gate, `group` up, ...); a = SiLU(gate_scale * g) * u.
cudaError_t launch_swiglu_post(const float* part, int splits, size_t split_stride, int rows,
                               int d_ff, float gate_scale, int group, __nv_bfloat16* out,
                               cudaStream_t s);

// ----------------------------------------------------------------- rows
struct RowUpdateParams {
  int rows = 0, d = 0;
  const float* y = nullptr;   // [splits, rows, d] sublayer output before normalisation
  int splits = 1;
  size_t split_stride = 0;    // elements
  float* h = nullptr;         // [rows, d] fp32 stream, updated in place
  __nv_bfloat16* hb = nullptr;  // [rows, d] bf16 copy for the next GEMM (may be null)
  const float* alpha = nullptr;  // [d]
  float norm_eps = 1e-20f;
  // optional re-injection: after the update, save the result to e_save (if
  // set) and then replace it by Norm(h + e) when e is set
  float* e_save = nullptr;
  const float* e = nullptr;
  __nv_bfloat16* out = nullptr;  // optional final output [rows, d] bf16
  // per-row loop counts (one decode step with a different k per sequence):
  // in recurrent loop `loop`, rows with row_k[r] < loop are left unchanged
  // and the re-injection applies only while loop < row_k[r].  A count
  // outside 1..k_hi leaves the row unchanged and sets kStatusBounds.  Null:
  // every row runs every loop.
  const int32_t* row_k = nullptr;
  int loop = 0, k_hi = 0;
  uint32_t* status = nullptr;
  // optional: the final rows quantised for the next projection, exactly as
  // launch_quant_mxfp8_f32 / launch_quant_nvfp4_f32 would (q_fmt
  // kOperandsMxfp8 or kOperandsNvfp4; codes [rows, d] or [rows, d / 2], scale
  // chunks over q_row_blocks = ceil(rows / 128) row blocks, NVFP4 tensor scale
  // q_g).  The scales of the padding rows of the last block are left as they
  // are: they only reach accumulator rows that are never stored.  Not with
  // row_k (skipped rows would keep stale codes).
  int q_fmt = 0;
  uint8_t* q_codes = nullptr;
  uint8_t* q_scales = nullptr;
  int q_row_blocks = 0;
  float q_g = 0.f;
  float q_r6 = 0.f;   // 1 / (6 q_g) in fp32: set by launch_row_update
};
cudaError_t launch_row_update(const RowUpdateParams& p, cudaStream_t s);

// bf16 [rows, d] -> fp32 stream + bf16 copy
cudaError_t launch_load_rows(const __nv_bfloat16* src, float* h, __nv_bfloat16* hb, int rows,
                             int d, cudaStream_t s);
// fp32 -> bf16 copy
cudaError_t launch_f32_to_bf16(const float* src, __nv_bfloat16* dst, size_t n, cudaStream_t s);

// ----------------------------------------------------------------- KV cache
// Where one layer's cache lives: sequence s, KV head h, slot t:
//   K at k_base + s*seq_stride + (h*cap + t)*hd, V at v_base + same (elements)

// Copy fresh K/V rows [rows, Hkv, hd] into cache slots.  Row r goes to
// sequence seq (or d_seq[r]) at position pos0 + r (or d_pos[r]); rows below
// `first_row` are skipped.
// row_k / loop: as in RowUpdateParams (rows whose loop count is below `loop`
// write nothing); null commits every row.
cudaError_t launch_kv_commit(const KvLayerView& kv, const __nv_bfloat16* k_new,
                             const __nv_bfloat16* v_new, int rows, int first_row, int seq,
                             int pos0, const int32_t* d_seq, const int32_t* d_pos,
                             uint32_t* status, cudaStream_t s, const int32_t* row_k = nullptr,
                             int loop = 0);

// ----------------------------------------------------------------- attention
struct PrefillAttnParams {
  const __nv_bfloat16* q = nullptr;     // [n, Hq, hd]
  const __nv_bfloat16* k_new = nullptr; // [n, Hkv, hd]  this call's keys (positions >= pos0)
  const __nv_bfloat16* v_new = nullptr;
  const float* gate = nullptr;          // [n, Hq]
  __nv_bfloat16* out = nullptr;         // [n, Hq*hd]
  KvLayerView kv;                       // earlier positions (< pos0)
  int seq = 0, pos0 = 0, n = 0;
  int n_q_heads = 0;
  int window = 0;                       // 0 = full attention
  float scale_log2 = 0.f;               // softmax_scale * log2(e)
  uint32_t* status = nullptr;
  int32_t* probe = nullptr;             // mask probe records [n, Hq, 4], or null
};
cudaError_t launch_prefill_attention(const PrefillAttnParams& p, cudaStream_t s);

// Tensor-core (tcgen05) prefill attention for head_dim 128 with a static
// softmax maximum m_log2 = softmax_scale * log2(e) * max_i s_qk[i]^2.
struct PrefillAttnTcParams {
  const __nv_bfloat16* q = nullptr;     // [n, Hq, hd] (set by the launcher)
  const float* gate = nullptr;          // [n, Hq]
  __nv_bfloat16* out = nullptr;         // [n, Hq*hd]
  int n = 0, pos0 = 0, seq = 0;
  int n_q_heads = 0, n_kv = 0;
  int cap = 0;                          // cache slots per (seq, head)
  int window = 0;                       // 0 = full attention
  int last_pos = 0;                     // pos0 + n - 1
  float scale_log2 = 0.f, m_log2 = 0.f;
  uint32_t* status = nullptr;
  int32_t* probe = nullptr;             // mask probe records [n, Hq, 4], or null
  // set by the launcher: this call's K / V [n, Hkv, hd] and the layer's cache
  // (K plane of (seq, head) at rows (seq * 2 * Hkv + head) * cap, V planes
  // after the Hkv K planes), read directly for key tiles gathered row by row
  const __nv_bfloat16* k_new = nullptr;
  const __nv_bfloat16* v_new = nullptr;
  const __nv_bfloat16* cache = nullptr;
};
bool prefill_attention_tc_supported(int head_dim, int pos0, int window, float m_log2);
cudaError_t launch_prefill_attention_tc(const PrefillAttnTcParams& p, const __nv_bfloat16* q,
                                        const __nv_bfloat16* k_new, const __nv_bfloat16* v_new,
                                        const KvLayerView& kv, cudaStream_t s);

struct DecodeAttnParams {
  const __nv_bfloat16* q = nullptr;     // [B, Hq, hd]
  const float* gate = nullptr;          // [B, Hq]
  __nv_bfloat16* out = nullptr;         // [B, Hq*hd]
  KvLayerView kv;
  const int32_t* d_seq = nullptr;
  const int32_t* d_pos = nullptr;
  int batch = 0, n_q_heads = 0, window = 0;
  int max_pos = 0;                      // upper bound of d_pos (grid sizing)
  int split_keys = 0;                   // keys per split
  float scale_log2 = 0.f;
  float* part_acc = nullptr;            // [B, Hq, n_splits, hd]
  float* part_ml = nullptr;             // [B, Hq, n_splits, 2]
  uint32_t* status = nullptr;
  int32_t* probe = nullptr;             // mask probe records [B, Hq, 4], or null
};
int decode_attention_splits(int max_pos, int window, int split_keys);
cudaError_t launch_decode_attention(const DecodeAttnParams& p, cudaStream_t s);
// merge the split partials (acc, (m, l)) of every (sequence, head), gate, store
cudaError_t launch_decode_combine(const DecodeAttnParams& p, int n_splits, cudaStream_t s);
// TMA-fed decode attention with a static softmax maximum (head_dim 128)
bool decode_attention_tma_supported(int head_dim, int window, int group);
int decode_attention_tma_splits(int max_pos, int window, int* split_tiles);
cudaError_t launch_decode_attention_tma(const DecodeAttnParams& p, float m_log2, cudaStream_t s);

// ----------------------------------------------------------------- vocabulary
// Embedding rows Norm(table[token]) as bf16 [n, d] (a token outside 0..vocab-1
// gives a zero row and kStatusBounds); logits z[r][v] *= scale[v]; one token
// per row of logits [n, vocab] (greedy at temperature 0, else Gumbel-max from
// the counter hash of (seed, steps[r], v)).
cudaError_t launch_embed(const __nv_bfloat16* table, int vocab, int d, const int32_t* tokens,
                         int n, __nv_bfloat16* out, uint32_t* status, cudaStream_t s);
cudaError_t launch_scale_columns(float* z, const float* scale, int rows, int cols, cudaStream_t s);
cudaError_t launch_sample(const float* logits, int n, int vocab, float temperature, uint32_t seed,
                          const int32_t* steps, int32_t* tokens, cudaStream_t s);

// ----------------------------------------------------------------- diagnostics
// Set `n_records` mask-probe records to {INT_MAX, -1, 0, 0}.
cudaError_t launch_probe_init(int32_t* probe, size_t n_records, cudaStream_t s);
// One kernel whose single thread waits on an mbarrier that nothing arrives at,
// giving up after `limit_ns` with kStatusTimeout in *status.
cudaError_t launch_wait_timeout(uint32_t* status, uint64_t limit_ns, cudaStream_t s);

}  // namespace dory
