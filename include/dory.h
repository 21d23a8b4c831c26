/*
 * dory.h -- C ABI of the B200 (sm_100a) looped nGPT forward-pass library.
 *
 * What it computes.  The forward pass of a looped normalized-GPT stack as the
 * Dory1.0-4B pages describe it:
 *   - "Dory1.0-4B: A Looped Normalized-GPT" (ai.info AI summary), Key
 *     Contributions item 1: an input block, a shared recurrent block applied k
 *     times, an output block (effective depth 32 + 40k sublayers);
 *     Methodology in Plain English: nGPT hypersphere residual updates
 *     h <- Norm(h + alpha * (Norm(f(h)) - h)) with learned per-channel alpha,
 *     GQA attention with sigmoid output gates interleaving sliding-window and
 *     full layers (RoPE per layer type), L2 norm of the gated attention output
 *     before the output projection and of the SwiGLU activations before the
 *     down-projection, and re-injection of the input block's output before
 *     every pass of the recurrent block;
 *   - "Dory 1.0 4B Benchmarks: How Do 1, 2 and 4 Loops Compare?" (goremy.ai),
 *     How does looping work at inference time?: k is chosen per request on the
 *     same weights; per-loop KV caching keeps one cache per loop, last-loop
 *     caching keeps one cache per recurrent attention layer that every loop
 *     overwrites, so its footprint is the one-loop size for any k.
 *
 * Conventions.
 *   - Every function returning int returns DORY_OK (0) or a negative
 *     dory_status.  Nothing aborts the process.
 *   - Memory is owned by the caller: the library never allocates device
 *     memory.  It keeps host-side metadata (handles, CUDA graphs, tensor-map
 *     descriptors) which dory_kv_free / dory_destroy release.
 *   - `stream` arguments are cudaStream_t values passed as void* (NULL = the
 *     legacy default stream).  Calls are asynchronous on that stream; outputs
 *     are valid once it has been synchronised.
 *   - Hidden states are bf16, row-major [rows, d_model].  Input rows are
 *     expected to have unit L2 norm and are not re-normalised.
 *   - Pointers named h_in / h_out may be device pointers or host pointers
 *     (pinned host memory gives overlapped copies); host buffers are staged
 *     through the workspace with cudaMemcpyAsync on `stream`.
 *   - Device pointers passed in must be 256-byte aligned (DORY_ERR_MISALIGNED).
 */
#ifndef DORY_H
#define DORY_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DORY_API __attribute__((visibility("default")))
#else
#define DORY_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dory_status {
  DORY_OK = 0,
  DORY_ERR_INVALID_ARG = -1,      /* null pointer, negative size, bad index      */
  DORY_ERR_BAD_CONFIG = -2,       /* unsupported shapes in dory_config            */
  DORY_ERR_K_RANGE = -3,          /* k outside 1..4 (1..8 with allow_extrapolated_k) */
  DORY_ERR_K_EXCEEDS_KMAX = -4,   /* per-loop cache allocated for fewer loops     */
  DORY_ERR_CTX_OVERFLOW = -5,     /* positions beyond the cache's max_ctx         */
  DORY_ERR_BUFFER_TOO_SMALL = -6, /* weight / kv / workspace buffer too small     */
  DORY_ERR_MISALIGNED = -7,       /* a device buffer is not 256-byte aligned      */
  DORY_ERR_CUDA = -8,             /* a CUDA runtime/driver call failed            */
  DORY_ERR_DEVICE_TIMEOUT = -9,   /* a kernel's bounded wait expired (device word) */
  DORY_ERR_UNSUPPORTED_ARCH = -10,/* device is not sm_100                         */
  DORY_ERR_DEVICE_BOUNDS = -11,   /* a kernel's bounds check fired (device word)   */
  DORY_ERR_SCRATCH_LIMIT = -12    /* rows exceed the library's built-in scratch    */
} dory_status;

typedef enum dory_weight_format {
  DORY_WEIGHTS_BF16 = 0,  /* bf16 weights, bf16 projection inputs                   */
  DORY_WEIGHTS_MXFP8 = 1, /* MXFP8 weights and projection inputs (see dory_config)  */
  DORY_WEIGHTS_NVFP4 = 2  /* NVFP4 weights and projection inputs (see dory_config)  */
} dory_weight_format;

typedef enum dory_kv_mode {
  DORY_KV_PER_LOOP = 0,   /* recurrent layers keep one cache per loop (k_max of them) */
  DORY_KV_LAST_LOOP = 1   /* one cache per layer; each loop overwrites the last        */
} dory_kv_mode;

/* Model shape.  Global block b (0-based over in+rec+out blocks) uses full
 * attention iff b % full_period == full_period - 1, otherwise a sliding window
 * of `window` keys ending at (and including) the query position.
 * Supported: head_dim 64 or 128; d_model == n_q_heads * head_dim;
 * n_q_heads % n_kv_heads == 0 with a group of at most 4; d_model and d_ff
 * multiples of 128; window >= 1. */
typedef struct dory_config {
  int32_t d_model;
  int32_t n_q_heads;
  int32_t n_kv_heads;
  int32_t head_dim;
  int32_t d_ff;
  int32_t n_in_blocks;
  int32_t n_rec_blocks;
  int32_t n_out_blocks;
  int32_t window;
  int32_t full_period;
  double rope_base_swa;     /* RoPE base of sliding-window layers          */
  double rope_base_full;    /* RoPE base of full-attention layers          */
  float softmax_scale;      /* logit = softmax_scale * q_hat . k_hat       */
  float gate_scale;         /* SwiGLU: SiLU(gate_scale * h Wg^T) * (h Wu^T) */
  float norm_eps;           /* Norm(x) = x / sqrt(max(sum x^2, norm_eps))  */
  int32_t allow_extrapolated_k; /* nonzero: accept k up to 8               */
  /* DORY_WEIGHTS_BF16, or DORY_WEIGHTS_MXFP8: the released MXFP8 checkpoint
   * format ("Dory1.0-4B: A Looped Normalized-GPT", Key Contributions item 4;
   * Methodology in Plain English: MXFP8 by standard post-training
   * quantisation), served as both operands of every projection in MXFP8:
   * blocks of 32 values along the reduction axis share an E8M0 scale
   * 2^(floor(log2 amax) - 8) and hold E4M3 elements (nearest, ties to even,
   * saturating at 448).  dory_create quantises the bf16 source matrices (which
   * must then be device pointers, 16-byte aligned); every projection input is
   * quantised on the fly (the attention output and the SwiGLU activations
   * after their L2 norm), and the products run on the block-scaled tensor
   * cores (tcgen05.mma kind::mxf8f6f4).
   * DORY_WEIGHTS_NVFP4: the released NVFP4 checkpoint format (same page, Key
   * Contributions item 4; Main Findings: NVFP4 after quantisation-aware
   * distillation), served as both operands of every projection in NVFP4:
   * blocks of 16 values along the reduction axis share an E4M3 scale
   * E4M3(amax_block / (6 g)) and hold E2M1 elements (nearest, ties to even,
   * saturating at 6) under a per-tensor fp32 scale g.  The weights' g is
   * amax / (6 * 448) over the matrices one GEMM reads together (q, k, v and
   * the gate rows; gate and up; W_o; W_down), computed by dory_create; every
   * projection input takes g = 1 / (6 * 448), since its rows are unit vectors
   * (no element above 1).  Products run on tcgen05.mma kind::mxf4nvf4 with the
   * two tensor scales applied in the epilogue.  Needs d_model and d_ff
   * multiples of 256; sources as for MXFP8. */
  int32_t weight_format;
} dory_config;

/* Source tensors of one block, row-major [out, in] bf16 matrices (as
 * uint16_t bit patterns) and fp32 vectors.  Host or device pointers. */
typedef struct dory_block_src {
  const uint16_t* wq;      /* [n_q_heads*head_dim, d_model]  */
  const uint16_t* wk;      /* [n_kv_heads*head_dim, d_model] */
  const uint16_t* wv;      /* [n_kv_heads*head_dim, d_model] */
  const uint16_t* wg;      /* [n_q_heads, d_model]  attention output gates */
  const uint16_t* wo;      /* [d_model, n_q_heads*head_dim] */
  const uint16_t* w_gate;  /* [d_ff, d_model]  */
  const uint16_t* w_up;    /* [d_ff, d_model]  */
  const uint16_t* w_down;  /* [d_model, d_ff]  */
  const float* alpha_attn; /* [d_model] */
  const float* alpha_mlp;  /* [d_model] */
  const float* s_qk;       /* [head_dim] */
} dory_block_src;

typedef struct dory_model dory_model;
typedef struct dory_kv dory_kv;

/* Bytes of the device buffer dory_create packs the weights into
 * (weights in the kernels' layout, a small device status area and about
 * 21 MB of stream-K partial slots for the prefill projections). */
DORY_API size_t dory_weight_bytes(const dory_config* cfg);

/* Validate `cfg`, check that the current device is sm_100, and pack the
 * weights of all blocks (`src[b]` for global block b) into `weight_buf`
 * (device, caller-owned, at least dory_weight_bytes, 256-byte aligned).
 * The copies are ordered on `stream`.  On success *out is a new handle. */
DORY_API int dory_create(const dory_config* cfg, void* weight_buf, size_t weight_bytes,
                const dory_block_src* src, int n_src, void* stream, dory_model** out);

/* Bytes of a KV cache: pure arithmetic, no allocation.  Per attention layer
 * (and per loop for recurrent layers under DORY_KV_PER_LOOP with `k_max`
 * loops) and per sequence: K and V, n_kv_heads * head_dim bf16 each, for
 * min(window, max_ctx) positions (sliding-window layers) or max_ctx
 * positions (full layers).  Under DORY_KV_LAST_LOOP the result does not
 * depend on k_max.  Returns 0 for invalid arguments. */
DORY_API size_t dory_kv_bytes(const dory_config* cfg, int mode, int max_seqs, int max_ctx, int k_max);

/* Bind a KV cache of `mode` to `kv_buf` (device, caller-owned,
 * >= dory_kv_bytes).  The contents are not touched. */
DORY_API int dory_kv_alloc(dory_model* m, int mode, int max_seqs, int max_ctx, int k_max,
                  void* kv_buf, size_t kv_bytes, dory_kv** out);

/* Byte offsets from kv_buf of the K and V entries of (global block `layer`,
 * loop `loop` (1-based; ignored unless the layer is recurrent and the mode is
 * per-loop), sequence `seq`, position `pos`, KV head `head`).  Each entry is
 * head_dim contiguous bf16.  Sliding-window layers are rings of
 * min(window, max_ctx) slots (slot = pos % capacity); full layers use slot = pos.
 * Within one (layer, loop, seq, head) the slots are contiguous (stride
 * head_dim * 2 bytes). */
DORY_API int dory_kv_layout(const dory_kv* kv, int layer, int loop, int seq, int pos, int head,
                   size_t* k_off, size_t* v_off);

/* Workspace bytes for calls of up to `max_tokens` rows (prefill tokens or
 * decode batch), 256-byte aligned base required. */
DORY_API size_t dory_workspace_bytes(const dory_model* m, int max_tokens);

/* Prefill `n_tokens` tokens of sequence `seq` at positions pos0 .. pos0+n-1
 * with k recurrent loops.  Chunked prefill is repeated calls with increasing
 * pos0; positions before pos0 must already be in the cache.  Under last-loop
 * caching the call's tokens at loop j attend to earlier positions' cached
 * entries and to this call's own loop-j keys; after the call the cache holds
 * loop k's entries.  h_in, h_out: [n_tokens, d_model] bf16 (host or device). */
DORY_API int dory_prefill(dory_model* m, dory_kv* kv, int seq, int pos0, int n_tokens,
                 const void* h_in, void* h_out, int k,
                 void* ws, size_t ws_bytes, void* stream);

/* One decode step for `batch` sequences: row i is sequence d_seq[i] at
 * position d_pos[i] (int32 device arrays, so a captured step replays across
 * steps).  Every row's positions before d_pos[i] must be cached.  h_in,
 * h_out: [batch, d_model] bf16 (host or device).  `max_pos_hint` is an upper
 * bound on every d_pos[i] (it sizes the split-KV grid; positions above it are
 * reported as DORY_ERR_DEVICE_BOUNDS by dory_device_status). */
DORY_API int dory_decode_step(dory_model* m, dory_kv* kv, int batch,
                     const int32_t* d_seq, const int32_t* d_pos, int max_pos_hint,
                     const void* h_in, void* h_out, int k,
                     void* ws, size_t ws_bytes, void* stream);

/* One decode step in which each sequence has its own loop count: row i runs
 * d_k[i] recurrent loops (the loop count as a per-request dial: "NVIDIA
 * Nemotron Labs Dory 1.0 4B: a looped (latent-recurrent) LLM with elastic
 * inference compute", Why it matters here; prompts routed to different loop
 * depths: "Dory1.0-4B: A Looped Normalized-GPT", Key Contributions).  Row i's
 * result equals dory_decode_step of that row alone with k = d_k[i].
 *   d_k    int32 device array [batch], each value in 1..k_hi (caller-owned,
 *          read by the kernels, so a captured step replays across steps);
 *   k_hi   the largest d_k[i]: the step runs k_hi loops and a row whose
 *          count is below the current loop is left unchanged and writes no
 *          cache entry.  It is checked like k of dory_decode_step
 *          (DORY_ERR_K_RANGE, DORY_ERR_K_EXCEEDS_KMAX); a d_k[i] outside
 *          1..k_hi leaves row i's recurrent loops undone and is reported as
 *          DORY_ERR_DEVICE_BOUNDS by dory_device_status.
 * Other arguments as for dory_decode_step.  Under per-loop caching each
 * sequence's earlier tokens must have been written with the same count. */
DORY_API int dory_decode_step_mixed(dory_model* m, dory_kv* kv, int batch,
                     const int32_t* d_seq, const int32_t* d_pos, const int32_t* d_k, int k_hi,
                     int max_pos_hint, const void* h_in, void* h_out,
                     void* ws, size_t ws_bytes, void* stream);

/* Synchronise `stream`, read and clear the model's device status word:
 * DORY_OK, DORY_ERR_DEVICE_TIMEOUT or DORY_ERR_DEVICE_BOUNDS. */
DORY_API int dory_device_status(dory_model* m, void* stream);

/* Kernel launches of the most recent dory_prefill / dory_decode_step, and how
 * many nGPT sublayer updates it applied (32 + 40k for the Dory shape). */
DORY_API int dory_last_call_stats(const dory_model* m, int* kernel_launches, int* sublayer_updates);

DORY_API const char* dory_error_string(int status);

/* dory_kv_free releases the cache handle (not its buffer) and the captured
 * graphs that refer to it.  dory_destroy releases the model handle and its
 * graphs; caches still bound to it become unusable but may still be freed. */
DORY_API void dory_kv_free(dory_kv* kv);
DORY_API void dory_destroy(dory_model* m);

/* ---------------------------------------------------------------------
 * Tokens in and out.  The pages describe the stack between its first and
 * last hidden states only ("Dory1.0-4B: A Looped Normalized-GPT", Overview:
 * no vocabulary, no head); these follow the nGPT backbone the model card
 * cites ("NVIDIA Nemotron Labs Dory 1.0 4B ...", Key ideas: every vector on
 * the unit sphere).  The vocabulary size is the caller's (a multiple of 256).
 * --------------------------------------------------------------------- */
typedef struct dory_vocab dory_vocab;

/* Bytes of the device buffer dory_vocab_create packs the tables into (0 for
 * invalid arguments). */
DORY_API size_t dory_vocab_bytes(const dory_config* cfg, int vocab);

/* Input table emb_in [vocab, d_model] and output table emb_out [vocab,
 * d_model] (bf16 bit patterns, rows expected unit-norm), per-token logit scale
 * s_z [vocab] (fp32); host or device pointers, copied into `buf` (device,
 * caller-owned, >= dory_vocab_bytes, 256-byte aligned) on `stream`. */
DORY_API int dory_vocab_create(dory_model* m, int vocab, const uint16_t* emb_in,
                               const uint16_t* emb_out, const float* logit_scale, void* buf,
                               size_t bytes, void* stream, dory_vocab** out);

/* h_out [n, d_model] bf16 (device) = Norm(emb_in[d_tokens[i]]): the unit-norm
 * input rows of dory_prefill / dory_decode_step.  d_tokens: int32 device.  A
 * token outside 0..vocab-1 gives a zero row and DORY_ERR_DEVICE_BOUNDS from
 * dory_device_status. */
DORY_API int dory_embed(dory_vocab* v, const int32_t* d_tokens, int n, void* h_out, void* stream);

/* logits [n, vocab] fp32 (device) = s_z[v] * (emb_out[v] . h[i]) for rows h
 * [n, d_model] bf16 (device), on the tensor-core GEMM. */
DORY_API int dory_lm_head(dory_vocab* v, const void* h, int n, float* logits, void* stream);

/* One token per row of logits [n, vocab] into d_tokens [n] (int32 device).
 * temperature 0: argmax (the lowest index among equal maxima).  temperature
 * > 0: the Gumbel-max draw argmax_v logits[v] / T - log(-log U_v), which
 * samples softmax(logits / T), with U_v = (H(H(H(seed) ^ d_steps[i]) ^ v) +
 * 0.5) / 2^32, H the lowbias32 hash (xorshift 16, * 0x7feb352d, xorshift 15,
 * * 0x846ca68b, xorshift 16), evaluated in double precision; d_steps [n]
 * (int32 device) is each row's step counter, so a draw is a pure function of
 * (seed, step, row's logits). */
DORY_API int dory_sample(dory_vocab* v, const float* logits, int n, float temperature,
                         uint32_t seed, const int32_t* d_steps, int32_t* d_tokens, void* stream);

DORY_API void dory_vocab_free(dory_vocab* v);

/* ---------------------------------------------------------------------
 * Per-kernel timing (diagnostics).  While enabled, calls whose CUDA graph is
 * captured afterwards record a CUDA event before and after every kernel they
 * launch (graphs captured without it are kept separately and stay
 * uninstrumented).  dory_profile_read synchronises on the most recent
 * instrumented call and returns, for one kernel kind, the summed device time
 * in milliseconds and the number of launches of that call.
 * --------------------------------------------------------------------- */
typedef enum dory_kernel_kind {
  DORY_KK_QKVG = 0,      /* QKV + gate projection with RoPE / QK-norm epilogue   */
  DORY_KK_ATTN = 1,      /* prefill attention, or decode split-KV + combine      */
  DORY_KK_OPROJ = 2,     /* output projection                                    */
  DORY_KK_GATEUP = 3,    /* gate/up projection with SwiGLU epilogue              */
  DORY_KK_DOWN = 4,      /* down projection                                      */
  DORY_KK_ROW = 5,       /* nGPT update / re-injection row kernels, input load   */
  DORY_KK_KVCOMMIT = 6,  /* KV-cache slot commits                                */
  DORY_KK_COUNT = 7
} dory_kernel_kind;

DORY_API int dory_profile_enable(dory_model* m, int enable);
DORY_API int dory_profile_read(dory_model* m, int kind, float* total_ms, int* launches);

/* ---------------------------------------------------------------------
 * Single-sublayer entry points (diagnostics and per-sublayer parity).
 * They run exactly the kernels the full pass runs for one sublayer of
 * global block `layer` at loop `loop`, on `n_rows` rows.
 * --------------------------------------------------------------------- */

/* Attention sublayer on rows h [n_rows, d_model] (fp32, device, updated in
 * place) of sequence `seq` at positions pos0.. (prefill semantics, the
 * call's keys committed to the cache after attention). */
DORY_API int dory_attention_sublayer(dory_model* m, dory_kv* kv, int layer, int loop, int seq,
                            int pos0, int n_rows, float* h, void* ws, size_t ws_bytes,
                            void* stream);

/* SwiGLU sublayer on rows h [n_rows, d_model] (fp32, device, in place). */
DORY_API int dory_mlp_sublayer(dory_model* m, int layer, int n_rows, float* h,
                      void* ws, size_t ws_bytes, void* stream);

/* The tensor-core GEMM alone: C[M,N] (fp32) = A[M,K] (bf16) * B[N,K]^T (bf16),
 * all row-major device buffers, K a multiple of 64, N a multiple of 128. */
DORY_API int dory_gemm_bf16(const void* A, const void* B, float* C, int M, int N, int K, void* stream);

/* The same GEMM with a stream-K tail, the schedule of the prefill output and
 * down projections.  A persistent grid of one CTA per SM runs whole
 * 128 x BN tiles (BN = 256 when N is a multiple of 256, else 128); when the
 * tiles leave a partial last wave, the last one-and-a-fraction waves are cut
 * into contiguous runs of k blocks of equal length, one per CTA, so every
 * CTA does the same work.  A tile split between two CTAs is finished by the
 * one holding its first k blocks, which adds the other's fp32 partial
 * (passed through `ws`) in a fixed order: results are identical from call to
 * call, and equal to dory_gemm_bf16's up to fp32 rounding.  `ws` (device,
 * dory_gemm_bf16_streamk_workspace_bytes(N), 256-byte aligned) must be
 * zero-filled before its first use; it keeps a launch counter between
 * calls, so calls sharing one `ws` must not overlap on the GPU.  Every CTA of
 * the grid must be resident at once: kernels running concurrently on other
 * streams can delay the partials.  A CTA that waits more than 2 s for one
 * gives up, stores its tile without it and sets the last 32-bit word of
 * `ws` nonzero (the output is then wrong; zero the word to clear it).
 * Grids of more than 160 CTAs run without the tail.  Same argument rules as
 * dory_gemm_bf16. */
DORY_API size_t dory_gemm_bf16_streamk_workspace_bytes(int N);
DORY_API int dory_gemm_bf16_streamk(const void* A, const void* B, float* C, int M, int N, int K,
                                    void* ws, size_t ws_bytes, void* stream);

/* The same GEMM with operands read transposed (MN-major): A is stored row-major
 * as [M][K] (a_mn = 0) or [K][M] (a_mn = 1), B as [N][K] (b_mn = 0) or [K][N]
 * (b_mn = 1); C[M,N] = A B^T in fp32.  Any K (rounded up inside, the tail read
 * as zeros); N a multiple of 128; the contiguous dimension of each operand a
 * multiple of 8 (16-byte rows).  The backward's dgrad (dX = dY W) and wgrad
 * (dW = dY^T X) products. */
DORY_API int dory_gemm_bf16_mn(const void* A, const void* B, float* C, int M, int N, int K,
                               int a_mn, int b_mn, void* stream);

/* Backward of one MLP sublayer, the building block of the training step that
 * truncated depth-one back-propagation runs over the final recurrent
 * invocation ("Dory1.0-4B: A Looped Normalized-GPT", Methodology in Plain
 * English).  Given the sublayer's input h_in [n_rows, d_model] and dL/dh_out
 * [n_rows, d_model] (fp32, device), recomputes the forward with the inference
 * path's bf16 operands and writes dL/dh_in [n_rows, d_model], dL/dW_gate and
 * dL/dW_up [d_ff, d_model], dL/dW_down [d_model, d_ff] (fp32, row-major like
 * the source matrices) and dL/dalpha_mlp [d_model] (fp32, summed over the
 * rows, deterministic).  All outputs are overwritten.  `ws`:
 * dory_mlp_backward_workspace_bytes(m, n_rows), 256-byte aligned; other
 * buffers 16-byte aligned.  bf16 weight format only (DORY_ERR_BAD_CONFIG
 * otherwise). */
DORY_API size_t dory_mlp_backward_workspace_bytes(const dory_model* m, int n_rows);

/* Backward of one attention sublayer on a training sequence: rows are the
 * positions 0..n_rows-1 of one sequence and every key is one of its own (no KV
 * cache is read or written).  Same page and section as the MLP sublayer's
 * backward.  Given h_in and dL/dh_out [n_rows, d_model] (fp32, device),
 * recomputes the forward (bf16 projection operands; the softmax with each
 * row's exact maximum) and writes dL/dh_in [n_rows, d_model], dL/dW_q
 * [n_q_heads*head_dim, d_model], dL/dW_k and dL/dW_v [n_kv_heads*head_dim,
 * d_model], dL/dW_gate [n_q_heads, d_model], dL/dW_o [d_model,
 * n_q_heads*head_dim], dL/dalpha_attn [d_model] and dL/ds_qk [head_dim]
 * (fp32; the last two summed deterministically).  Attention runs per KV head
 * on the tensor cores with the score matrix of the group's stacked queries
 * held in the workspace, so the workspace
 * (dory_attention_backward_workspace_bytes) grows with n_rows squared.  bf16
 * weight format only (DORY_ERR_BAD_CONFIG otherwise). */
/* Depth-one truncated back-propagation through the stack for one training
 * sequence ("Dory1.0-4B: A Looped Normalized-GPT", Methodology in Plain
 * English: only the final recurrent invocation is trained).  h_in [n_rows,
 * d_model] (fp32, device; the sequence's positions 0..n_rows-1) runs forward
 * as a prefill into `kv` (sequence 0, max_ctx >= n_rows): the input block,
 * k - 1 loops of the recurrent block with re-injection, the final loop and the
 * output block; the loops before the last are not differentiated, so their
 * output x_k is a constant.  dL/dh_out [n_rows, d_model] then flows back
 * through the output block and the final recurrent invocation.  Writes the
 * output (h_out, optional), dL/dx_k [n_rows, d_model] (dx) and into `grads`
 * the fp32 gradients of every trained block -- the n_rec_blocks recurrent
 * blocks then the n_out_blocks output blocks, each as W_q, W_k, W_v, W_gate,
 * W_o, W_mlp_gate, W_up, W_down (the shapes of dory_block_src), alpha_attn,
 * alpha_mlp, s_qk, each tensor 256-byte aligned at the offset
 * dory_last_loop_grad_layout reports (offsets[i * 11 + t] for trained block
 * i, tensor t; it returns the total bytes).  bf16 weight format only. */
DORY_API size_t dory_last_loop_grad_layout(const dory_model* m, size_t* offsets);
DORY_API size_t dory_last_loop_backward_workspace_bytes(const dory_model* m, int n_rows);
DORY_API int dory_last_loop_backward(dory_model* m, dory_kv* kv, int n_rows, const float* h_in,
                                     const float* dh_out, int k, float* h_out, float* dx,
                                     void* grads, size_t grad_bytes, void* ws, size_t ws_bytes,
                                     void* stream);

DORY_API size_t dory_attention_backward_workspace_bytes(const dory_model* m, int n_rows);
DORY_API int dory_attention_sublayer_backward(dory_model* m, int layer, int n_rows,
                                              const float* h_in, const float* dh_out, float* dh_in,
                                              float* d_wq, float* d_wk, float* d_wv, float* d_wg,
                                              float* d_wo, float* d_alpha, float* d_s_qk, void* ws,
                                              size_t ws_bytes, void* stream);
DORY_API int dory_mlp_sublayer_backward(dory_model* m, int layer, int n_rows, const float* h_in,
                                        const float* dh_out, float* dh_in, float* d_w_gate,
                                        float* d_w_up, float* d_w_down, float* d_alpha, void* ws,
                                        size_t ws_bytes, void* stream);

/* MXFP8 quantisation along K of bf16 rows src [rows, K] (device, K a multiple
 * of 128): E4M3 codes [rows, K] bytes into `codes`, E8M0 scale codes into
 * `scales` (dory_mxfp8_scale_bytes) in 512-byte chunks, one per 128 rows x
 * 128 K: chunk (kc, rb) at (kc * ceil(rows/128) + rb) * 512, the scale of row
 * rb*128 + 32*j + i and K block q (0..3) of the chunk at byte i*16 + j*4 + q;
 * padding rows of the last chunk hold code 127.  Same rule as weight_format
 * DORY_WEIGHTS_MXFP8. */
DORY_API int dory_quant_mxfp8(const void* src, int rows, int K, void* codes, void* scales,
                              void* stream);
DORY_API size_t dory_mxfp8_scale_bytes(int rows, int K);

/* The block-scaled (MXFP8 x MXFP8) tensor-core GEMM alone: quantises A [M,K]
 * and B [N,K] (bf16, device) into `ws` (dory_gemm_mxfp8_workspace_bytes, 256-byte
 * aligned) and writes C = Q(A) Q(B)^T in fp32, split over K into k_splits
 * slices C[s][M][N] (1..8) whose sum is the product.  K a multiple of 128. */
DORY_API size_t dory_gemm_mxfp8_workspace_bytes(int M, int N, int K);
DORY_API int dory_gemm_mxfp8(const void* A, const void* B, float* C, int M, int N, int K,
                             int k_splits, void* ws, size_t ws_bytes, void* stream);

/* NVFP4 quantisation along K of bf16 rows src [rows, K] (device, K a multiple
 * of 256) under the tensor scale g: g > 0 as given, else g = amax / (6 * 448)
 * of src computed on the device and written to d_g (a device float, also used
 * as scratch).  Packed E2M1 codes [rows, K / 2] bytes into `codes` (element 2i
 * in the low nibble of byte i), E4M3 block scale codes into `scales`
 * (dory_nvfp4_scale_bytes) in 2048-byte chunks, one per 128 rows x 256 K:
 * chunk (kc, rb) at (kc * ceil(rows/128) + rb) * 2048, the scale of row
 * rb*128 + 32*j + i and 16-block b (0..15) of the chunk at byte
 * (b / 4) * 512 + i*16 + j*4 + b % 4; padding rows of the last chunk hold
 * 0x38 (1.0).  Same rule as weight_format DORY_WEIGHTS_NVFP4. */
DORY_API int dory_quant_nvfp4(const void* src, int rows, int K, float g, float* d_g, void* codes,
                              void* scales, void* stream);
DORY_API size_t dory_nvfp4_scale_bytes(int rows, int K);

/* The block-scaled (NVFP4 x NVFP4) tensor-core GEMM alone: quantises A [M,K]
 * under tensor scale g_a and B [N,K] under g_b (bf16, device; both scales
 * > 0) into `ws` (dory_gemm_nvfp4_workspace_bytes, 256-byte aligned) and
 * writes C = Q(A) Q(B)^T in fp32 (the product of the two tensor scales
 * applied to the accumulators), split over K into k_splits slices C[s][M][N]
 * (1..8) whose sum is the product.  K a multiple of 256. */
DORY_API size_t dory_gemm_nvfp4_workspace_bytes(int M, int N, int K);
DORY_API int dory_gemm_nvfp4(const void* A, const void* B, float* C, int M, int N, int K,
                             float g_a, float g_b, int k_splits, void* ws, size_t ws_bytes,
                             void* stream);

/* ---------------------------------------------------------------------
 * Mask and failure-path diagnostics.
 * --------------------------------------------------------------------- */

/* Mask probe.  The attention of a looped nGPT block is causal, and a
 * sliding-window layer sees only the last `window` keys up to and including
 * the query ("Dory1.0-4B: A Looped Normalized-GPT", Methodology in Plain
 * English: interleaved sliding-window and full-attention layers).  While a
 * probe is set, every attention launch of global block `layer` in later calls
 * (dory_prefill, dory_decode_step(_mixed), dory_attention_sublayer) first
 * resets and then fills, per (row, query head), the record
 *   {first key position given a nonzero softmax weight, last such position,
 *    number of such keys, sum of their positions mod 2^32}
 * in d_probe: int32 [max_rows][n_q_heads][4], device, caller-owned, 16-byte
 * aligned.  Rows are the call's tokens (prefill) or batch rows (decode).  A
 * recurrent block's record holds its last loop's launch (every loop uses the
 * same mask).  A call with more rows than max_rows fails with DORY_ERR_CUDA.
 * Calls captured while a probe is set use separate CUDA graphs with the
 * recording kernels; d_probe = NULL switches the probe off (layer and
 * max_rows are then ignored). */
DORY_API int dory_debug_mask_probe(dory_model* m, int layer, int32_t* d_probe, int max_rows);

/* Prefill projections with the nGPT update h <- Norm(h + alpha * (Norm(y) - h))
 * (and the loop re-injection) applied in the output / down projection's
 * epilogue, a cluster of CTAs covering each row of d_model columns and
 * exchanging per-row partial sums through distributed shared memory
 * ("Dory1.0-4B: A Looped Normalized-GPT", Methodology in Plain English).
 * enable = 1 makes later prefill calls use it; the default (enable = 0) is the
 * unfused path (projection to fp32, then a row kernel), measured faster on
 * B200 at the 4B shape; decode steps always use the unfused path.  Returns
 * DORY_ERR_BAD_CONFIG when d_model has no fused kernel (not a multiple of 384,
 * 256 or 128 with at most 8 CTAs per row); such models always run unfused. */
DORY_API int dory_debug_fused_update(dory_model* m, int enable);

/* Stream-K tails in the prefill output and down projections (the schedule of
 * dory_gemm_bf16_streamk over the model's own slots).  enable = 1 makes later
 * prefill calls use them; the default (enable = 0) runs whole tiles only,
 * measured faster on B200 at the 4B shape under its power cap: with every SM
 * busy through the last wave the clock drops more than the idle share of that
 * wave costs.  Returns DORY_ERR_BAD_CONFIG where the device has more SMs than
 * the model buffer has slots (the tails then stay off). */
DORY_API int dory_debug_stream_k(dory_model* m, int enable);

/* Attention kernels launched by the most recent call, by kind:
 * counts[0] tensor-core (tcgen05) prefill attention, counts[1] mma.sync
 * prefill attention (head_dim 64, or a pos0 / window that is not a multiple
 * of 128), counts[2] TMA-fed decode attention, counts[3] cp.async decode
 * attention (head_dim 64, or a window that is not a multiple of 64). */
DORY_API int dory_debug_attention_paths(const dory_model* m, int32_t counts[4]);

/* Failure-path test aid (no counterpart on the pages).  Every wait inside the
 * library's kernels gives up after a bounded time and records a timeout in the
 * model's device status word instead of hanging the GPU.  This launches one
 * small kernel whose only wait is on a barrier that nothing ever completes,
 * with a limit of `limit_us` microseconds (1 .. 1000000); no copy or MMA is in
 * flight.  After it, dory_device_status returns DORY_ERR_DEVICE_TIMEOUT once
 * (and clears the word). */
DORY_API int dory_debug_wait_timeout(dory_model* m, uint32_t limit_us, void* stream);

/* ---------------------------------------------------------------------
 * Allocation-free variant (no counterpart in the paper: a deployment aid).
 *
 * Some callers cannot allocate device memory at all: code running where
 * cudaMalloc is forbidden or unavailable (inside another allocator's hooks,
 * in a process whose memory pool is fixed up front, or in a plugin that
 * receives only its input and output buffers).  They cannot provide the
 * workspace that dory_mlp_sublayer needs.  dory_mlp_sublayer_noalloc runs
 * the same SwiGLU sublayer (same kernels, same results) with its scratch --
 * the bf16 copy of h, the SwiGLU activations and the fp32 projection output
 * -- in a fixed array of DORY_NOALLOC_SCRATCH_BYTES that is part of the
 * library itself: every GPU that loads the library holds this array until the
 * process exits.  The caller passes only the rows h [n_rows, d_model] (fp32,
 * device, updated in place).
 *
 * Limit: with A(x) = x rounded up to 256, the call needs
 *   A(2*n_rows*d_model) + A(2*n_rows*d_ff) + A(4*n_rows*d_model)
 * bytes; larger n_rows return DORY_ERR_SCRATCH_LIMIT without launching
 * anything (about 227 rows for d_model 3072, d_ff 9216).
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  The call itself allocates nothing.  All calls
 * share the one array and it keeps the last call's contents; each call writes
 * every scratch byte before reading it, so nothing needs clearing.  Calls
 * that may overlap on the GPU (different streams, or graphs replayed
 * concurrently) race on the array: serialise them.
 * --------------------------------------------------------------------- */
#define DORY_NOALLOC_SCRATCH_BYTES (8u << 20)

DORY_API int dory_mlp_sublayer_noalloc(dory_model* m, int layer, int n_rows, float* h,
                                       void* stream);
/* (Models with block-scaled weights, MXFP8 or NVFP4, return DORY_ERR_BAD_CONFIG.) */

#ifdef __cplusplus
}
#endif

#endif /* DORY_H */
