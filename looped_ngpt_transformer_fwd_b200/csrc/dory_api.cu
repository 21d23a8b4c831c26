// C ABI of the looped nGPT forward-pass library: model and KV-cache handles,
// weight packing, workspace layout, and the loop controller that runs
//   input block (once) -> recurrent block (k times, re-injecting the input
//   block's output before every pass) -> output block (once)
// ("Dory1.0-4B: A Looped Normalized-GPT", Key Contributions item 1 and
// Methodology in Plain English; "Dory 1.0 4B Benchmarks: How Do 1, 2 and 4
// Loops Compare?", How does looping work at inference time?) as one CUDA graph
// per call shape.  The recurrent blocks' weights are the same device pointers
// in every loop: re-read, never copied.  KV caches follow the per-loop (one
// cache per loop of a recurrent layer) or last-loop (one cache per layer,
// overwritten by every loop) mode of the same passages.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <map>
#include <mutex>
#include <set>
#include <memory>
#include <new>
#include <tuple>
#include <vector>

#include "dory.h"
#include "common.cuh"
#include "kernels.h"

using namespace dory;

namespace {

constexpr size_t kAlign = 256;
constexpr int kMaxDecodeRows = 256;     // decode batch limit of a workspace
constexpr int kMaxDecodeSplits = 64;    // split-KV slices per (sequence, head)
constexpr int kMaxKSplits = 8;

size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }

bool is_aligned(const void* p, size_t a = kAlign) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

bool is_device_ptr(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

struct BlockW {
  __nv_bfloat16* wqkvg = nullptr;   // [n_qkvg, d]: q | k | v | gate rows
  __nv_bfloat16* wo = nullptr;      // [d, Hq*hd]
  __nv_bfloat16* wgu = nullptr;     // [2*ff, d]: 128 gate rows, 128 up rows, ...
  __nv_bfloat16* wd = nullptr;      // [d, ff]
  float* alpha_attn = nullptr;
  float* alpha_mlp = nullptr;
  float* s_qk = nullptr;
  bool full = false;
  bool recurrent = false;
  float m_log2 = 0.f;   // static softmax maximum: softmax_scale * log2(e) * max s_qk^2
  // B-operand tensor maps, box rows 128 and 256
  CUtensorMap tm_qkvg[2], tm_o[2], tm_gu[2], tm_d[2];
  // W_o / W_down for the fused projection + nGPT update (box rows = one MMA's N)
  CUtensorMap tm_o_n, tm_d_n;
  // Block-scaled weights (weight_format MXFP8: E4M3 codes, E8M0 scale chunks;
  // NVFP4: packed E2M1 codes, E4M3 scale chunks), scale chunks covering whole
  // 256-row tiles; gate / up rows interleaved in groups of 64
  uint8_t *q8 = nullptr, *o8 = nullptr, *gu8 = nullptr, *d8 = nullptr;
  uint8_t *qsf = nullptr, *osf = nullptr, *gusf = nullptr, *dsf = nullptr;
  CUtensorMap tm8_qkvg, tm8_o, tm8_gu, tm8_d;                  // 128-row boxes (decode)
  CUtensorMap tm8_qkvg_256, tm8_o_256, tm8_gu_256, tm8_d_256;  // 256-row boxes (prefill)
  // NVFP4 tensor scales of the four projections' weights (one per GEMM: the
  // q | k | v | gate rows share one, as do the gate and up rows), on the
  // device (tscale) and copied to the host once they are computed
  float* tscale = nullptr;
  float g_qkvg = 1.f, g_o = 1.f, g_gu = 1.f, g_d = 1.f;
};

// Tensor scale of every NVFP4 projection input: the rows are unit vectors
// (the stream h, and the attention output and SwiGLU activations after their
// L2 norm), so no element exceeds 1 and g = 1 / (6 * 448) keeps every block
// scale amax / (6 g) <= 448 within E4M3's range.
constexpr float kNvfp4ActScale = static_cast<float>(1.0 / 2688.0);

struct GraphKey {
  int phase, k, n, seq, pos0, max_pos, prof;
  const void *src, *dst, *ws;
  uint64_t kv;              // unique id of the KV cache (handles may be recycled)
  const void *dseq, *dpos;
  const void* dk;           // per-row loop counts (mixed-k decode), else null
  const void* probe;        // mask-probe records (diagnostics), else null
  int probe_layer;
  int fused;                // nGPT update fused into the prefill projections (bit 0), stream-K tails (bit 1)
  bool operator<(const GraphKey& o) const {
    return std::tie(phase, k, n, seq, pos0, max_pos, prof, src, dst, ws, kv, dseq, dpos, dk, probe,
                    probe_layer, fused) <
           std::tie(o.phase, o.k, o.n, o.seq, o.pos0, o.max_pos, o.prof, o.src, o.dst, o.ws, o.kv,
                    o.dseq, o.dpos, o.dk, o.probe, o.probe_layer, o.fused);
  }
};

// attention kernels launched by one call, by kind (see dory_debug_attention_paths)
enum { kPathPrefillTc = 0, kPathPrefillMma = 1, kPathDecodeTma = 2, kPathDecodeCp = 3, kPaths = 4 };

// events around one kernel launch of an instrumented graph
struct Mark {
  int kind;
  cudaEvent_t start, end;
};

struct GraphEntry {
  cudaGraphExec_t exec = nullptr;
  int launches = 0, sublayers = 0;
  int paths[kPaths] = {0, 0, 0, 0};
  uint64_t last_use = 0;
  std::vector<Mark> marks;
};

void destroy_entry(GraphEntry& g) {
  if (g.exec) cudaGraphExecDestroy(g.exec);
  for (auto& mk : g.marks) {
    cudaEventDestroy(mk.start);
    cudaEventDestroy(mk.end);
  }
  g.marks.clear();
  g.exec = nullptr;
}

}  // namespace

struct dory_model {
  dory_config cfg;
  int d, hq, hkv, hd, ff, d_attn, n_qkvg, nb;
  int ld_qkvg;   // row pitch (floats) of the decode QKVG partial products: n_qkvg rounded up to 32
  // fused projection + nGPT update (prefill): columns per CTA (0 = not
  // available for this d_model), CTAs per cluster, and whether it is used.
  // Off by default: with an 8-CTA cluster per 3072-column row only 15 clusters
  // (120 of 148 SMs) are co-resident, and a 4096-token projection then takes
  // three waves; the unfused projection + row kernel measured faster.
  int ngpt_bnc = 0, ngpt_cluster = 0;
  bool fused_update = false;
  int mx = kOperandsBf16;   // block-scaled weights and projection inputs (MXFP8 or NVFP4)
  // stream-K tail of the prefill output and down projections (GemmParams.sk).
  // Off by default: at 4096 tokens it measured 3 % slower per step on B200
  // under the 1000 W cap (output projection 4.97 against 4.54 ms per step,
  // down 11.9 against 11.6): with every SM busy to the end the clock drops
  // (median 1510 against 1560 MHz), and split tiles add epilogues.
  float* sk_ws = nullptr;
  uint32_t* sk_sync = nullptr;
  bool stream_k = false;
  int device = 0, num_sms = 148;
  uint8_t* wbuf = nullptr;
  size_t wbytes = 0;
  uint32_t* status = nullptr;
  double* inv_freq_swa = nullptr;
  double* inv_freq_full = nullptr;
  std::vector<BlockW> blocks;
  cudaStream_t cap_stream = nullptr;
  // the attention backward runs its KV heads concurrently on these (created on
  // first use, forked from and joined to the caller's stream by events)
  std::vector<cudaStream_t> aux_streams;
  std::vector<cudaEvent_t> aux_events;
  cudaEvent_t fork_event = nullptr;
  std::map<GraphKey, GraphEntry> graphs;
  uint64_t tick = 0;
  int last_launches = 0, last_sublayers = 0;
  int last_paths[kPaths] = {0, 0, 0, 0};
  // counters of the call being enqueued
  int cur_launches = 0, cur_sublayers = 0;
  int cur_paths[kPaths] = {0, 0, 0, 0};
  // mask probe (diagnostics): records of attention launches of block probe_layer
  int32_t* probe = nullptr;
  int probe_layer = -1, probe_rows = 0;
  // per-kernel timing
  bool profile = false;
  std::vector<Mark>* cur_marks = nullptr;      // marks of the graph being captured
  const std::vector<Mark>* last_marks = nullptr;
  std::set<dory_kv*> caches;                   // live KV caches bound to this model
};

// tensors of one trained block's gradients, in the order of dory_last_loop_grad_layout
constexpr int kGradTensors = 11;

struct dory_kv {
  dory_model* m = nullptr;
  uint64_t uid = 0;
  int mode = 0, max_seqs = 0, max_ctx = 0, k_max = 1;
  uint8_t* buf = nullptr;
  size_t bytes = 0;
  // per block: first slot's byte offset, capacity, number of loop slots
  std::vector<size_t> base;
  std::vector<int> cap, loops;
  std::vector<int> seq_k;   // per sequence: k of its last prefill (per-loop mode checks)
};

namespace {

// ------------------------------------------------------------------ layouts
int n_blocks(const dory_config* c) { return c->n_in_blocks + c->n_rec_blocks + c->n_out_blocks; }

bool is_full(const dory_config* c, int b) { return (b % c->full_period) == c->full_period - 1; }

bool is_recurrent(const dory_config* c, int b) {
  return b >= c->n_in_blocks && b < c->n_in_blocks + c->n_rec_blocks;
}

int validate_config(const dory_config* c) {
  if (!c) return DORY_ERR_INVALID_ARG;
  if (c->head_dim != 64 && c->head_dim != 128) return DORY_ERR_BAD_CONFIG;
  if (c->n_q_heads <= 0 || c->n_kv_heads <= 0 || c->n_q_heads % c->n_kv_heads) return DORY_ERR_BAD_CONFIG;
  if (c->n_q_heads / c->n_kv_heads > 4) return DORY_ERR_BAD_CONFIG;
  if (c->d_model != c->n_q_heads * c->head_dim) return DORY_ERR_BAD_CONFIG;
  if (c->d_model % 128 || c->d_ff % 128 || c->d_model > 4096 || c->d_model < 128) return DORY_ERR_BAD_CONFIG;
  if (c->n_in_blocks < 1 || c->n_rec_blocks < 1 || c->n_out_blocks < 1) return DORY_ERR_BAD_CONFIG;
  if (c->window < 1 || c->full_period < 1) return DORY_ERR_BAD_CONFIG;
  if (!(c->rope_base_swa > 1.0) || !(c->rope_base_full > 1.0)) return DORY_ERR_BAD_CONFIG;
  if (!(c->softmax_scale > 0.f) || !(c->norm_eps > 0.f)) return DORY_ERR_BAD_CONFIG;
  if (c->weight_format != DORY_WEIGHTS_BF16 && c->weight_format != DORY_WEIGHTS_MXFP8 &&
      c->weight_format != DORY_WEIGHTS_NVFP4)
    return DORY_ERR_BAD_CONFIG;
  // NVFP4 GEMMs take K in steps of 256
  if (c->weight_format == DORY_WEIGHTS_NVFP4 && (c->d_model % 256 || c->d_ff % 256))
    return DORY_ERR_BAD_CONFIG;
  return DORY_OK;
}

// stream-K slots of the prefill output / down projections kept in the model
// buffer (a CTA per SM: enough for B200's 148; larger grids run without)
constexpr int kSkMaxGrid = 160;

struct WeightLayout {
  size_t header = 0;                 // status word + RoPE tables + stream-K workspace
  size_t sk = 0;                     // stream-K workspace (gemm_sk_workspace_bytes)
  size_t per_block = 0;
  size_t off_qkvg = 0, off_o = 0, off_gu = 0, off_d = 0, off_aa = 0, off_am = 0, off_sqk = 0;
  // MXFP8 / NVFP4: codes and scale chunks of the four matrices; NVFP4 tensor
  // scales (4 floats) and an amax scratch word
  size_t off_q8 = 0, off_qsf = 0, off_o8 = 0, off_osf = 0, off_gu8 = 0, off_gusf = 0, off_d8 = 0,
         off_dsf = 0, off_ts = 0;
  size_t total = 0;
};

WeightLayout weight_layout(const dory_config* c) {
  WeightLayout L;
  const size_t d = c->d_model, hd = c->head_dim, da = size_t(c->n_q_heads) * hd, ff = c->d_ff;
  const size_t nq = da + 2 * size_t(c->n_kv_heads) * hd + c->n_q_heads;
  L.sk = align_up(64) + 2 * align_up(hd / 2 * sizeof(double));
  L.header = L.sk + align_up(gemm_sk_workspace_bytes(kSkMaxGrid, 256));
  size_t o = 0;
  if (c->weight_format == DORY_WEIGHTS_MXFP8) {
    L.off_q8 = o;   o = align_up(o + nq * d);
    // weight scale chunks cover whole 256-row tiles
    L.off_qsf = o;  o = align_up(o + mxfp8_scale_bytes(int(nq), int(d), 256));
    L.off_o8 = o;   o = align_up(o + d * da);
    L.off_osf = o;  o = align_up(o + mxfp8_scale_bytes(int(d), int(da), 256));
    L.off_gu8 = o;  o = align_up(o + 2 * ff * d);
    L.off_gusf = o; o = align_up(o + mxfp8_scale_bytes(int(2 * ff), int(d), 256));
    L.off_d8 = o;   o = align_up(o + d * ff);
    L.off_dsf = o;  o = align_up(o + mxfp8_scale_bytes(int(d), int(ff), 256));
  } else if (c->weight_format == DORY_WEIGHTS_NVFP4) {
    L.off_q8 = o;   o = align_up(o + nq * d / 2);
    L.off_qsf = o;  o = align_up(o + nvfp4_scale_bytes(int(nq), int(d), 256));
    L.off_o8 = o;   o = align_up(o + d * da / 2);
    L.off_osf = o;  o = align_up(o + nvfp4_scale_bytes(int(d), int(da), 256));
    L.off_gu8 = o;  o = align_up(o + 2 * ff * d / 2);
    L.off_gusf = o; o = align_up(o + nvfp4_scale_bytes(int(2 * ff), int(d), 256));
    L.off_d8 = o;   o = align_up(o + d * ff / 2);
    L.off_dsf = o;  o = align_up(o + nvfp4_scale_bytes(int(d), int(ff), 256));
    L.off_ts = o;   o = align_up(o + 8 * sizeof(float));
  } else {
    L.off_qkvg = o; o = align_up(o + nq * d * 2);
    L.off_o = o;    o = align_up(o + d * da * 2);
    L.off_gu = o;   o = align_up(o + 2 * ff * d * 2);
    L.off_d = o;    o = align_up(o + d * ff * 2);
  }
  L.off_aa = o;   o = align_up(o + d * 4);
  L.off_am = o;   o = align_up(o + d * 4);
  L.off_sqk = o;  o = align_up(o + hd * 4);
  L.per_block = o;
  L.total = L.header + L.per_block * n_blocks(c);
  return L;
}

struct WsLayout {
  size_t h32, e32, hb, st_in, st_out, q, kf, vf, gate, o, y, a, dacc, dml, rope_swa, rope_full,
      part, x8, xsf, total;
  int y_rows;
};

WsLayout ws_layout(const dory_model* m, int T) {
  WsLayout L;
  const size_t d = m->d, da = m->d_attn, kvw = size_t(m->hkv) * m->hd, ff = m->ff;
  const int dec_rows = std::min(T, kMaxDecodeRows);
  L.y_rows = std::max(T, kMaxKSplits * dec_rows);
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes); return at; };
  L.h32 = take(size_t(T) * d * 4);
  L.e32 = take(size_t(T) * d * 4);
  L.hb = take(size_t(T) * d * 2);
  L.st_in = take(size_t(T) * d * 2);
  L.st_out = take(size_t(T) * d * 2);
  L.q = take(size_t(T) * da * 2);
  L.kf = take(size_t(T) * kvw * 2);
  L.vf = take(size_t(T) * kvw * 2);
  L.gate = take(size_t(T) * m->hq * 4);
  L.o = take(size_t(T) * da * 2);
  L.y = take(size_t(L.y_rows) * d * 4);
  L.a = take(size_t(T) * ff * 2);
  L.dacc = take(size_t(dec_rows) * m->hq * kMaxDecodeSplits * m->hd * 4);
  L.dml = take(size_t(dec_rows) * m->hq * kMaxDecodeSplits * 2 * 4);
  L.rope_swa = take(size_t(T) * (m->hd / 2) * 8);
  L.rope_full = take(size_t(T) * (m->hd / 2) * 8);
  // K-split partial products of the decode QKVG and gate/up projections
  L.part = take(size_t(dec_rows) * kMaxKSplits * std::max<size_t>(m->ld_qkvg, 2 * ff) * 4);
  // block-scaled modes: the current projection's input as codes and scale
  // chunks
  const int kmax = std::max(m->d, std::max(m->d_attn, m->ff));
  L.x8 = m->mx ? take(size_t(T) * kmax) : o;
  L.xsf = m->mx ? take(m->mx == kOperandsNvfp4 ? nvfp4_scale_bytes(T, kmax)
                                                : mxfp8_scale_bytes(T, kmax))
                : o;
  L.total = o;
  return L;
}

struct Ws {
  float *h32, *e32, *y, *gate, *dacc, *dml, *part;
  __nv_bfloat16 *hb, *st_in, *st_out, *q, *kf, *vf, *o, *a;
  float2 *rope_swa, *rope_full;
  uint8_t *x8, *xsf;
};

Ws ws_bind(const dory_model* m, void* base, int T) {
  const WsLayout L = ws_layout(m, T);
  uint8_t* b = static_cast<uint8_t*>(base);
  Ws w;
  w.h32 = reinterpret_cast<float*>(b + L.h32);
  w.e32 = reinterpret_cast<float*>(b + L.e32);
  w.hb = reinterpret_cast<__nv_bfloat16*>(b + L.hb);
  w.st_in = reinterpret_cast<__nv_bfloat16*>(b + L.st_in);
  w.st_out = reinterpret_cast<__nv_bfloat16*>(b + L.st_out);
  w.q = reinterpret_cast<__nv_bfloat16*>(b + L.q);
  w.kf = reinterpret_cast<__nv_bfloat16*>(b + L.kf);
  w.vf = reinterpret_cast<__nv_bfloat16*>(b + L.vf);
  w.gate = reinterpret_cast<float*>(b + L.gate);
  w.o = reinterpret_cast<__nv_bfloat16*>(b + L.o);
  w.y = reinterpret_cast<float*>(b + L.y);
  w.a = reinterpret_cast<__nv_bfloat16*>(b + L.a);
  w.dacc = reinterpret_cast<float*>(b + L.dacc);
  w.dml = reinterpret_cast<float*>(b + L.dml);
  w.rope_swa = reinterpret_cast<float2*>(b + L.rope_swa);
  w.rope_full = reinterpret_cast<float2*>(b + L.rope_full);
  w.part = reinterpret_cast<float*>(b + L.part);
  w.x8 = b + L.x8;
  w.xsf = b + L.xsf;
  return w;
}

KvLayerView kv_view(const dory_kv* kv, int b, int loop) {
  const dory_model* m = kv->m;
  KvLayerView v;
  const int slot = (kv->loops[b] > 1) ? (loop - 1) : 0;
  const size_t cap = kv->cap[b];
  const size_t seq_elems = 2 * size_t(m->hkv) * cap * m->hd;
  uint8_t* base = kv->buf + kv->base[b] + size_t(slot) * kv->max_seqs * seq_elems * 2;
  v.k_base = reinterpret_cast<__nv_bfloat16*>(base);
  v.v_base = v.k_base + size_t(m->hkv) * cap * m->hd;
  v.seq_stride = seq_elems;
  v.cap = kv->cap[b];
  v.n_kv = m->hkv;
  v.hd = m->hd;
  v.max_seqs = kv->max_seqs;
  v.max_ctx = kv->max_ctx;
  return v;
}

// ------------------------------------------------------------------ kernels of one block
struct CallCtx {
  dory_model* m;
  dory_kv* kv;
  Ws w;
  int n;                 // rows
  bool decode;
  int seq, pos0;         // prefill
  const int32_t *dseq, *dpos;
  int max_pos;
  int k;                 // loops run (the largest per-row count when dk is set)
  const int32_t* dk = nullptr;   // decode: per-row loop counts, or null
  cudaStream_t s;
  // block-scaled modes: the last row update already wrote the stream's codes
  // and scales into the projection-input buffer (w.x8 / w.xsf)
  bool h_quantized = false;
};

#define DORY_TRY(expr)                         \
  do {                                         \
    cudaError_t _e = (expr);                   \
    if (_e != cudaSuccess) return _e;          \
  } while (0)

// Bracket one kernel launch with events when the graph being captured is
// instrumented; counts the launch either way.
struct Launch {
  dory_model* m;
  cudaStream_t s;
  Mark mk{};
  bool on = false;
  Launch(dory_model* m_, cudaStream_t s_, int kind) : m(m_), s(s_) {
    ++m->cur_launches;
    if (m->cur_marks && cudaEventCreate(&mk.start) == cudaSuccess) {
      if (cudaEventCreate(&mk.end) == cudaSuccess) {
        mk.kind = kind;
        // external records become event nodes of the captured graph
        on = cudaEventRecordWithFlags(mk.start, s, cudaEventRecordExternal) == cudaSuccess;
        if (!on) {
          cudaEventDestroy(mk.start);
          cudaEventDestroy(mk.end);
        }
      } else {
        cudaEventDestroy(mk.start);
      }
    }
  }
  ~Launch() {
    if (on) {
      if (cudaEventRecordWithFlags(mk.end, s, cudaEventRecordExternal) == cudaSuccess) {
        m->cur_marks->push_back(mk);
      } else {
        cudaEventDestroy(mk.start);
        cudaEventDestroy(mk.end);
      }
    }
  }
};

int pick_k_splits(const dory_model* m, int M, int N, int BN, int K) {
  const int tiles = ((M + 127) / 128) * ((N + BN - 1) / BN);
  if (tiles >= m->num_sms / 2) return 1;
  const int kstep = m->mx == kOperandsNvfp4 ? 256 : (m->mx ? 128 : 64);   // K per pipeline stage
  int s = std::max(1, m->num_sms / tiles);
  s = std::min(s, kMaxKSplits);
  s = std::min(s, std::max(1, (K / kstep) / 4));
  // the kernel gives each split ceil(kb / s) k-blocks: drop splits left empty
  const int kb = K / kstep, per = (kb + s - 1) / s;
  return (kb + per - 1) / per;
}

// The A operand of a projection over this call's rows: the bf16 rows, or in
// the block-scaled modes their MXFP8 / NVFP4 codes and scales (from the fp32
// stream `f32`, or from bf16 rows scaled to unit L2 norm first when
// `normalize`; the norms before the output and down projections are applied
// here, where quantisation makes them matter).  Sets the tensor map and the
// block-scaled fields of g (NVFP4: alpha starts as the inputs' tensor scale).
cudaError_t projection_input(CallCtx& c, CUtensorMap* tm, GemmParams& g, const __nv_bfloat16* rows,
                             const float* f32, int K, bool normalize) {
  dory_model* m = c.m;
  if (!m->mx) {
    if (!make_tmap_bf16(tm, rows, c.n, K, 128)) return cudaErrorInvalidValue;
    return cudaSuccess;
  }
  const bool nv = m->mx == kOperandsNvfp4;
  const bool ready = f32 && c.h_quantized;   // the row kernel quantised the stream already
  c.h_quantized = false;                     // any other input overwrites the buffer
  if (!ready) {
    Launch L(m, c.s, DORY_KK_ROW);
    const float eps = m->cfg.norm_eps;
    const int nrm = normalize ? 1 : 0;
    const __nv_bfloat16* seg[1] = {rows};
    if (nv && f32) {
      DORY_TRY(launch_quant_nvfp4_f32(f32, c.n, K, 0, eps, nullptr, kNvfp4ActScale, c.w.x8,
                                      c.w.xsf, c.s));
    } else if (nv) {
      DORY_TRY(launch_quant_nvfp4_bf16(seg, nullptr, 1, 0, c.n, 128, K, nrm, eps, nullptr,
                                       kNvfp4ActScale, c.w.x8, c.w.xsf, c.s));
    } else if (f32) {
      DORY_TRY(launch_quant_mxfp8_f32(f32, c.n, K, 0, eps, c.w.x8, c.w.xsf, c.s));
    } else {
      DORY_TRY(launch_quant_mxfp8_bf16(seg, nullptr, 1, 0, c.n, 128, K, nrm, eps, c.w.x8, c.w.xsf,
                                       c.s));
    }
  }
  // NVFP4 rows hold K / 2 bytes (two codes per byte)
  if (!make_tmap_u8(tm, c.w.x8, c.n, nv ? K / 2 : K, 128)) return cudaErrorInvalidValue;
  g.mx = m->mx;
  g.sfa = c.w.xsf;
  g.sfa_blocks = (c.n + 127) / 128;
  g.alpha = nv ? kNvfp4ActScale : 1.f;
  return cudaSuccess;
}

// Let a row update quantise its result for the next projection (the stream
// is the input of the QKVG and gate / up projections), sparing a pass of the
// stand-alone quantiser.  Not with per-row loop counts: rows whose loops are
// done are skipped and would keep stale codes.
void fuse_stream_quant(CallCtx& c, RowUpdateParams& r) {
  if (!c.m->mx || c.dk) return;
  r.q_fmt = c.m->mx;
  r.q_codes = c.w.x8;
  r.q_scales = c.w.xsf;
  r.q_row_blocks = (c.n + 127) / 128;
  r.q_g = kNvfp4ActScale;
}

// B operand (weights) of the block-scaled GEMMs: scale chunks and their row
// blocks (weights' chunks cover whole 256-row tiles), and for NVFP4 the
// weights' tensor scale g_w into alpha
void mx_weights(GemmParams& g, const uint8_t* sf, int n_rows, float g_w) {
  g.sfb = sf;
  g.sfb_blocks = (n_rows + 255) / 256 * 2;
  if (g.mx == kOperandsNvfp4) g.alpha *= g_w;
}

// Launch-shape switches a captured graph depends on (GraphKey.fused).
int graph_modes(const dory_model* m) { return (m->fused_update ? 1 : 0) | (m->stream_k ? 2 : 0); }

// Prefill output / down projections: the stream-K tail over the model's
// slots (the launcher keeps it only where the tiles leave a partial wave).
void streamk_tail(const CallCtx& c, GemmParams& g) {
  if (c.decode || !c.m->stream_k || !c.m->sk_ws) return;
  g.sk = 1;
  g.sk_ws = c.m->sk_ws;
  g.sk_sync = c.m->sk_sync;
}

// Prefill projections with the nGPT update in their epilogue (a cluster of
// CTAs covers each row); decode keeps K-split GEMMs and the row kernel, which
// spread its few rows' weight stream over all SMs.
bool use_fused(const CallCtx& c) {
  return !c.decode && !c.dk && !c.m->mx && c.m->fused_update && c.m->ngpt_bnc > 0;
}

cudaError_t attention_sublayer(CallCtx& c, int b, int loop, float* h, __nv_bfloat16* hb,
                               bool commit_after) {
  dory_model* m = c.m;
  const BlockW& W = m->blocks[b];
  CUtensorMap tmA;
  GemmParams g;
  DORY_TRY(projection_input(c, &tmA, g, hb, h, m->d, false));
  if (m->mx) mx_weights(g, W.qsf, m->n_qkvg, W.g_qkvg);
  const float2* rope = W.full ? c.w.rope_full : c.w.rope_swa;
  if (c.decode) {
    // few rows: spread the weight stream over the SMs with K splits, then a
    // row kernel applies RoPE / QK-norm / gates to the summed partials
    g.M = c.n; g.N = m->n_qkvg; g.K = m->d;
    g.epi = kEpiStoreF32;
    g.k_splits = pick_k_splits(m, c.n, m->n_qkvg, 128, m->d);
    // rows of the partial products start on 128-byte boundaries whatever the
    // number of gate columns (vector and bulk stores need 16-byte alignment)
    g.out_f32 = c.w.part; g.ld_out = m->ld_qkvg; g.split_stride = size_t(c.n) * m->ld_qkvg;
    g.status = m->status;
    {
      Launch L(m, c.s, DORY_KK_QKVG);
      DORY_TRY(launch_gemm(tmA, m->mx ? W.tm8_qkvg : W.tm_qkvg[0], g, 128, m->hd, m->num_sms, c.s));
    }
    QkvgPostParams pp;
    pp.part = c.w.part; pp.splits = g.k_splits; pp.split_stride = g.split_stride; pp.ld = m->ld_qkvg;
    pp.rows = c.n; pp.n_q_heads = m->hq; pp.n_kv_heads = m->hkv; pp.hd = m->hd;
    pp.s_qk = W.s_qk; pp.rope = rope; pp.norm_eps = m->cfg.norm_eps;
    pp.q_out = c.w.q; pp.k_out = c.w.kf; pp.v_out = c.w.vf; pp.gate_out = c.w.gate;
    // this step's keys and values go to the cache here (no separate commit)
    pp.commit = 1;
    pp.kv = kv_view(c.kv, b, loop);
    pp.d_seq = c.dseq; pp.d_pos = c.dpos;
    pp.row_k = W.recurrent ? c.dk : nullptr; pp.loop = loop;
    pp.status = m->status;
    {
      Launch L(m, c.s, DORY_KK_QKVG);
      DORY_TRY(launch_qkvg_post(pp, c.s));
    }
  } else {
    g.M = c.n; g.N = m->n_qkvg; g.K = m->d;
    g.epi = kEpiQKVG;
    g.q_out = c.w.q; g.k_out = c.w.kf; g.v_out = c.w.vf; g.gate_out = c.w.gate;
    g.n_q_heads = m->hq; g.n_kv_heads = m->hkv;
    g.s_qk = W.s_qk;
    g.rope = rope;
    g.norm_eps = m->cfg.norm_eps;
    g.status = m->status;
    Launch L(m, c.s, DORY_KK_QKVG);
    // block-scaled: 128-column tiles keep two accumulators, so the QKVG
    // epilogue overlaps the next tile's MMAs
    if (m->mx)
      DORY_TRY(launch_gemm(tmA, W.tm8_qkvg, g, 128, m->hd, m->num_sms, c.s));
    else
      DORY_TRY(launch_gemm(tmA, W.tm_qkvg[1], g, 256, m->hd, m->num_sms, c.s));
  }

  const KvLayerView view = kv_view(c.kv, b, loop);
  const int window = W.full ? 0 : m->cfg.window;
  const float scale_log2 = m->cfg.softmax_scale * 1.4426950408889634f;
  int32_t* probe = (m->probe && b == m->probe_layer) ? m->probe : nullptr;
  if (probe) {
    if (c.n > m->probe_rows) return cudaErrorInvalidValue;
    Launch L(m, c.s, DORY_KK_ATTN);
    DORY_TRY(launch_probe_init(probe, size_t(c.n) * m->hq, c.s));
  }
  if (c.decode) {
    DecodeAttnParams a;
    a.q = c.w.q; a.gate = c.w.gate; a.out = c.w.o; a.kv = view;
    a.d_seq = c.dseq; a.d_pos = c.dpos;
    a.batch = c.n; a.n_q_heads = m->hq; a.window = window; a.max_pos = c.max_pos;
    const int max_keys = window > 0 ? std::min(c.max_pos + 1, window) : c.max_pos + 1;
    int sk = (max_keys + kMaxDecodeSplits - 1) / kMaxDecodeSplits;
    sk = std::max(512, (sk + 63) / 64 * 64);
    a.split_keys = sk;
    a.scale_log2 = scale_log2;
    a.part_acc = c.w.dacc; a.part_ml = c.w.dml;
    a.status = m->status;
    a.probe = probe;
    {
      Launch L(m, c.s, DORY_KK_ATTN);
      ++m->cur_launches;   // split-KV kernel + combine kernel
      if (decode_attention_tma_supported(m->hd, window, m->hq / m->hkv) && 2.f * W.m_log2 < 120.f) {
        ++m->cur_paths[kPathDecodeTma];
        DORY_TRY(launch_decode_attention_tma(a, W.m_log2, c.s));
      } else {
        ++m->cur_paths[kPathDecodeCp];
        DORY_TRY(launch_decode_attention(a, c.s));
      }
    }
  } else {
    if (prefill_attention_tc_supported(m->hd, c.pos0, window, W.m_log2)) {
      PrefillAttnTcParams a;
      a.gate = c.w.gate; a.out = c.w.o; a.n = c.n; a.pos0 = c.pos0; a.seq = c.seq;
      a.n_q_heads = m->hq; a.n_kv = m->hkv; a.cap = view.cap; a.window = window;
      a.last_pos = c.pos0 + c.n - 1; a.scale_log2 = scale_log2; a.m_log2 = W.m_log2;
      a.status = m->status;
      a.probe = probe;
      ++m->cur_paths[kPathPrefillTc];
      Launch L(m, c.s, DORY_KK_ATTN);
      DORY_TRY(launch_prefill_attention_tc(a, c.w.q, c.w.kf, c.w.vf, view, c.s));
    } else {
      PrefillAttnParams a;
      a.q = c.w.q; a.k_new = c.w.kf; a.v_new = c.w.vf; a.gate = c.w.gate; a.out = c.w.o;
      a.kv = view; a.seq = c.seq; a.pos0 = c.pos0; a.n = c.n; a.n_q_heads = m->hq;
      a.window = window; a.scale_log2 = scale_log2; a.status = m->status;
      a.probe = probe;
      ++m->cur_paths[kPathPrefillMma];
      Launch L(m, c.s, DORY_KK_ATTN);
      DORY_TRY(launch_prefill_attention(a, c.s));
    }
    if (commit_after) {
      const int first = W.full ? 0 : std::max(0, c.n - view.cap);
      Launch L(m, c.s, DORY_KK_KVCOMMIT);
      DORY_TRY(launch_kv_commit(view, c.w.kf, c.w.vf, c.n, first, c.seq, c.pos0, nullptr, nullptr,
                                m->status, c.s));
    }
  }

  // output projection, then the nGPT update of the stream
  CUtensorMap tmO;
  GemmParams go;
  DORY_TRY(projection_input(c, &tmO, go, c.w.o, nullptr, m->d_attn, true));
  if (m->mx) mx_weights(go, W.osf, m->d, W.g_o);
  if (use_fused(c)) {
    NgptGemmParams f;
    f.M = c.n; f.N = m->d; f.K = m->d_attn; f.cluster = m->ngpt_cluster;
    f.h = h; f.hb = hb; f.alpha = W.alpha_attn; f.norm_eps = m->cfg.norm_eps;
    f.status = m->status;
    {
      Launch L(m, c.s, DORY_KK_OPROJ);
      DORY_TRY(launch_gemm_ngpt(tmO, W.tm_o_n, f, c.s));
    }
    ++c.m->cur_sublayers;
    return cudaSuccess;
  }
  const int bn_o = c.decode ? 128 : 256;
  go.M = c.n; go.N = m->d; go.K = m->d_attn;
  go.epi = kEpiStoreF32;
  go.k_splits = c.decode ? pick_k_splits(m, c.n, m->d, bn_o, m->d_attn) : 1;
  go.out_f32 = c.w.y; go.ld_out = m->d; go.split_stride = size_t(c.n) * m->d;
  go.status = m->status;
  streamk_tail(c, go);
  {
    Launch L(m, c.s, DORY_KK_OPROJ);
    const CUtensorMap& tb = m->mx ? (bn_o == 256 ? W.tm8_o_256 : W.tm8_o) : W.tm_o[bn_o == 256];
    DORY_TRY(launch_gemm(tmO, tb, go, bn_o, m->hd, m->num_sms, c.s));
  }

  RowUpdateParams r;
  r.rows = c.n; r.d = m->d; r.y = c.w.y; r.splits = go.k_splits; r.split_stride = go.split_stride;
  r.h = h; r.hb = hb; r.alpha = W.alpha_attn; r.norm_eps = m->cfg.norm_eps;
  r.row_k = W.recurrent ? c.dk : nullptr; r.loop = loop; r.k_hi = c.k; r.status = m->status;
  fuse_stream_quant(c, r);
  {
    Launch L(m, c.s, DORY_KK_ROW);
    DORY_TRY(launch_row_update(r, c.s));
  }
  c.h_quantized = r.q_fmt != 0;
  ++c.m->cur_sublayers;
  return cudaSuccess;
}

// `reinject`: after the update, x <- Norm(x + e); `save_e`: store the update
// result as e first; `out`: also write the result as bf16 there.
cudaError_t mlp_sublayer(CallCtx& c, int b, float* h, __nv_bfloat16* hb, bool save_e,
                         bool reinject, __nv_bfloat16* out, int loop = 1) {
  dory_model* m = c.m;
  const BlockW& W = m->blocks[b];
  CUtensorMap tmA;
  GemmParams g;
  DORY_TRY(projection_input(c, &tmA, g, hb, h, m->d, false));
  if (m->mx) mx_weights(g, W.gusf, 2 * m->ff, W.g_gu);
  // gate and up rows alternate in groups of half a GEMM tile: 128 (bf16,
  // 256-column tiles), 64 (block-scaled, 128-column tiles with two
  // accumulators, so the SwiGLU epilogue overlaps the next tile's MMAs)
  const int gu_group = m->mx ? 64 : 128;
  if (c.decode) {
    g.M = c.n; g.N = 2 * m->ff; g.K = m->d;
    g.epi = kEpiStoreF32;
    g.k_splits = pick_k_splits(m, c.n, 2 * m->ff, 128, m->d);
    g.out_f32 = c.w.part; g.ld_out = 2 * m->ff; g.split_stride = size_t(c.n) * 2 * m->ff;
    g.status = m->status;
    {
      Launch L(m, c.s, DORY_KK_GATEUP);
      DORY_TRY(launch_gemm(tmA, m->mx ? W.tm8_gu : W.tm_gu[0], g, 128, m->hd, m->num_sms, c.s));
    }
    Launch L(m, c.s, DORY_KK_GATEUP);
    DORY_TRY(launch_swiglu_post(c.w.part, g.k_splits, g.split_stride, c.n, m->ff,
                                m->cfg.gate_scale, gu_group, c.w.a, c.s));
  } else {
    g.M = c.n; g.N = 2 * m->ff; g.K = m->d;
    g.epi = kEpiSwiGLU;
    g.out_act = c.w.a; g.ld_act = m->ff; g.gate_scale = m->cfg.gate_scale;
    g.status = m->status;
    Launch L(m, c.s, DORY_KK_GATEUP);
    if (m->mx)
      DORY_TRY(launch_gemm(tmA, W.tm8_gu, g, 128, m->hd, m->num_sms, c.s));
    else
      DORY_TRY(launch_gemm(tmA, W.tm_gu[1], g, 256, m->hd, m->num_sms, c.s));
  }

  CUtensorMap tmAct;
  GemmParams gd;
  DORY_TRY(projection_input(c, &tmAct, gd, c.w.a, nullptr, m->ff, true));
  if (m->mx) mx_weights(gd, W.dsf, m->d, W.g_d);
  if (use_fused(c)) {
    NgptGemmParams f;
    f.M = c.n; f.N = m->d; f.K = m->ff; f.cluster = m->ngpt_cluster;
    f.h = h; f.hb = hb; f.alpha = W.alpha_mlp; f.norm_eps = m->cfg.norm_eps;
    f.e_save = save_e ? c.w.e32 : nullptr;
    f.e = reinject ? c.w.e32 : nullptr;
    f.out = out;
    f.status = m->status;
    {
      Launch L(m, c.s, DORY_KK_DOWN);
      DORY_TRY(launch_gemm_ngpt(tmAct, W.tm_d_n, f, c.s));
    }
    ++c.m->cur_sublayers;
    return cudaSuccess;
  }
  const int bn_d = c.decode ? 128 : 256;
  gd.M = c.n; gd.N = m->d; gd.K = m->ff;
  gd.epi = kEpiStoreF32;
  gd.k_splits = c.decode ? pick_k_splits(m, c.n, m->d, bn_d, m->ff) : 1;
  gd.out_f32 = c.w.y; gd.ld_out = m->d; gd.split_stride = size_t(c.n) * m->d;
  gd.status = m->status;
  // the activations (rows x d_ff) outweigh W_down (d x d_ff) once rows > d:
  // N tiles fastest, and W_down's loads marked evict-last in L2 (every wave
  // reads all of it again; the hint trims the re-reads a little)
  gd.raster_n = c.n > m->d ? 1 : 0;
  gd.l2_hint = gd.raster_n;
  streamk_tail(c, gd);
  {
    Launch L(m, c.s, DORY_KK_DOWN);
    const CUtensorMap& tb = m->mx ? (bn_d == 256 ? W.tm8_d_256 : W.tm8_d) : W.tm_d[bn_d == 256];
    DORY_TRY(launch_gemm(tmAct, tb, gd, bn_d, m->hd, m->num_sms, c.s));
  }

  RowUpdateParams r;
  r.rows = c.n; r.d = m->d; r.y = c.w.y; r.splits = gd.k_splits; r.split_stride = gd.split_stride;
  r.h = h; r.hb = hb; r.alpha = W.alpha_mlp; r.norm_eps = m->cfg.norm_eps;
  r.e_save = save_e ? c.w.e32 : nullptr;
  r.e = reinject ? c.w.e32 : nullptr;
  r.out = out;
  r.row_k = W.recurrent ? c.dk : nullptr; r.loop = loop; r.k_hi = c.k; r.status = m->status;
  fuse_stream_quant(c, r);
  {
    Launch L(m, c.s, DORY_KK_ROW);
    DORY_TRY(launch_row_update(r, c.s));
  }
  c.h_quantized = r.q_fmt != 0;
  ++c.m->cur_sublayers;
  return cudaSuccess;
}

// (cos, sin) tables of this call's positions for both RoPE bases
cudaError_t enqueue_rope_tables(CallCtx& c) {
  dory_model* m = c.m;
  const int pos0 = c.decode ? 0 : c.pos0;
  const int32_t* dpos = c.decode ? c.dpos : nullptr;
  {
    Launch L(m, c.s, DORY_KK_ROW);
    DORY_TRY(launch_rope_table(m->inv_freq_swa, m->hd, c.n, pos0, dpos, c.w.rope_swa, c.s));
  }
  Launch L(m, c.s, DORY_KK_ROW);
  DORY_TRY(launch_rope_table(m->inv_freq_full, m->hd, c.n, pos0, dpos, c.w.rope_full, c.s));
  return cudaSuccess;
}

// The whole stack for one call, enqueued on c.s.
cudaError_t enqueue_stack(CallCtx& c, const __nv_bfloat16* src, __nv_bfloat16* dst) {
  dory_model* m = c.m;
  const dory_config* cfg = &m->cfg;
  const int n_in = cfg->n_in_blocks, n_rec = cfg->n_rec_blocks, nb = m->nb;
  {
    Launch L(m, c.s, DORY_KK_ROW);
    DORY_TRY(launch_load_rows(src, c.w.h32, c.w.hb, c.n, m->d, c.s));
  }
  DORY_TRY(enqueue_rope_tables(c));
  const bool last_loop = c.kv->mode == DORY_KV_LAST_LOOP;
  for (int b = 0; b < n_in; ++b) {
    DORY_TRY(attention_sublayer(c, b, 1, c.w.h32, c.w.hb, true));
    const bool last = b == n_in - 1;
    // the input block's output e is saved and re-injected before loop 1
    DORY_TRY(mlp_sublayer(c, b, c.w.h32, c.w.hb, last, last, nullptr));
  }
  for (int j = 1; j <= c.k; ++j) {
    for (int b = n_in; b < n_in + n_rec; ++b) {
      // last-loop caching: this call's keys reach the cache after the final loop only
      const bool commit = !last_loop || j == c.k;
      DORY_TRY(attention_sublayer(c, b, j, c.w.h32, c.w.hb, commit));
      const bool reinject = (b == n_in + n_rec - 1) && j < c.k;
      // with per-row loop counts the row kernels refine both decisions per row
      DORY_TRY(mlp_sublayer(c, b, c.w.h32, c.w.hb, false, reinject, nullptr, j));
    }
  }
  for (int b = n_in + n_rec; b < nb; ++b) {
    DORY_TRY(attention_sublayer(c, b, 1, c.w.h32, c.w.hb, true));
    DORY_TRY(mlp_sublayer(c, b, c.w.h32, c.w.hb, false, false, b == nb - 1 ? dst : nullptr));
  }
  return cudaSuccess;
}

// Capture (or reuse) the graph for this call and launch it on `stream`.
int run_graph(dory_model* m, const GraphKey& key, CallCtx& c, const __nv_bfloat16* src,
              __nv_bfloat16* dst, cudaStream_t stream) {
  auto it = m->graphs.find(key);
  if (it == m->graphs.end()) {
    if (m->graphs.size() >= 16) {   // evict the least recently used graph
      auto lru = m->graphs.begin();
      for (auto g = m->graphs.begin(); g != m->graphs.end(); ++g)
        if (g->second.last_use < lru->second.last_use) lru = g;
      if (m->last_marks == &lru->second.marks) m->last_marks = nullptr;
      destroy_entry(lru->second);
      m->graphs.erase(lru);
    }
    m->cur_launches = 0;
    m->cur_sublayers = 0;
    for (int i = 0; i < kPaths; ++i) m->cur_paths[i] = 0;
    GraphEntry ent;
    m->cur_marks = key.prof ? &ent.marks : nullptr;
    c.s = m->cap_stream;
    if (cudaStreamBeginCapture(m->cap_stream, cudaStreamCaptureModeThreadLocal) != cudaSuccess)
      return DORY_ERR_CUDA;
    cudaError_t e = enqueue_stack(c, src, dst);
    m->cur_marks = nullptr;
    cudaGraph_t graph = nullptr;
    cudaError_t e2 = cudaStreamEndCapture(m->cap_stream, &graph);
    if (e != cudaSuccess || e2 != cudaSuccess || !graph) {
      if (graph) cudaGraphDestroy(graph);
      destroy_entry(ent);
      cudaGetLastError();
      return DORY_ERR_CUDA;
    }
    e = cudaGraphInstantiate(&ent.exec, graph, 0);
    cudaGraphDestroy(graph);
    if (e != cudaSuccess) {
      destroy_entry(ent);
      return DORY_ERR_CUDA;
    }
    ent.launches = m->cur_launches;
    ent.sublayers = m->cur_sublayers;
    for (int i = 0; i < kPaths; ++i) ent.paths[i] = m->cur_paths[i];
    it = m->graphs.emplace(key, ent).first;
  }
  it->second.last_use = ++m->tick;
  if (cudaGraphLaunch(it->second.exec, stream) != cudaSuccess) return DORY_ERR_CUDA;
  m->last_launches = it->second.launches;
  m->last_sublayers = it->second.sublayers;
  for (int i = 0; i < kPaths; ++i) m->last_paths[i] = it->second.paths[i];
  if (key.prof) m->last_marks = &it->second.marks;
  return DORY_OK;
}

int check_k(const dory_model* m, const dory_kv* kv, int k) {
  const int kmax = m->cfg.allow_extrapolated_k ? 8 : 4;
  if (k < 1 || k > kmax) return DORY_ERR_K_RANGE;
  if (kv->mode == DORY_KV_PER_LOOP && k > kv->k_max) return DORY_ERR_K_EXCEEDS_KMAX;
  return DORY_OK;
}

void fill_inv_freq(std::vector<double>& v, double base, int hd) {
  v.resize(hd / 2);
  for (int i = 0; i < hd / 2; ++i) v[i] = pow(base, -2.0 * i / hd);
}

}  // namespace

// ======================================================================== ABI
extern "C" {

const char* dory_error_string(int status) {
  switch (status) {
    case DORY_OK: return "ok";
    case DORY_ERR_INVALID_ARG: return "invalid argument";
    case DORY_ERR_BAD_CONFIG: return "unsupported model configuration";
    case DORY_ERR_K_RANGE: return "loop count k out of range";
    case DORY_ERR_K_EXCEEDS_KMAX: return "k exceeds the per-loop cache's k_max";
    case DORY_ERR_CTX_OVERFLOW: return "positions exceed the cache's max_ctx";
    case DORY_ERR_BUFFER_TOO_SMALL: return "buffer too small";
    case DORY_ERR_MISALIGNED: return "device buffer not 256-byte aligned";
    case DORY_ERR_CUDA: return "CUDA call failed";
    case DORY_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait expired";
    case DORY_ERR_UNSUPPORTED_ARCH: return "device is not sm_100 (B200)";
    case DORY_ERR_DEVICE_BOUNDS: return "a kernel's bounds check fired";
    case DORY_ERR_SCRATCH_LIMIT: return "too many rows for the built-in scratch array";
    default: return "unknown status";
  }
}

size_t dory_weight_bytes(const dory_config* cfg) {
  if (validate_config(cfg) != DORY_OK) return 0;
  return weight_layout(cfg).total;
}

int dory_create(const dory_config* cfg, void* weight_buf, size_t weight_bytes,
                const dory_block_src* src, int n_src, void* stream, dory_model** out) {
  if (!out || !weight_buf || !src) return DORY_ERR_INVALID_ARG;
  *out = nullptr;
  int st = validate_config(cfg);
  if (st != DORY_OK) return st;
  if (n_src != n_blocks(cfg)) return DORY_ERR_INVALID_ARG;
  const WeightLayout L = weight_layout(cfg);
  if (weight_bytes < L.total) return DORY_ERR_BUFFER_TOO_SMALL;
  if (!is_aligned(weight_buf)) return DORY_ERR_MISALIGNED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DORY_ERR_CUDA;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return DORY_ERR_CUDA;
  if (prop.major != 10 || prop.minor != 0) return DORY_ERR_UNSUPPORTED_ARCH;
  for (int b = 0; b < n_src; ++b) {
    const dory_block_src& s = src[b];
    if (!s.wq || !s.wk || !s.wv || !s.wg || !s.wo || !s.w_gate || !s.w_up || !s.w_down ||
        !s.alpha_attn || !s.alpha_mlp || !s.s_qk)
      return DORY_ERR_INVALID_ARG;
    // MXFP8 / NVFP4 weights are quantised by kernels that read the bf16 matrices
    if (cfg->weight_format != DORY_WEIGHTS_BF16) {
      const void* mats[8] = {s.wq, s.wk, s.wv, s.wg, s.wo, s.w_gate, s.w_up, s.w_down};
      for (const void* p : mats)
        if (!is_device_ptr(p) || !is_aligned(p, 16)) return DORY_ERR_INVALID_ARG;
    }
  }

  std::unique_ptr<dory_model> m(new (std::nothrow) dory_model());
  if (!m) return DORY_ERR_INVALID_ARG;
  m->cfg = *cfg;
  m->d = cfg->d_model; m->hq = cfg->n_q_heads; m->hkv = cfg->n_kv_heads; m->hd = cfg->head_dim;
  m->ff = cfg->d_ff; m->d_attn = m->hq * m->hd;
  m->n_qkvg = m->d_attn + 2 * m->hkv * m->hd + m->hq;
  m->ld_qkvg = (m->n_qkvg + 31) / 32 * 32;
  m->mx = cfg->weight_format == DORY_WEIGHTS_MXFP8   ? kOperandsMxfp8
          : cfg->weight_format == DORY_WEIGHTS_NVFP4 ? kOperandsNvfp4
                                                     : kOperandsBf16;
  m->ngpt_bnc = ngpt_gemm_cols_per_cta(m->d);
  m->ngpt_cluster = m->ngpt_bnc ? m->d / m->ngpt_bnc : 0;
  m->nb = n_blocks(cfg);
  m->device = dev;
  m->num_sms = prop.multiProcessorCount;
  m->wbuf = static_cast<uint8_t*>(weight_buf);
  m->wbytes = weight_bytes;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  uint8_t* hdr = m->wbuf;
  m->status = reinterpret_cast<uint32_t*>(hdr);
  m->inv_freq_swa = reinterpret_cast<double*>(hdr + align_up(64));
  m->inv_freq_full = reinterpret_cast<double*>(hdr + align_up(64) + align_up(m->hd / 2 * sizeof(double)));
  static thread_local std::vector<double> fs, ff;
  fill_inv_freq(fs, cfg->rope_base_swa, m->hd);
  fill_inv_freq(ff, cfg->rope_base_full, m->hd);
  if (m->num_sms <= kSkMaxGrid) {
    const size_t slots = static_cast<size_t>(kSkMaxGrid) * 128 * 256 * 4;
    m->sk_ws = reinterpret_cast<float*>(hdr + L.sk);
    m->sk_sync = reinterpret_cast<uint32_t*>(hdr + L.sk + (slots + 255) / 256 * 256);
    if (cudaMemsetAsync(m->sk_sync, 0, (3 + 4 * kSkMaxGrid) * sizeof(uint32_t), s) != cudaSuccess)
      return DORY_ERR_CUDA;
  }
  if (cudaMemsetAsync(m->status, 0, 64, s) != cudaSuccess ||
      cudaMemcpyAsync(m->inv_freq_swa, fs.data(), fs.size() * sizeof(double), cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(m->inv_freq_full, ff.data(), ff.size() * sizeof(double), cudaMemcpyHostToDevice, s) != cudaSuccess)
    return DORY_ERR_CUDA;

  const size_t d = m->d, hd = m->hd, da = m->d_attn, F = m->ff;
  m->blocks.resize(m->nb);
  for (int b = 0; b < m->nb; ++b) {
    BlockW& W = m->blocks[b];
    uint8_t* base = m->wbuf + L.header + L.per_block * b;
    W.wqkvg = reinterpret_cast<__nv_bfloat16*>(base + L.off_qkvg);
    W.wo = reinterpret_cast<__nv_bfloat16*>(base + L.off_o);
    W.wgu = reinterpret_cast<__nv_bfloat16*>(base + L.off_gu);
    W.wd = reinterpret_cast<__nv_bfloat16*>(base + L.off_d);
    W.alpha_attn = reinterpret_cast<float*>(base + L.off_aa);
    W.alpha_mlp = reinterpret_cast<float*>(base + L.off_am);
    W.s_qk = reinterpret_cast<float*>(base + L.off_sqk);
    W.full = is_full(cfg, b);
    W.recurrent = is_recurrent(cfg, b);
    const dory_block_src& S = src[b];
    const size_t kvr = size_t(m->hkv) * hd;
    cudaError_t e = cudaSuccess;
    bool ok = true;
    if (m->mx) {
      // MXFP8 weights quantised on the device from the bf16 sources (rows
      // quantised independently along K: the q | k | v | gate rows of the
      // fused projection keep their own scales; gate / up rows interleaved in
      // groups of 64, half a 128-column tile)
      W.q8 = base + L.off_q8;   W.qsf = base + L.off_qsf;
      W.o8 = base + L.off_o8;   W.osf = base + L.off_osf;
      W.gu8 = base + L.off_gu8; W.gusf = base + L.off_gusf;
      W.d8 = base + L.off_d8;   W.dsf = base + L.off_dsf;
      const __nv_bfloat16* qs[4] = {reinterpret_cast<const __nv_bfloat16*>(S.wq),
                                    reinterpret_cast<const __nv_bfloat16*>(S.wk),
                                    reinterpret_cast<const __nv_bfloat16*>(S.wv),
                                    reinterpret_cast<const __nv_bfloat16*>(S.wg)};
      const int qrows[4] = {0, int(da), int(da + kvr), int(da + 2 * kvr)};
      const __nv_bfloat16* os[1] = {reinterpret_cast<const __nv_bfloat16*>(S.wo)};
      const __nv_bfloat16* gs[2] = {reinterpret_cast<const __nv_bfloat16*>(S.w_gate),
                                    reinterpret_cast<const __nv_bfloat16*>(S.w_up)};
      const __nv_bfloat16* ds[1] = {reinterpret_cast<const __nv_bfloat16*>(S.w_down)};
      const float eps = cfg->norm_eps;
      if (m->mx == kOperandsNvfp4) {
        // one tensor scale per GEMM's weights: q | k | v | gate together,
        // gate and up together (g = amax / (6 * 448) over the group)
        W.tscale = reinterpret_cast<float*>(base + L.off_ts);
        uint32_t* amax = reinterpret_cast<uint32_t*>(W.tscale + 4);
        const size_t qcounts[4] = {da * d, kvr * d, kvr * d, size_t(m->hq) * d};
        const size_t ocount[1] = {d * da}, gcounts[2] = {F * d, F * d}, dcount[1] = {d * F};
        e = e ? e : launch_nvfp4_tensor_scale(qs, qcounts, 4, amax, W.tscale + 0, s);
        e = e ? e : launch_nvfp4_tensor_scale(os, ocount, 1, amax, W.tscale + 1, s);
        e = e ? e : launch_nvfp4_tensor_scale(gs, gcounts, 2, amax, W.tscale + 2, s);
        e = e ? e : launch_nvfp4_tensor_scale(ds, dcount, 1, amax, W.tscale + 3, s);
        e = e ? e : launch_quant_nvfp4_bf16(qs, qrows, 4, 0, m->n_qkvg, 256, int(d), 0, eps,
                                            W.tscale + 0, 0.f, W.q8, W.qsf, s);
        e = e ? e : launch_quant_nvfp4_bf16(os, nullptr, 1, 0, int(d), 256, int(da), 0, eps,
                                            W.tscale + 1, 0.f, W.o8, W.osf, s);
        e = e ? e : launch_quant_nvfp4_bf16(gs, nullptr, 2, 64, int(2 * F), 256, int(d), 0, eps,
                                            W.tscale + 2, 0.f, W.gu8, W.gusf, s);
        e = e ? e : launch_quant_nvfp4_bf16(ds, nullptr, 1, 0, int(d), 256, int(F), 0, eps,
                                            W.tscale + 3, 0.f, W.d8, W.dsf, s);
      } else {
        e = e ? e : launch_quant_mxfp8_bf16(qs, qrows, 4, 0, m->n_qkvg, 256, int(d), 0, eps, W.q8,
                                            W.qsf, s);
        e = e ? e : launch_quant_mxfp8_bf16(os, nullptr, 1, 0, int(d), 256, int(da), 0, eps, W.o8,
                                            W.osf, s);
        e = e ? e : launch_quant_mxfp8_bf16(gs, nullptr, 2, 64, int(2 * F), 256, int(d), 0, eps,
                                            W.gu8, W.gusf, s);
        e = e ? e : launch_quant_mxfp8_bf16(ds, nullptr, 1, 0, int(d), 256, int(F), 0, eps, W.d8,
                                            W.dsf, s);
      }
      // tensor maps over the code bytes (NVFP4: K / 2 per row)
      const size_t kd = m->mx == kOperandsNvfp4 ? d / 2 : d;
      const size_t kda = m->mx == kOperandsNvfp4 ? da / 2 : da;
      const size_t kF = m->mx == kOperandsNvfp4 ? F / 2 : F;
      ok &= make_tmap_u8(&W.tm8_qkvg, W.q8, m->n_qkvg, kd, 128);
      ok &= make_tmap_u8(&W.tm8_o, W.o8, d, kda, 128);
      ok &= make_tmap_u8(&W.tm8_gu, W.gu8, 2 * F, kd, 128);
      ok &= make_tmap_u8(&W.tm8_d, W.d8, d, kF, 128);
      ok &= make_tmap_u8(&W.tm8_qkvg_256, W.q8, m->n_qkvg, kd, 256);
      ok &= make_tmap_u8(&W.tm8_o_256, W.o8, d, kda, 256);
      ok &= make_tmap_u8(&W.tm8_gu_256, W.gu8, 2 * F, kd, 256);
      ok &= make_tmap_u8(&W.tm8_d_256, W.d8, d, kF, 256);
    } else {
      uint8_t* q = reinterpret_cast<uint8_t*>(W.wqkvg);
      e = e ? e : cudaMemcpyAsync(q, S.wq, da * d * 2, cudaMemcpyDefault, s);
      e = e ? e : cudaMemcpyAsync(q + da * d * 2, S.wk, kvr * d * 2, cudaMemcpyDefault, s);
      e = e ? e : cudaMemcpyAsync(q + (da + kvr) * d * 2, S.wv, kvr * d * 2, cudaMemcpyDefault, s);
      e = e ? e : cudaMemcpyAsync(q + (da + 2 * kvr) * d * 2, S.wg, size_t(m->hq) * d * 2, cudaMemcpyDefault, s);
      e = e ? e : cudaMemcpyAsync(W.wo, S.wo, d * da * 2, cudaMemcpyDefault, s);
      // gate/up interleaved in groups of 128 rows (the SwiGLU epilogue's tile halves)
      for (size_t t = 0; t < F / 128 && e == cudaSuccess; ++t) {
        uint8_t* g = reinterpret_cast<uint8_t*>(W.wgu) + (2 * t) * 128 * d * 2;
        e = cudaMemcpyAsync(g, reinterpret_cast<const uint8_t*>(S.w_gate) + t * 128 * d * 2,
                            128 * d * 2, cudaMemcpyDefault, s);
        e = e ? e : cudaMemcpyAsync(g + 128 * d * 2, reinterpret_cast<const uint8_t*>(S.w_up) + t * 128 * d * 2,
                                    128 * d * 2, cudaMemcpyDefault, s);
      }
      e = e ? e : cudaMemcpyAsync(W.wd, S.w_down, d * F * 2, cudaMemcpyDefault, s);
      for (int i = 0; i < 2; ++i) {
        const uint32_t box = i ? 256 : 128;
        ok &= make_tmap_bf16(&W.tm_qkvg[i], W.wqkvg, m->n_qkvg, d, box);
        ok &= make_tmap_bf16(&W.tm_o[i], W.wo, d, da, box);
        ok &= make_tmap_bf16(&W.tm_d[i], W.wd, d, F, box);
      }
      ok &= make_tmap_bf16(&W.tm_gu[0], W.wgu, 2 * F, d, 128);
      ok &= make_tmap_bf16(&W.tm_gu[1], W.wgu, 2 * F, d, 256);
      if (m->ngpt_bnc) {
        const uint32_t box = m->ngpt_bnc > 256 ? m->ngpt_bnc / 2 : m->ngpt_bnc;
        ok &= make_tmap_bf16(&W.tm_o_n, W.wo, d, da, box);
        ok &= make_tmap_bf16(&W.tm_d_n, W.wd, d, F, box);
      }
    }
    e = e ? e : cudaMemcpyAsync(W.alpha_attn, S.alpha_attn, d * 4, cudaMemcpyDefault, s);
    e = e ? e : cudaMemcpyAsync(W.alpha_mlp, S.alpha_mlp, d * 4, cudaMemcpyDefault, s);
    e = e ? e : cudaMemcpyAsync(W.s_qk, S.s_qk, hd * 4, cudaMemcpyDefault, s);
    if (e != cudaSuccess) return DORY_ERR_CUDA;
    if (!ok) return DORY_ERR_CUDA;
  }
  // static softmax maxima from the packed s_qk vectors, and the NVFP4 weight
  // tensor scales (one-time host read: the GEMM epilogues take them as
  // launch parameters)
  {
    std::vector<float> sq(size_t(m->nb) * hd), ts(size_t(m->nb) * 4, 1.f);
    for (int b = 0; b < m->nb; ++b) {
      if (cudaMemcpyAsync(sq.data() + size_t(b) * hd, m->blocks[b].s_qk, hd * 4,
                          cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return DORY_ERR_CUDA;
      if (m->blocks[b].tscale &&
          cudaMemcpyAsync(ts.data() + size_t(b) * 4, m->blocks[b].tscale, 4 * sizeof(float),
                          cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return DORY_ERR_CUDA;
    }
    if (cudaStreamSynchronize(s) != cudaSuccess) return DORY_ERR_CUDA;
    for (int b = 0; b < m->nb; ++b) {
      float mx = 0.f;
      for (size_t i = 0; i < hd; ++i) mx = std::max(mx, sq[size_t(b) * hd + i] * sq[size_t(b) * hd + i]);
      BlockW& W = m->blocks[b];
      W.m_log2 = cfg->softmax_scale * 1.4426950408889634f * mx;
      W.g_qkvg = ts[size_t(b) * 4 + 0];
      W.g_o = ts[size_t(b) * 4 + 1];
      W.g_gu = ts[size_t(b) * 4 + 2];
      W.g_d = ts[size_t(b) * 4 + 3];
    }
  }
  if (cudaStreamCreateWithFlags(&m->cap_stream, cudaStreamNonBlocking) != cudaSuccess)
    return DORY_ERR_CUDA;
  *out = m.release();
  return DORY_OK;
}

size_t dory_kv_bytes(const dory_config* cfg, int mode, int max_seqs, int max_ctx, int k_max) {
  if (validate_config(cfg) != DORY_OK || max_seqs <= 0 || max_ctx <= 0 || k_max < 1) return 0;
  if (mode != DORY_KV_PER_LOOP && mode != DORY_KV_LAST_LOOP) return 0;
  const size_t per_pos = 2 * size_t(cfg->n_kv_heads) * cfg->head_dim * 2;
  size_t total = 0;
  for (int b = 0; b < n_blocks(cfg); ++b) {
    const size_t loops = (mode == DORY_KV_PER_LOOP && is_recurrent(cfg, b)) ? k_max : 1;
    const size_t cap = is_full(cfg, b) ? size_t(max_ctx) : std::min<size_t>(cfg->window, max_ctx);
    total += loops * size_t(max_seqs) * cap * per_pos;
  }
  return total;
}

int dory_kv_alloc(dory_model* m, int mode, int max_seqs, int max_ctx, int k_max, void* kv_buf,
                  size_t kv_bytes, dory_kv** out) {
  if (!m || !kv_buf || !out || max_seqs <= 0 || max_ctx <= 0 || k_max < 1) return DORY_ERR_INVALID_ARG;
  *out = nullptr;
  if (mode != DORY_KV_PER_LOOP && mode != DORY_KV_LAST_LOOP) return DORY_ERR_INVALID_ARG;
  if (k_max > (m->cfg.allow_extrapolated_k ? 8 : 4)) return DORY_ERR_K_RANGE;
  if (!is_aligned(kv_buf)) return DORY_ERR_MISALIGNED;
  const size_t need = dory_kv_bytes(&m->cfg, mode, max_seqs, max_ctx, k_max);
  if (kv_bytes < need) return DORY_ERR_BUFFER_TOO_SMALL;
  std::unique_ptr<dory_kv> kv(new (std::nothrow) dory_kv());
  if (!kv) return DORY_ERR_INVALID_ARG;
  kv->m = m; kv->mode = mode; kv->max_seqs = max_seqs; kv->max_ctx = max_ctx; kv->k_max = k_max;
  kv->buf = static_cast<uint8_t*>(kv_buf); kv->bytes = kv_bytes;
  size_t off = 0;
  const size_t per_pos = 2 * size_t(m->hkv) * m->hd * 2;
  for (int b = 0; b < m->nb; ++b) {
    const int loops = (mode == DORY_KV_PER_LOOP && m->blocks[b].recurrent) ? k_max : 1;
    const int cap = m->blocks[b].full ? max_ctx : std::min(m->cfg.window, max_ctx);
    kv->base.push_back(off);
    kv->cap.push_back(cap);
    kv->loops.push_back(loops);
    off += size_t(loops) * max_seqs * cap * per_pos;
  }
  kv->seq_k.assign(max_seqs, 0);
  static std::atomic<uint64_t> next_uid{0};
  kv->uid = ++next_uid;
  m->caches.insert(kv.get());
  *out = kv.release();
  return DORY_OK;
}

int dory_kv_layout(const dory_kv* kv, int layer, int loop, int seq, int pos, int head,
                   size_t* k_off, size_t* v_off) {
  if (!kv || !k_off || !v_off) return DORY_ERR_INVALID_ARG;
  const dory_model* m = kv->m;
  if (layer < 0 || layer >= m->nb || seq < 0 || seq >= kv->max_seqs || head < 0 || head >= m->hkv)
    return DORY_ERR_INVALID_ARG;
  if (pos < 0 || pos >= kv->max_ctx) return DORY_ERR_CTX_OVERFLOW;
  if (kv->loops[layer] > 1 && (loop < 1 || loop > kv->loops[layer])) return DORY_ERR_INVALID_ARG;
  const KvLayerView v = kv_view(kv, layer, kv->loops[layer] > 1 ? loop : 1);
  const size_t elem = (size_t(seq) * v.seq_stride + (size_t(head) * v.cap + pos % v.cap) * v.hd);
  *k_off = reinterpret_cast<const uint8_t*>(v.k_base + elem) - kv->buf;
  *v_off = reinterpret_cast<const uint8_t*>(v.v_base + elem) - kv->buf;
  return DORY_OK;
}

size_t dory_workspace_bytes(const dory_model* m, int max_tokens) {
  if (!m || max_tokens <= 0) return 0;
  return ws_layout(m, max_tokens).total;
}

int dory_prefill(dory_model* m, dory_kv* kv, int seq, int pos0, int n_tokens, const void* h_in,
                 void* h_out, int k, void* ws, size_t ws_bytes, void* stream) {
  if (!m || !kv || kv->m != m || !h_in || !h_out || !ws || n_tokens <= 0 || pos0 < 0)
    return DORY_ERR_INVALID_ARG;
  if (seq < 0 || seq >= kv->max_seqs) return DORY_ERR_INVALID_ARG;
  int st = check_k(m, kv, k);
  if (st != DORY_OK) return st;
  if (size_t(pos0) + n_tokens > size_t(kv->max_ctx)) return DORY_ERR_CTX_OVERFLOW;
  if (!is_aligned(ws)) return DORY_ERR_MISALIGNED;
  if (ws_bytes < ws_layout(m, n_tokens).total) return DORY_ERR_BUFFER_TOO_SMALL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool in_dev = is_device_ptr(h_in), out_dev = is_device_ptr(h_out);
  if ((in_dev && !is_aligned(h_in, 16)) || (out_dev && !is_aligned(h_out, 16))) return DORY_ERR_MISALIGNED;
  CallCtx c;
  c.m = m; c.kv = kv; c.w = ws_bind(m, ws, n_tokens); c.n = n_tokens; c.decode = false;
  c.seq = seq; c.pos0 = pos0; c.dseq = nullptr; c.dpos = nullptr; c.max_pos = pos0 + n_tokens - 1;
  c.k = k; c.s = s;
  const size_t bytes = size_t(n_tokens) * m->d * 2;
  const __nv_bfloat16* src = in_dev ? static_cast<const __nv_bfloat16*>(h_in) : c.w.st_in;
  __nv_bfloat16* dst = out_dev ? static_cast<__nv_bfloat16*>(h_out) : c.w.st_out;
  if (!in_dev && cudaMemcpyAsync(c.w.st_in, h_in, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return DORY_ERR_CUDA;
  GraphKey key{0, k, n_tokens, seq, pos0, 0, m->profile ? 1 : 0, src, dst, ws, kv->uid, nullptr, nullptr,
               nullptr, m->probe, m->probe ? m->probe_layer : -1, graph_modes(m)};
  st = run_graph(m, key, c, src, dst, s);
  if (st != DORY_OK) return st;
  if (!out_dev && cudaMemcpyAsync(h_out, c.w.st_out, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return DORY_ERR_CUDA;
  kv->seq_k[seq] = k;
  return DORY_OK;
}

namespace {

// One decode step; d_k (device, per row) null means every row runs k loops,
// else row r runs d_k[r] loops (1..k) and k is the largest of them.
int decode_step_impl(dory_model* m, dory_kv* kv, int batch, const int32_t* d_seq,
                     const int32_t* d_pos, const int32_t* d_k, int max_pos_hint, const void* h_in,
                     void* h_out, int k, void* ws, size_t ws_bytes, void* stream) {
  if (!m || !kv || kv->m != m || !d_seq || !d_pos || !h_in || !h_out || !ws || batch <= 0)
    return DORY_ERR_INVALID_ARG;
  if (batch > kMaxDecodeRows) return DORY_ERR_INVALID_ARG;
  int st = check_k(m, kv, k);
  if (st != DORY_OK) return st;
  if (max_pos_hint < 0) return DORY_ERR_INVALID_ARG;
  if (max_pos_hint >= kv->max_ctx) return DORY_ERR_CTX_OVERFLOW;
  if (!is_aligned(ws)) return DORY_ERR_MISALIGNED;
  if (ws_bytes < ws_layout(m, batch).total) return DORY_ERR_BUFFER_TOO_SMALL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool in_dev = is_device_ptr(h_in), out_dev = is_device_ptr(h_out);
  CallCtx c;
  c.m = m; c.kv = kv; c.w = ws_bind(m, ws, batch); c.n = batch; c.decode = true;
  c.seq = 0; c.pos0 = 0; c.dseq = d_seq; c.dpos = d_pos; c.max_pos = max_pos_hint;
  c.k = k; c.dk = d_k; c.s = s;
  const size_t bytes = size_t(batch) * m->d * 2;
  const __nv_bfloat16* src = in_dev ? static_cast<const __nv_bfloat16*>(h_in) : c.w.st_in;
  __nv_bfloat16* dst = out_dev ? static_cast<__nv_bfloat16*>(h_out) : c.w.st_out;
  if (!in_dev && cudaMemcpyAsync(c.w.st_in, h_in, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return DORY_ERR_CUDA;
  GraphKey key{1, k, batch, 0, 0, max_pos_hint, m->profile ? 1 : 0, src, dst, ws, kv->uid, d_seq, d_pos,
               d_k, m->probe, m->probe ? m->probe_layer : -1, graph_modes(m)};
  st = run_graph(m, key, c, src, dst, s);
  if (st != DORY_OK) return st;
  if (!out_dev && cudaMemcpyAsync(h_out, c.w.st_out, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return DORY_ERR_CUDA;
  return DORY_OK;
}

}  // namespace

int dory_decode_step(dory_model* m, dory_kv* kv, int batch, const int32_t* d_seq,
                     const int32_t* d_pos, int max_pos_hint, const void* h_in, void* h_out, int k,
                     void* ws, size_t ws_bytes, void* stream) {
  return decode_step_impl(m, kv, batch, d_seq, d_pos, nullptr, max_pos_hint, h_in, h_out, k, ws,
                          ws_bytes, stream);
}

int dory_decode_step_mixed(dory_model* m, dory_kv* kv, int batch, const int32_t* d_seq,
                           const int32_t* d_pos, const int32_t* d_k, int k_hi, int max_pos_hint,
                           const void* h_in, void* h_out, void* ws, size_t ws_bytes,
                           void* stream) {
  if (!d_k || !is_device_ptr(d_k)) return DORY_ERR_INVALID_ARG;
  return decode_step_impl(m, kv, batch, d_seq, d_pos, d_k, max_pos_hint, h_in, h_out, k_hi, ws,
                          ws_bytes, stream);
}

int dory_device_status(dory_model* m, void* stream) {
  if (!m) return DORY_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, m->status, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return DORY_ERR_CUDA;
  if (word) {
    if (cudaMemsetAsync(m->status, 0, 4, s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
      return DORY_ERR_CUDA;
  }
  if (word & kStatusTimeout) return DORY_ERR_DEVICE_TIMEOUT;
  if (word & kStatusBounds) return DORY_ERR_DEVICE_BOUNDS;
  return DORY_OK;
}

int dory_last_call_stats(const dory_model* m, int* kernel_launches, int* sublayer_updates) {
  if (!m) return DORY_ERR_INVALID_ARG;
  if (kernel_launches) *kernel_launches = m->last_launches;
  if (sublayer_updates) *sublayer_updates = m->last_sublayers;
  return DORY_OK;
}

int dory_profile_enable(dory_model* m, int enable) {
  if (!m) return DORY_ERR_INVALID_ARG;
  m->profile = enable != 0;
  return DORY_OK;
}

int dory_profile_read(dory_model* m, int kind, float* total_ms, int* launches) {
  if (!m || !total_ms || kind < 0 || kind >= DORY_KK_COUNT) return DORY_ERR_INVALID_ARG;
  if (!m->last_marks) return DORY_ERR_INVALID_ARG;
  float tot = 0.f;
  int cnt = 0;
  for (const Mark& mk : *m->last_marks) {
    if (mk.kind != kind) continue;
    if (cudaEventSynchronize(mk.end) != cudaSuccess) return DORY_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, mk.start, mk.end) != cudaSuccess) return DORY_ERR_CUDA;
    tot += ms;
    ++cnt;
  }
  *total_ms = tot;
  if (launches) *launches = cnt;
  return DORY_OK;
}

void dory_kv_free(dory_kv* kv) {
  if (!kv) return;
  if (dory_model* m = kv->m) {
    // graphs captured for this cache bake its addresses: drop them
    for (auto it = m->graphs.begin(); it != m->graphs.end();) {
      if (it->first.kv == kv->uid) {
        if (m->last_marks == &it->second.marks) m->last_marks = nullptr;
        destroy_entry(it->second);
        it = m->graphs.erase(it);
      } else {
        ++it;
      }
    }
    m->caches.erase(kv);
  }
  delete kv;
}

void dory_destroy(dory_model* m) {
  if (!m) return;
  for (auto& g : m->graphs) destroy_entry(g.second);
  for (dory_kv* kv : m->caches) kv->m = nullptr;   // caches outliving the model stay freeable
  if (m->cap_stream) cudaStreamDestroy(m->cap_stream);
  for (cudaStream_t x : m->aux_streams) cudaStreamDestroy(x);
  for (cudaEvent_t x : m->aux_events) cudaEventDestroy(x);
  if (m->fork_event) cudaEventDestroy(m->fork_event);
  delete m;
}

int dory_attention_sublayer(dory_model* m, dory_kv* kv, int layer, int loop, int seq, int pos0,
                            int n_rows, float* h, void* ws, size_t ws_bytes, void* stream) {
  if (!m || !kv || kv->m != m || !h || !ws || n_rows <= 0 || pos0 < 0) return DORY_ERR_INVALID_ARG;
  if (layer < 0 || layer >= m->nb || seq < 0 || seq >= kv->max_seqs) return DORY_ERR_INVALID_ARG;
  if (kv->loops[layer] > 1 && (loop < 1 || loop > kv->loops[layer])) return DORY_ERR_INVALID_ARG;
  if (size_t(pos0) + n_rows > size_t(kv->max_ctx)) return DORY_ERR_CTX_OVERFLOW;
  if (!is_aligned(ws) || !is_aligned(h, 16)) return DORY_ERR_MISALIGNED;
  if (ws_bytes < ws_layout(m, n_rows).total) return DORY_ERR_BUFFER_TOO_SMALL;
  CallCtx c;
  c.m = m; c.kv = kv; c.w = ws_bind(m, ws, n_rows); c.n = n_rows; c.decode = false;
  c.seq = seq; c.pos0 = pos0; c.dseq = nullptr; c.dpos = nullptr; c.max_pos = pos0 + n_rows - 1;
  c.k = 1; c.s = static_cast<cudaStream_t>(stream);
  m->cur_launches = m->cur_sublayers = 0;
  for (int i = 0; i < kPaths; ++i) m->cur_paths[i] = 0;
  if (launch_f32_to_bf16(h, c.w.hb, size_t(n_rows) * m->d, c.s) != cudaSuccess) return DORY_ERR_CUDA;
  if (enqueue_rope_tables(c) != cudaSuccess) return DORY_ERR_CUDA;
  if (attention_sublayer(c, layer, kv->loops[layer] > 1 ? loop : 1, h, c.w.hb, true) != cudaSuccess)
    return DORY_ERR_CUDA;
  for (int i = 0; i < kPaths; ++i) m->last_paths[i] = m->cur_paths[i];
  return DORY_OK;
}

int dory_mlp_sublayer(dory_model* m, int layer, int n_rows, float* h, void* ws, size_t ws_bytes,
                      void* stream) {
  if (!m || !h || !ws || n_rows <= 0 || layer < 0 || layer >= m->nb) return DORY_ERR_INVALID_ARG;
  if (!is_aligned(ws) || !is_aligned(h, 16)) return DORY_ERR_MISALIGNED;
  if (ws_bytes < ws_layout(m, n_rows).total) return DORY_ERR_BUFFER_TOO_SMALL;
  CallCtx c;
  c.m = m; c.kv = nullptr; c.w = ws_bind(m, ws, n_rows); c.n = n_rows; c.decode = false;
  c.seq = 0; c.pos0 = 0; c.dseq = nullptr; c.dpos = nullptr; c.max_pos = 0; c.k = 1;
  c.s = static_cast<cudaStream_t>(stream);
  m->cur_launches = m->cur_sublayers = 0;
  if (launch_f32_to_bf16(h, c.w.hb, size_t(n_rows) * m->d, c.s) != cudaSuccess) return DORY_ERR_CUDA;
  if (mlp_sublayer(c, layer, h, c.w.hb, false, false, nullptr) != cudaSuccess) return DORY_ERR_CUDA;
  return DORY_OK;
}

}  // extern "C"

namespace {

// Scratch of the MLP-sublayer backward for R rows.
struct BwdLayout {
  size_t hb, gu, a, y, dy, da, dgu, dg, du, dhx, part, total;
  int grid;
};

BwdLayout bwd_layout(const dory_model* m, int R) {
  BwdLayout L;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes); return at; };
  const size_t r = size_t(R), d = m->d, ff = m->ff;
  L.grid = mlp_bwd_row_grid(R, m->num_sms);
  L.hb = take(r * d * 2);          // bf16 copy of h (both GEMMs' operand)
  L.gu = take(r * 2 * ff * 4);     // [g | u] products, packed like W_gu
  L.a = take(r * ff * 2);          // SwiGLU activations (bf16)
  L.y = take(r * d * 4);           // down projection
  L.dy = take(r * d * 2);          // dL/dy (bf16 operand)
  L.da = take(r * ff * 4);         // dL/da
  L.dgu = take(r * 2 * ff * 2);    // dL/d[g | u], packed (dgrad operand)
  L.dg = take(r * ff * 2);         // dL/dg, dL/du (wgrad operands)
  L.du = take(r * ff * 2);
  L.dhx = take(r * d * 4);         // dL/dh through the gate / up projection
  L.part = take(size_t(L.grid) * d * 4);
  L.total = o;
  return L;
}

// C[M, N] (fp32, row pitch ld_out, 0 = N) = op(A) op(B)^T on the tcgen05
// GEMM; A is stored [M][K] or, with a_mn, [K][M]; B [N][K] or, with b_mn,
// [K][N]; lda / ldb: their row pitches in elements (0 = the row length).  K
// is rounded up to the 64-element step: the maps' K extent is K, so the tail
// reads zeros.
cudaError_t gemm_f32(const dory_model* m, const void* A, int a_mn, const void* B, int b_mn,
                     float* C, int M, int N, int K, cudaStream_t s, int ld_out = 0, int lda = 0,
                     int ldb = 0, int causal = kCausalNone, int causal_T = 0) {
  const int BN = (N % 256 == 0) ? 256 : 128;
  CUtensorMap ta, tb;
  const bool ok =
      (a_mn ? make_tmap_bf16_mn(&ta, A, K, M, lda) : make_tmap_bf16_ld(&ta, A, M, K, lda ? lda : K, 128)) &&
      (b_mn ? make_tmap_bf16_mn(&tb, B, K, N, ldb) : make_tmap_bf16_ld(&tb, B, N, K, ldb ? ldb : K, BN));
  if (!ok) return cudaErrorInvalidValue;
  GemmParams p;
  p.M = M; p.N = N; p.K = (K + 63) / 64 * 64;
  p.epi = kEpiStoreF32; p.out_f32 = C; p.ld_out = ld_out > 0 ? ld_out : N;
  p.a_mn = a_mn; p.b_mn = b_mn;
  p.causal = causal; p.causal_T = causal_T;
  p.status = m->status;
  return launch_gemm(ta, tb, p, BN, 128, m->num_sms, s);
}

// Scratch of the attention-sublayer backward for a T-row training sequence.
struct AttnBwdLayout {
  size_t hb, raw, qh, kh, vb, gate, rope, qs, ks, vs, S, P, Os, o, y, dy, part, dout, dOs, dS, dV,
      dQ, dK, dq_hat, dk_hat, dv, d_raw, dhx, dW, ds_part, total;
  int Tp, grid_row, grid_qk;
};

AttnBwdLayout attn_bwd_layout(const dory_model* m, int T) {
  AttnBwdLayout L;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes); return at; };
  const size_t t = size_t(T), d = m->d, hq = m->hq, hkv = m->hkv, hd = m->hd, G = hq / hkv;
  const size_t da = hq * hd, ldq = m->ld_qkvg;
  L.Tp = (T + 7) / 8 * 8;
  const size_t tp = size_t(L.Tp);
  L.grid_row = mlp_bwd_row_grid(T, m->num_sms);
  L.grid_qk = qk_bwd_grid(m->num_sms);
  L.hb = take(t * d * 2);
  L.raw = take(t * ldq * 4);               // q | k | v | gate logits before the epilogue
  L.qh = take(t * hq * hd * 2);
  L.kh = take(t * hkv * hd * 2);
  L.vb = take(t * hkv * hd * 2);
  L.gate = take(t * hq * 4);
  L.rope = take(t * (hd / 2) * 8);
  L.qs = take(hkv * G * t * hd * 2);       // per KV head: its group's queries stacked
  L.ks = take(hkv * t * hd * 2);
  L.vs = take(hkv * t * hd * 2);
  L.S = take(hkv * G * t * tp * 4);        // per KV head: S, then dP
  L.P = take(hkv * G * t * tp * 2);        // P of every KV head
  L.Os = take(hkv * G * t * hd * 4);       // P V before the gate
  L.o = take(t * da * 2);
  L.y = take(t * d * 4);
  L.dy = take(t * d * 2);
  L.part = take(size_t(L.grid_row) * d * 4);
  L.dout = take(t * da * 4);
  L.dOs = take(hkv * G * t * hd * 2);
  L.dS = take(hkv * G * t * tp * 2);
  L.dV = take(hkv * t * hd * 4);
  L.dQ = take(hkv * G * t * hd * 4);
  L.dK = take(hkv * t * hd * 4);
  L.dq_hat = take(t * hq * hd * 4);
  L.dk_hat = take(t * hkv * hd * 4);
  L.dv = take(t * hkv * hd * 4);
  L.d_raw = take(t * ldq * 2);
  L.dhx = take(t * d * 4);
  L.dW = take(size_t(m->n_qkvg) * d * 4);
  L.ds_part = take(size_t(L.grid_qk) * hd * 4);
  L.total = o;
  return L;
}

}  // namespace

extern "C" {

size_t dory_mlp_backward_workspace_bytes(const dory_model* m, int n_rows) {
  if (!m || n_rows <= 0) return 0;
  return bwd_layout(m, n_rows).total;
}

int dory_mlp_sublayer_backward(dory_model* m, int layer, int n_rows, const float* h_in,
                               const float* dh_out, float* dh_in, float* d_w_gate, float* d_w_up,
                               float* d_w_down, float* d_alpha, void* ws, size_t ws_bytes,
                               void* stream) {
  if (!m || !h_in || !dh_out || !dh_in || !d_w_gate || !d_w_up || !d_w_down || !d_alpha || !ws ||
      n_rows <= 0 || layer < 0 || layer >= m->nb)
    return DORY_ERR_INVALID_ARG;
  if (m->mx) return DORY_ERR_BAD_CONFIG;   // bf16 weights only
  const void* ptrs[8] = {h_in, dh_out, dh_in, d_w_gate, d_w_up, d_w_down, d_alpha, nullptr};
  for (int i = 0; i < 7; ++i)
    if (!is_aligned(ptrs[i], 16)) return DORY_ERR_MISALIGNED;
  if (!is_aligned(ws)) return DORY_ERR_MISALIGNED;
  const BwdLayout L = bwd_layout(m, n_rows);
  if (ws_bytes < L.total) return DORY_ERR_BUFFER_TOO_SMALL;
  uint8_t* b = static_cast<uint8_t*>(ws);
  auto bf = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(b + off); };
  auto f32 = [&](size_t off) { return reinterpret_cast<float*>(b + off); };
  const BlockW& W = m->blocks[layer];
  const int R = n_rows, d = m->d, ff = m->ff;
  const float eps = m->cfg.norm_eps, gs = m->cfg.gate_scale;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  // forward again (the same bf16 operands as the inference path)
  e = e ? e : launch_f32_to_bf16(h_in, bf(L.hb), size_t(R) * d, s);
  e = e ? e : gemm_f32(m, bf(L.hb), 0, W.wgu, 0, f32(L.gu), R, 2 * ff, d, s);
  e = e ? e : launch_swiglu_post(f32(L.gu), 1, size_t(R) * 2 * ff, R, ff, gs, 128, bf(L.a), s);
  e = e ? e : gemm_f32(m, bf(L.a), 0, W.wd, 0, f32(L.y), R, d, ff, s);
  // the nGPT update's backward: dh (direct part), dL/dy, dalpha partials
  e = e ? e : launch_mlp_bwd_row(f32(L.y), h_in, W.alpha_mlp, dh_out, R, d, eps, dh_in, bf(L.dy),
                                 f32(L.part), L.grid, s);
  // down projection: da = dy W_d (W_d [d][ff] read MN-major), dW_d = dy^T a
  e = e ? e : gemm_f32(m, bf(L.dy), 0, W.wd, 1, f32(L.da), R, ff, d, s);
  e = e ? e : gemm_f32(m, bf(L.dy), 1, bf(L.a), 1, d_w_down, d, ff, R, s);
  // SwiGLU, then the gate / up projection: dh += d[g | u] W_gu, dW_g = dg^T h_b, dW_u = du^T h_b
  e = e ? e : launch_swiglu_bwd(f32(L.gu), f32(L.da), R, ff, 128, gs, bf(L.dgu), bf(L.dg),
                                bf(L.du), s);
  e = e ? e : gemm_f32(m, bf(L.dgu), 0, W.wgu, 1, f32(L.dhx), R, d, 2 * ff, s);
  e = e ? e : gemm_f32(m, bf(L.dg), 1, bf(L.hb), 1, d_w_gate, ff, d, R, s);
  e = e ? e : gemm_f32(m, bf(L.du), 1, bf(L.hb), 1, d_w_up, ff, d, R, s);
  e = e ? e : launch_add_inplace(dh_in, f32(L.dhx), size_t(R) * d, s);
  e = e ? e : launch_colsum(f32(L.part), L.grid, d, d_alpha, s);
  return e == cudaSuccess ? DORY_OK : DORY_ERR_CUDA;
}

}  // extern "C"

namespace {

// n auxiliary streams of the model (created on first use)
bool aux_streams(dory_model* m, int n) {
  if (!m->fork_event && cudaEventCreateWithFlags(&m->fork_event, cudaEventDisableTiming) != cudaSuccess)
    return false;
  while (static_cast<int>(m->aux_streams.size()) < n) {
    cudaStream_t x;
    cudaEvent_t ev;
    if (cudaStreamCreateWithFlags(&x, cudaStreamNonBlocking) != cudaSuccess) return false;
    if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) {
      cudaStreamDestroy(x);
      return false;
    }
    m->aux_streams.push_back(x);
    m->aux_events.push_back(ev);
  }
  return true;
}

// Work recorded on `s` so far happens before what is enqueued next on the
// first n auxiliary streams, and what those hold happens before what is
// enqueued next on `s`.
cudaError_t fork_streams(dory_model* m, int n, cudaStream_t s) {
  cudaError_t e = cudaEventRecord(m->fork_event, s);
  for (int i = 0; i < n && e == cudaSuccess; ++i) e = cudaStreamWaitEvent(m->aux_streams[i], m->fork_event, 0);
  return e;
}
cudaError_t join_streams(dory_model* m, int n, cudaStream_t s) {
  cudaError_t e = cudaSuccess;
  for (int i = 0; i < n && e == cudaSuccess; ++i) {
    e = cudaEventRecord(m->aux_events[i], m->aux_streams[i]);
    e = e ? e : cudaStreamWaitEvent(s, m->aux_events[i], 0);
  }
  return e;
}

}  // namespace

extern "C" {

size_t dory_attention_backward_workspace_bytes(const dory_model* m, int n_rows) {
  if (!m || n_rows <= 0) return 0;
  return attn_bwd_layout(m, n_rows).total;
}

int dory_attention_sublayer_backward(dory_model* m, int layer, int n_rows, const float* h_in,
                                     const float* dh_out, float* dh_in, float* d_wq, float* d_wk,
                                     float* d_wv, float* d_wg, float* d_wo, float* d_alpha,
                                     float* d_s_qk, void* ws, size_t ws_bytes, void* stream) {
  if (!m || !h_in || !dh_out || !dh_in || !d_wq || !d_wk || !d_wv || !d_wg || !d_wo || !d_alpha ||
      !d_s_qk || !ws || n_rows <= 0 || layer < 0 || layer >= m->nb)
    return DORY_ERR_INVALID_ARG;
  if (m->mx) return DORY_ERR_BAD_CONFIG;   // bf16 weights only
  const void* ptrs[10] = {h_in, dh_out, dh_in, d_wq, d_wk, d_wv, d_wg, d_wo, d_alpha, d_s_qk};
  for (const void* q : ptrs)
    if (!is_aligned(q, 16)) return DORY_ERR_MISALIGNED;
  if (!is_aligned(ws)) return DORY_ERR_MISALIGNED;
  const AttnBwdLayout L = attn_bwd_layout(m, n_rows);
  if (ws_bytes < L.total) return DORY_ERR_BUFFER_TOO_SMALL;
  uint8_t* b = static_cast<uint8_t*>(ws);
  auto bf = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(b + off); };
  auto f32 = [&](size_t off) { return reinterpret_cast<float*>(b + off); };
  const BlockW& W = m->blocks[layer];
  const int T = n_rows, Tp = L.Tp, d = m->d, hq = m->hq, hkv = m->hkv, hd = m->hd;
  const int G = hq / hkv, da = hq * hd, nq = m->n_qkvg, ldq = m->ld_qkvg;
  const int window = W.full ? 0 : m->cfg.window;
  const float eps = m->cfg.norm_eps, scale = m->cfg.softmax_scale;
  const size_t head_q = size_t(G) * T * hd, head_kv = size_t(T) * hd, head_p = size_t(G) * T * Tp;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float2* rope = reinterpret_cast<float2*>(b + L.rope);
  cudaError_t e = cudaSuccess;

  // ---- forward again: projections, q_hat / k_hat / v / gates, attention, y
  e = e ? e : launch_f32_to_bf16(h_in, bf(L.hb), size_t(T) * d, s);
  e = e ? e : launch_rope_table(W.full ? m->inv_freq_full : m->inv_freq_swa, hd, T, 0, nullptr,
                                rope, s);
  e = e ? e : gemm_f32(m, bf(L.hb), 0, W.wqkvg, 0, f32(L.raw), T, nq, d, s, ldq);
  if (e == cudaSuccess) {
    QkvgPostParams pp;
    pp.part = f32(L.raw); pp.splits = 1; pp.split_stride = size_t(T) * ldq; pp.ld = ldq;
    pp.rows = T; pp.n_q_heads = hq; pp.n_kv_heads = hkv; pp.hd = hd;
    pp.s_qk = W.s_qk; pp.rope = rope; pp.norm_eps = eps;
    pp.q_out = bf(L.qh); pp.k_out = bf(L.kh); pp.v_out = bf(L.vb); pp.gate_out = f32(L.gate);
    e = launch_qkvg_post(pp, s);
  }
  // the KV heads run concurrently, one auxiliary stream each
  if (!aux_streams(m, hkv)) return DORY_ERR_CUDA;
  e = e ? e : fork_streams(m, hkv, s);
  for (int h = 0; h < hkv && e == cudaSuccess; ++h) {
    cudaStream_t hs = m->aux_streams[h];
    __nv_bfloat16* qs = bf(L.qs) + h * head_q;
    __nv_bfloat16* ks = bf(L.ks) + h * head_kv;
    __nv_bfloat16* vs = bf(L.vs) + h * head_kv;
    __nv_bfloat16* P = bf(L.P) + h * head_p;
    float* S = f32(L.S) + h * head_p;
    e = e ? e : launch_gather_heads(bf(L.qh), T, hq, h * G, G, hd, qs, hs);
    e = e ? e : launch_gather_heads(bf(L.kh), T, hkv, h, 1, hd, ks, hs);
    e = e ? e : launch_gather_heads(bf(L.vb), T, hkv, h, 1, hd, vs, hs);
    e = e ? e : gemm_f32(m, qs, 0, ks, 0, S, G * T, T, hd, hs, Tp, 0, 0, kCausalTiles, T);
    e = e ? e : launch_softmax_rows(S, G * T, T, Tp, window, scale, P, hs);
    e = e ? e : gemm_f32(m, P, 0, vs, 1, f32(L.Os) + h * head_q, G * T, hd, T, hs, 0, Tp, 0,
                         kCausalKeysK, T);                                          // P V
  }
  e = e ? e : join_streams(m, hkv, s);
  e = e ? e : launch_gated_output(f32(L.Os), f32(L.gate), T, hq, G, hd, bf(L.o), s);
  e = e ? e : gemm_f32(m, bf(L.o), 0, W.wo, 0, f32(L.y), T, d, da, s);

  // ---- backward: nGPT update, output projection, gates
  e = e ? e : launch_mlp_bwd_row(f32(L.y), h_in, W.alpha_attn, dh_out, T, d, eps, dh_in, bf(L.dy),
                                 f32(L.part), L.grid_row, s);
  e = e ? e : gemm_f32(m, bf(L.dy), 0, W.wo, 1, f32(L.dout), T, da, d, s);       // do = dy W_o
  e = e ? e : gemm_f32(m, bf(L.dy), 1, bf(L.o), 1, d_wo, d, da, T, s);          // dW_o = dy^T o
  e = e ? e : cudaMemsetAsync(b + L.d_raw, 0, size_t(T) * ldq * 2, s);
  e = e ? e : launch_gate_bwd(f32(L.dout), f32(L.Os), f32(L.gate), T, hq, G, hd, bf(L.dOs),
                              bf(L.d_raw), ldq, da + 2 * hkv * hd, s);
  // ---- attention, the KV heads concurrently (each writes its own rows of
  // dq_hat / dk_hat / dv)
  e = e ? e : fork_streams(m, hkv, s);
  for (int h = 0; h < hkv && e == cudaSuccess; ++h) {
    cudaStream_t hs = m->aux_streams[h];
    const __nv_bfloat16* qs = bf(L.qs) + h * head_q;
    const __nv_bfloat16* ks = bf(L.ks) + h * head_kv;
    const __nv_bfloat16* vs = bf(L.vs) + h * head_kv;
    const __nv_bfloat16* P = bf(L.P) + h * head_p;
    const __nv_bfloat16* dOs = bf(L.dOs) + h * head_q;
    float* dP = f32(L.S) + h * head_p;
    __nv_bfloat16* dS = bf(L.dS) + h * head_p;
    float* dV = f32(L.dV) + h * head_kv;
    float* dQ = f32(L.dQ) + h * head_q;
    float* dK = f32(L.dK) + h * head_kv;
    e = e ? e : gemm_f32(m, dOs, 0, vs, 0, dP, G * T, T, hd, hs, Tp, 0, 0, kCausalTiles,
                         T);                                                        // dP = dO V^T
    e = e ? e : launch_softmax_bwd_rows(P, dP, G * T, T, Tp, window, scale, dS, hs);
    e = e ? e : gemm_f32(m, P, 1, dOs, 1, dV, T, hd, G * T, hs, 0, Tp, 0, kCausalRowsK,
                         T);                                                        // dV = P^T dO
    e = e ? e : gemm_f32(m, dS, 0, ks, 1, dQ, G * T, hd, T, hs, 0, Tp, 0, kCausalKeysK,
                         T);                                                        // dQ = dS K
    e = e ? e : gemm_f32(m, dS, 1, qs, 1, dK, T, hd, G * T, hs, 0, Tp, 0, kCausalRowsK,
                         T);                                                        // dK = dS^T Q
    e = e ? e : launch_scatter_heads(dQ, T, G, hd, hq, h * G, f32(L.dq_hat), hs);
    e = e ? e : launch_scatter_heads(dK, T, 1, hd, hkv, h, f32(L.dk_hat), hs);
    e = e ? e : launch_scatter_heads(dV, T, 1, hd, hkv, h, f32(L.dv), hs);
  }
  e = e ? e : join_streams(m, hkv, s);
  // ---- QK norm and RoPE, then the projection's dgrad and wgrad
  e = e ? e : launch_v_grad(f32(L.dv), T, hkv, hd, bf(L.d_raw), ldq, da + hkv * hd, s);
  e = e ? e : launch_qk_bwd(f32(L.raw), ldq, f32(L.dq_hat), f32(L.dk_hat), W.s_qk, rope, T, hq,
                            hkv, hd, eps, bf(L.d_raw), ldq, f32(L.ds_part), L.grid_qk, s);
  e = e ? e : gemm_f32(m, bf(L.d_raw), 0, W.wqkvg, 1, f32(L.dhx), T, d, nq, s, 0, ldq);
  e = e ? e : launch_add_inplace(dh_in, f32(L.dhx), size_t(T) * d, s);
  e = e ? e : gemm_f32(m, bf(L.d_raw), 1, bf(L.hb), 1, f32(L.dW), nq, d, T, s, 0, ldq);
  if (e == cudaSuccess) {
    const size_t row = size_t(d) * 4;
    const size_t kvr = size_t(hkv) * hd;
    const uint8_t* dW = b + L.dW;
    e = cudaMemcpyAsync(d_wq, dW, size_t(da) * row, cudaMemcpyDeviceToDevice, s);
    e = e ? e : cudaMemcpyAsync(d_wk, dW + size_t(da) * row, kvr * row, cudaMemcpyDeviceToDevice, s);
    e = e ? e : cudaMemcpyAsync(d_wv, dW + (da + kvr) * row, kvr * row, cudaMemcpyDeviceToDevice, s);
    e = e ? e : cudaMemcpyAsync(d_wg, dW + (da + 2 * kvr) * row, size_t(hq) * row,
                                cudaMemcpyDeviceToDevice, s);
  }
  e = e ? e : launch_colsum(f32(L.part), L.grid_row, d, d_alpha, s);
  e = e ? e : launch_colsum(f32(L.ds_part), L.grid_qk, hd, d_s_qk, s);
  return e == cudaSuccess ? DORY_OK : DORY_ERR_CUDA;
}

size_t dory_last_loop_grad_layout(const dory_model* m, size_t* offsets) {
  if (!m) return 0;
  const size_t d = m->d, hd = m->hd, da = size_t(m->hq) * hd, kvr = size_t(m->hkv) * hd,
               ff = m->ff;
  const size_t sizes[kGradTensors] = {da * d, kvr * d, kvr * d, size_t(m->hq) * d, d * da,
                                      ff * d, ff * d, d * ff, d, d, hd};
  const int trained = m->cfg.n_rec_blocks + m->cfg.n_out_blocks;
  size_t o = 0;
  for (int i = 0; i < trained; ++i)
    for (int t = 0; t < kGradTensors; ++t) {
      if (offsets) offsets[i * kGradTensors + t] = o;
      o = align_up(o + sizes[t] * 4);
    }
  return o;
}

size_t dory_last_loop_backward_workspace_bytes(const dory_model* m, int n_rows) {
  if (!m || n_rows <= 0) return 0;
  const size_t act = align_up(size_t(n_rows) * m->d * 4);
  const int saved = 2 * (m->cfg.n_rec_blocks + m->cfg.n_out_blocks);
  return align_up(ws_layout(m, n_rows).total) + (saved + 2) * act +
         std::max(bwd_layout(m, n_rows).total, attn_bwd_layout(m, n_rows).total);
}

int dory_last_loop_backward(dory_model* m, dory_kv* kv, int n_rows, const float* h_in,
                            const float* dh_out, int k, float* h_out, float* dx, void* grads,
                            size_t grad_bytes, void* ws, size_t ws_bytes, void* stream) {
  if (!m || !kv || kv->m != m || !h_in || !dh_out || !dx || !grads || !ws || n_rows <= 0)
    return DORY_ERR_INVALID_ARG;
  if (m->mx) return DORY_ERR_BAD_CONFIG;   // bf16 weights only
  if (k < 1 || k > (m->cfg.allow_extrapolated_k ? 8 : 4)) return DORY_ERR_K_RANGE;
  if (kv->mode == DORY_KV_PER_LOOP && k > kv->k_max) return DORY_ERR_K_EXCEEDS_KMAX;
  if (n_rows > kv->max_ctx) return DORY_ERR_CTX_OVERFLOW;
  if (!is_aligned(h_in, 16) || !is_aligned(dh_out, 16) || !is_aligned(dx, 16) ||
      (h_out && !is_aligned(h_out, 16)) || !is_aligned(grads) || !is_aligned(ws))
    return DORY_ERR_MISALIGNED;
  if (grad_bytes < dory_last_loop_grad_layout(m, nullptr) ||
      ws_bytes < dory_last_loop_backward_workspace_bytes(m, n_rows))
    return DORY_ERR_BUFFER_TOO_SMALL;
  const int T = n_rows, n_in = m->cfg.n_in_blocks, n_rec = m->cfg.n_rec_blocks, nb = m->nb;
  const size_t act = align_up(size_t(T) * m->d * 4);
  uint8_t* b = static_cast<uint8_t*>(ws);
  uint8_t* saved = b + align_up(ws_layout(m, T).total);
  const int n_saved = 2 * (nb - n_in);
  float* A = reinterpret_cast<float*>(saved + size_t(n_saved) * act);
  float* Bf = reinterpret_cast<float*>(saved + size_t(n_saved + 1) * act);
  uint8_t* sub = saved + size_t(n_saved + 2) * act;
  const size_t sub_bytes = ws_bytes - size_t(sub - b);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto save = [&](int i, const float* h) {
    return cudaMemcpyAsync(saved + size_t(i) * act, h, size_t(T) * m->d * 4,
                           cudaMemcpyDeviceToDevice, s);
  };

  // ---- forward: the stack as a prefill of the sequence at position 0, the
  // inputs of the final recurrent invocation's and the output block's
  // sublayers saved
  CallCtx c;
  c.m = m; c.kv = kv; c.w = ws_bind(m, b, T); c.n = T; c.decode = false;
  c.seq = 0; c.pos0 = 0; c.dseq = nullptr; c.dpos = nullptr; c.max_pos = T - 1; c.k = k;
  c.s = s;
  m->cur_launches = m->cur_sublayers = 0;
  for (int i = 0; i < kPaths; ++i) m->cur_paths[i] = 0;
  cudaError_t e = cudaMemcpyAsync(c.w.h32, h_in, size_t(T) * m->d * 4, cudaMemcpyDeviceToDevice, s);
  e = e ? e : launch_f32_to_bf16(c.w.h32, c.w.hb, size_t(T) * m->d, s);
  e = e ? e : enqueue_rope_tables(c);
  const bool last_loop = kv->mode == DORY_KV_LAST_LOOP;
  for (int blk = 0; blk < n_in && e == cudaSuccess; ++blk) {
    const bool last = blk == n_in - 1;
    e = attention_sublayer(c, blk, 1, c.w.h32, c.w.hb, true);
    e = e ? e : mlp_sublayer(c, blk, c.w.h32, c.w.hb, last, last, nullptr);
  }
  int si = 0;
  for (int j = 1; j <= k && e == cudaSuccess; ++j) {
    for (int blk = n_in; blk < n_in + n_rec && e == cudaSuccess; ++blk) {
      const bool commit = !last_loop || j == k;
      if (j == k) e = save(si++, c.w.h32);
      e = e ? e : attention_sublayer(c, blk, j, c.w.h32, c.w.hb, commit);
      if (j == k) e = e ? e : save(si++, c.w.h32);
      const bool reinject = (blk == n_in + n_rec - 1) && j < k;
      e = e ? e : mlp_sublayer(c, blk, c.w.h32, c.w.hb, false, reinject, nullptr, j);
    }
  }
  for (int blk = n_in + n_rec; blk < nb && e == cudaSuccess; ++blk) {
    e = save(si++, c.w.h32);
    e = e ? e : attention_sublayer(c, blk, 1, c.w.h32, c.w.hb, true);
    e = e ? e : save(si++, c.w.h32);
    e = e ? e : mlp_sublayer(c, blk, c.w.h32, c.w.hb, false, false, nullptr);
  }
  if (e == cudaSuccess && h_out)
    e = cudaMemcpyAsync(h_out, c.w.h32, size_t(T) * m->d * 4, cudaMemcpyDeviceToDevice, s);
  e = e ? e : cudaMemcpyAsync(A, dh_out, size_t(T) * m->d * 4, cudaMemcpyDeviceToDevice, s);
  for (int i = 0; i < kPaths; ++i) m->last_paths[i] = m->cur_paths[i];
  if (e != cudaSuccess) return DORY_ERR_CUDA;

  // ---- backward through the output block, then the final recurrent invocation
  size_t off[kGradTensors * 64];
  const int trained = nb - n_in;
  if (trained > 64) return DORY_ERR_BAD_CONFIG;
  dory_last_loop_grad_layout(m, off);
  uint8_t* g = static_cast<uint8_t*>(grads);
  auto gp = [&](int blk, int t) { return reinterpret_cast<float*>(g + off[(blk - n_in) * kGradTensors + t]); };
  for (int i = n_saved - 1; i >= 0; --i) {
    const int blk = n_in + i / 2;
    const float* hin = reinterpret_cast<const float*>(saved + size_t(i) * act);
    int st;
    if (i % 2 == 1)
      st = dory_mlp_sublayer_backward(m, blk, T, hin, A, Bf, gp(blk, 5), gp(blk, 6), gp(blk, 7),
                                      gp(blk, 9), sub, sub_bytes, stream);
    else
      st = dory_attention_sublayer_backward(m, blk, T, hin, A, Bf, gp(blk, 0), gp(blk, 1),
                                            gp(blk, 2), gp(blk, 3), gp(blk, 4), gp(blk, 8),
                                            gp(blk, 10), sub, sub_bytes, stream);
    if (st != DORY_OK) return st;
    std::swap(A, Bf);
  }
  if (cudaMemcpyAsync(dx, A, size_t(T) * m->d * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return DORY_ERR_CUDA;
  return DORY_OK;
}

int dory_gemm_bf16_mn(const void* A, const void* B, float* C, int M, int N, int K, int a_mn,
                      int b_mn, void* stream) {
  if (!A || !B || !C || M <= 0 || N <= 0 || K <= 0 || N % 128) return DORY_ERR_INVALID_ARG;
  if ((a_mn && M % 8) || (b_mn && N % 8) || (!a_mn && K % 8) || (!b_mn && K % 8))
    return DORY_ERR_INVALID_ARG;
  if (!is_aligned(A, 16) || !is_aligned(B, 16) || !is_aligned(C, 16)) return DORY_ERR_MISALIGNED;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return DORY_ERR_CUDA;
  const int BN = (N % 256 == 0) ? 256 : 128;
  CUtensorMap ta, tb;
  const bool ok = (a_mn ? make_tmap_bf16_mn(&ta, A, K, M) : make_tmap_bf16(&ta, A, M, K, 128)) &&
                  (b_mn ? make_tmap_bf16_mn(&tb, B, K, N) : make_tmap_bf16(&tb, B, N, K, BN));
  if (!ok) return DORY_ERR_CUDA;
  GemmParams p;
  p.M = M; p.N = N; p.K = (K + 63) / 64 * 64;
  p.epi = kEpiStoreF32; p.out_f32 = C; p.ld_out = N;
  p.a_mn = a_mn ? 1 : 0; p.b_mn = b_mn ? 1 : 0;
  if (launch_gemm(ta, tb, p, BN, 128, sms, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DORY_ERR_CUDA;
  return DORY_OK;
}

int dory_debug_mask_probe(dory_model* m, int layer, int32_t* d_probe, int max_rows) {
  if (!m) return DORY_ERR_INVALID_ARG;
  if (!d_probe) {
    m->probe = nullptr;
    m->probe_layer = -1;
    m->probe_rows = 0;
    return DORY_OK;
  }
  if (layer < 0 || layer >= m->nb || max_rows <= 0) return DORY_ERR_INVALID_ARG;
  if (!is_aligned(d_probe, 16)) return DORY_ERR_MISALIGNED;
  m->probe = d_probe;
  m->probe_layer = layer;
  m->probe_rows = max_rows;
  return DORY_OK;
}

int dory_debug_fused_update(dory_model* m, int enable) {
  if (!m) return DORY_ERR_INVALID_ARG;
  m->fused_update = enable != 0;
  return m->ngpt_bnc > 0 ? DORY_OK : DORY_ERR_BAD_CONFIG;
}

int dory_debug_stream_k(dory_model* m, int enable) {
  if (!m) return DORY_ERR_INVALID_ARG;
  m->stream_k = enable != 0;
  return m->sk_ws ? DORY_OK : DORY_ERR_BAD_CONFIG;
}

int dory_debug_attention_paths(const dory_model* m, int32_t* counts) {
  if (!m || !counts) return DORY_ERR_INVALID_ARG;
  for (int i = 0; i < kPaths; ++i) counts[i] = m->last_paths[i];
  return DORY_OK;
}

int dory_debug_wait_timeout(dory_model* m, uint32_t limit_us, void* stream) {
  if (!m || limit_us == 0 || limit_us > 1000000u) return DORY_ERR_INVALID_ARG;
  if (launch_wait_timeout(m->status, uint64_t(limit_us) * 1000ull, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return DORY_ERR_CUDA;
  return DORY_OK;
}

int dory_quant_mxfp8(const void* src, int rows, int K, void* codes, void* scales, void* stream) {
  if (!src || !codes || !scales || rows <= 0 || K <= 0 || K % 128) return DORY_ERR_INVALID_ARG;
  if (!is_aligned(src, 16) || !is_aligned(codes, 16)) return DORY_ERR_MISALIGNED;
  const __nv_bfloat16* seg[1] = {static_cast<const __nv_bfloat16*>(src)};
  if (launch_quant_mxfp8_bf16(seg, nullptr, 1, 0, rows, 128, K, 0, 1e-20f, static_cast<uint8_t*>(codes),
                              static_cast<uint8_t*>(scales),
                              static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DORY_ERR_CUDA;
  return DORY_OK;
}

size_t dory_mxfp8_scale_bytes(int rows, int K) {
  if (rows <= 0 || K <= 0 || K % 128) return 0;
  return mxfp8_scale_bytes(rows, K);
}

size_t dory_gemm_mxfp8_workspace_bytes(int M, int N, int K) {
  if (M <= 0 || N <= 0 || K <= 0 || K % 128) return 0;
  return align_up(size_t(M) * K) + align_up(mxfp8_scale_bytes(M, K)) + align_up(size_t(N) * K) +
         align_up(mxfp8_scale_bytes(N, K, 256));
}

int dory_gemm_mxfp8(const void* A, const void* B, float* C, int M, int N, int K, int k_splits,
                    void* ws, size_t ws_bytes, void* stream) {
  if (!A || !B || !C || !ws || M <= 0 || N <= 0 || K <= 0 || K % 128 || k_splits < 1 ||
      k_splits > kMaxKSplits)
    return DORY_ERR_INVALID_ARG;
  if (!is_aligned(A, 16) || !is_aligned(B, 16) || !is_aligned(C, 16) || !is_aligned(ws))
    return DORY_ERR_MISALIGNED;
  if (ws_bytes < dory_gemm_mxfp8_workspace_bytes(M, N, K)) return DORY_ERR_BUFFER_TOO_SMALL;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return DORY_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* a8 = static_cast<uint8_t*>(ws);
  uint8_t* asf = a8 + align_up(size_t(M) * K);
  uint8_t* b8 = asf + align_up(mxfp8_scale_bytes(M, K));
  uint8_t* bsf = b8 + align_up(size_t(N) * K);
  const __nv_bfloat16* sa[1] = {static_cast<const __nv_bfloat16*>(A)};
  const __nv_bfloat16* sb[1] = {static_cast<const __nv_bfloat16*>(B)};
  // 256-column tiles (one accumulator) when N allows, else 128 (two); B's
  // scale chunks cover whole tiles
  const int BN = (N % 256 == 0) ? 256 : 128;
  if (launch_quant_mxfp8_bf16(sa, nullptr, 1, 0, M, 128, K, 0, 1e-20f, a8, asf, s) != cudaSuccess ||
      launch_quant_mxfp8_bf16(sb, nullptr, 1, 0, N, BN, K, 0, 1e-20f, b8, bsf, s) != cudaSuccess)
    return DORY_ERR_CUDA;
  CUtensorMap ta, tb;
  if (!make_tmap_u8(&ta, a8, M, K, 128) || !make_tmap_u8(&tb, b8, N, K, BN)) return DORY_ERR_CUDA;
  GemmParams p;
  p.M = M; p.N = N; p.K = K; p.epi = kEpiStoreF32; p.out_f32 = C; p.ld_out = N;
  p.k_splits = k_splits; p.split_stride = size_t(M) * N;
  p.mx = kOperandsMxfp8; p.sfa = asf; p.sfb = bsf; p.sfa_blocks = (M + 127) / 128;
  p.sfb_blocks = (N + BN - 1) / BN * (BN / 128);
  if (launch_gemm(ta, tb, p, BN, 128, sms, s) != cudaSuccess) return DORY_ERR_CUDA;
  return DORY_OK;
}

int dory_quant_nvfp4(const void* src, int rows, int K, float g, float* d_g, void* codes,
                     void* scales, void* stream) {
  if (!src || !codes || !scales || rows <= 0 || K <= 0 || K % 256) return DORY_ERR_INVALID_ARG;
  if (!(g > 0.f) && !d_g) return DORY_ERR_INVALID_ARG;
  if (!is_aligned(src, 16) || !is_aligned(codes, 16)) return DORY_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const __nv_bfloat16* seg[1] = {static_cast<const __nv_bfloat16*>(src)};
  if (!(g > 0.f)) {
    // the tensor scale from the data: amax / (6 * 448), computed into d_g
    const size_t count[1] = {size_t(rows) * K};
    if (launch_nvfp4_tensor_scale(seg, count, 1, reinterpret_cast<uint32_t*>(d_g), d_g, s) !=
        cudaSuccess)
      return DORY_ERR_CUDA;
  }
  if (launch_quant_nvfp4_bf16(seg, nullptr, 1, 0, rows, 128, K, 0, 1e-20f, g > 0.f ? nullptr : d_g,
                              g, static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales),
                              s) != cudaSuccess)
    return DORY_ERR_CUDA;
  return DORY_OK;
}

size_t dory_nvfp4_scale_bytes(int rows, int K) {
  if (rows <= 0 || K <= 0 || K % 256) return 0;
  return nvfp4_scale_bytes(rows, K);
}

size_t dory_gemm_nvfp4_workspace_bytes(int M, int N, int K) {
  if (M <= 0 || N <= 0 || K <= 0 || K % 256) return 0;
  return align_up(size_t(M) * K / 2) + align_up(nvfp4_scale_bytes(M, K)) +
         align_up(size_t(N) * K / 2) + align_up(nvfp4_scale_bytes(N, K, 256));
}

int dory_gemm_nvfp4(const void* A, const void* B, float* C, int M, int N, int K, float g_a,
                    float g_b, int k_splits, void* ws, size_t ws_bytes, void* stream) {
  if (!A || !B || !C || !ws || M <= 0 || N <= 0 || K <= 0 || K % 256 || k_splits < 1 ||
      k_splits > kMaxKSplits || !(g_a > 0.f) || !(g_b > 0.f))
    return DORY_ERR_INVALID_ARG;
  if (!is_aligned(A, 16) || !is_aligned(B, 16) || !is_aligned(C, 16) || !is_aligned(ws))
    return DORY_ERR_MISALIGNED;
  if (ws_bytes < dory_gemm_nvfp4_workspace_bytes(M, N, K)) return DORY_ERR_BUFFER_TOO_SMALL;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return DORY_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* a4 = static_cast<uint8_t*>(ws);
  uint8_t* asf = a4 + align_up(size_t(M) * K / 2);
  uint8_t* b4 = asf + align_up(nvfp4_scale_bytes(M, K));
  uint8_t* bsf = b4 + align_up(size_t(N) * K / 2);
  const __nv_bfloat16* sa[1] = {static_cast<const __nv_bfloat16*>(A)};
  const __nv_bfloat16* sb[1] = {static_cast<const __nv_bfloat16*>(B)};
  const int BN = (N % 256 == 0) ? 256 : 128;
  if (launch_quant_nvfp4_bf16(sa, nullptr, 1, 0, M, 128, K, 0, 1e-20f, nullptr, g_a, a4, asf, s) !=
          cudaSuccess ||
      launch_quant_nvfp4_bf16(sb, nullptr, 1, 0, N, BN, K, 0, 1e-20f, nullptr, g_b, b4, bsf, s) !=
          cudaSuccess)
    return DORY_ERR_CUDA;
  CUtensorMap ta, tb;
  if (!make_tmap_u8(&ta, a4, M, K / 2, 128) || !make_tmap_u8(&tb, b4, N, K / 2, BN))
    return DORY_ERR_CUDA;
  GemmParams p;
  p.M = M; p.N = N; p.K = K; p.epi = kEpiStoreF32; p.out_f32 = C; p.ld_out = N;
  p.k_splits = k_splits; p.split_stride = size_t(M) * N;
  p.mx = kOperandsNvfp4; p.sfa = asf; p.sfb = bsf; p.sfa_blocks = (M + 127) / 128;
  p.sfb_blocks = (N + BN - 1) / BN * (BN / 128);
  p.alpha = g_a * g_b;
  if (launch_gemm(ta, tb, p, BN, 128, sms, s) != cudaSuccess) return DORY_ERR_CUDA;
  return DORY_OK;
}

int dory_gemm_bf16(const void* A, const void* B, float* C, int M, int N, int K, void* stream) {
  if (!A || !B || !C || M <= 0 || N <= 0 || K <= 0 || K % 64 || N % 128) return DORY_ERR_INVALID_ARG;
  if (!is_aligned(A, 16) || !is_aligned(B, 16) || !is_aligned(C, 16)) return DORY_ERR_MISALIGNED;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return DORY_ERR_CUDA;
  const int BN = (N % 256 == 0) ? 256 : 128;
  CUtensorMap ta, tb;
  if (!make_tmap_bf16(&ta, A, M, K, 128) || !make_tmap_bf16(&tb, B, N, K, BN)) return DORY_ERR_CUDA;
  GemmParams p;
  p.M = M; p.N = N; p.K = K; p.epi = kEpiStoreF32; p.out_f32 = C; p.ld_out = N;
  if (launch_gemm(ta, tb, p, BN, 128, sms, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DORY_ERR_CUDA;
  return DORY_OK;
}

size_t dory_gemm_bf16_streamk_workspace_bytes(int N) {
  return gemm_sk_workspace_bytes(kSkMaxGrid, N % 256 == 0 ? 256 : 128);
}

int dory_gemm_bf16_streamk(const void* A, const void* B, float* C, int M, int N, int K, void* ws,
                           size_t ws_bytes, void* stream) {
  if (!A || !B || !C || !ws || M <= 0 || N <= 0 || K <= 0 || K % 64 || N % 128)
    return DORY_ERR_INVALID_ARG;
  if (!is_aligned(A, 16) || !is_aligned(B, 16) || !is_aligned(C, 16) || !is_aligned(ws, 256))
    return DORY_ERR_MISALIGNED;
  if (ws_bytes < dory_gemm_bf16_streamk_workspace_bytes(N)) return DORY_ERR_BUFFER_TOO_SMALL;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return DORY_ERR_CUDA;
  const int BN = (N % 256 == 0) ? 256 : 128;
  CUtensorMap ta, tb;
  if (!make_tmap_bf16(&ta, A, M, K, 128) || !make_tmap_bf16(&tb, B, N, K, BN)) return DORY_ERR_CUDA;
  GemmParams p;
  p.M = M; p.N = N; p.K = K; p.epi = kEpiStoreF32; p.out_f32 = C; p.ld_out = N;
  if (sms <= kSkMaxGrid) {
    const size_t slots = static_cast<size_t>(kSkMaxGrid) * 128 * BN * 4;
    uint8_t* w = static_cast<uint8_t*>(ws);
    p.sk = 1;
    p.sk_ws = reinterpret_cast<float*>(w);
    p.sk_sync = reinterpret_cast<uint32_t*>(w + (slots + 255) / 256 * 256);
    p.status = p.sk_sync + 2 + 4 * kSkMaxGrid;
  }
  if (launch_gemm(ta, tb, p, BN, 128, sms, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DORY_ERR_CUDA;
  return DORY_OK;
}

}  // extern "C"

// ================================================================ vocabulary
struct dory_vocab {
  dory_model* m = nullptr;
  int vocab = 0;
  __nv_bfloat16* emb_in = nullptr;
  __nv_bfloat16* emb_out = nullptr;
  float* scale = nullptr;
  CUtensorMap tm_out;   // emb_out as the B operand, 256-row boxes
};

namespace {
struct VocabLayout {
  size_t in, out, scale, total;
};
VocabLayout vocab_layout(const dory_config* c, int vocab) {
  VocabLayout L;
  size_t o = 0;
  L.in = o;    o = align_up(o + size_t(vocab) * c->d_model * 2);
  L.out = o;   o = align_up(o + size_t(vocab) * c->d_model * 2);
  L.scale = o; o = align_up(o + size_t(vocab) * 4);
  L.total = o;
  return L;
}
}  // namespace

extern "C" {

size_t dory_vocab_bytes(const dory_config* cfg, int vocab) {
  if (validate_config(cfg) != DORY_OK || vocab <= 0 || vocab % 256) return 0;
  return vocab_layout(cfg, vocab).total;
}

int dory_vocab_create(dory_model* m, int vocab, const uint16_t* emb_in, const uint16_t* emb_out,
                      const float* logit_scale, void* buf, size_t bytes, void* stream,
                      dory_vocab** out) {
  if (!m || !emb_in || !emb_out || !logit_scale || !buf || !out || vocab <= 0 || vocab % 256)
    return DORY_ERR_INVALID_ARG;
  *out = nullptr;
  if (!is_aligned(buf)) return DORY_ERR_MISALIGNED;
  const VocabLayout L = vocab_layout(&m->cfg, vocab);
  if (bytes < L.total) return DORY_ERR_BUFFER_TOO_SMALL;
  std::unique_ptr<dory_vocab> v(new (std::nothrow) dory_vocab());
  if (!v) return DORY_ERR_INVALID_ARG;
  uint8_t* b = static_cast<uint8_t*>(buf);
  v->m = m;
  v->vocab = vocab;
  v->emb_in = reinterpret_cast<__nv_bfloat16*>(b + L.in);
  v->emb_out = reinterpret_cast<__nv_bfloat16*>(b + L.out);
  v->scale = reinterpret_cast<float*>(b + L.scale);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t tb = size_t(vocab) * m->d * 2;
  if (cudaMemcpyAsync(v->emb_in, emb_in, tb, cudaMemcpyDefault, s) != cudaSuccess ||
      cudaMemcpyAsync(v->emb_out, emb_out, tb, cudaMemcpyDefault, s) != cudaSuccess ||
      cudaMemcpyAsync(v->scale, logit_scale, size_t(vocab) * 4, cudaMemcpyDefault, s) != cudaSuccess)
    return DORY_ERR_CUDA;
  if (!make_tmap_bf16(&v->tm_out, v->emb_out, vocab, m->d, 256)) return DORY_ERR_CUDA;
  *out = v.release();
  return DORY_OK;
}

int dory_embed(dory_vocab* v, const int32_t* d_tokens, int n, void* h_out, void* stream) {
  if (!v || !v->m || !d_tokens || !h_out || n <= 0) return DORY_ERR_INVALID_ARG;
  if (!is_aligned(h_out, 16)) return DORY_ERR_MISALIGNED;
  if (launch_embed(v->emb_in, v->vocab, v->m->d, d_tokens, n, static_cast<__nv_bfloat16*>(h_out),
                   v->m->status, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DORY_ERR_CUDA;
  return DORY_OK;
}

int dory_lm_head(dory_vocab* v, const void* h, int n, float* logits, void* stream) {
  if (!v || !v->m || !h || !logits || n <= 0) return DORY_ERR_INVALID_ARG;
  if (!is_aligned(h, 16) || !is_aligned(logits, 16)) return DORY_ERR_MISALIGNED;
  dory_model* m = v->m;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  CUtensorMap ta;
  if (!make_tmap_bf16(&ta, h, n, m->d, 128)) return DORY_ERR_CUDA;
  GemmParams p;
  p.M = n; p.N = v->vocab; p.K = m->d; p.epi = kEpiStoreF32; p.out_f32 = logits;
  p.ld_out = v->vocab; p.status = m->status;
  if (launch_gemm(ta, v->tm_out, p, 256, m->hd, m->num_sms, s) != cudaSuccess ||
      launch_scale_columns(logits, v->scale, n, v->vocab, s) != cudaSuccess)
    return DORY_ERR_CUDA;
  return DORY_OK;
}

int dory_sample(dory_vocab* v, const float* logits, int n, float temperature, uint32_t seed,
                const int32_t* d_steps, int32_t* d_tokens, void* stream) {
  if (!v || !logits || !d_tokens || n <= 0 || !(temperature >= 0.f)) return DORY_ERR_INVALID_ARG;
  if (temperature > 0.f && !d_steps) return DORY_ERR_INVALID_ARG;
  if (launch_sample(logits, n, v->vocab, temperature, seed, d_steps, d_tokens,
                    static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DORY_ERR_CUDA;
  return DORY_OK;
}

void dory_vocab_free(dory_vocab* v) { delete v; }

}  // extern "C"

// ========================================================== allocation-free MLP
// Scratch of dory_mlp_sublayer_noalloc, part of the library image: no call
// ever allocates it.  Host code must not hand the symbol itself to a kernel;
// it looks up the device address per device below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[DORY_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kNoallocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoallocMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once
// per device, with that device current).
void* noalloc_scratch(int dev) {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) {
      cudaGetLastError();
      return nullptr;
    }
    g_noalloc_ptr[dev] = ptr;
  }
  return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" int dory_mlp_sublayer_noalloc(dory_model* m, int layer, int n_rows, float* h,
                                         void* stream) {
  if (!m || !h || n_rows <= 0 || layer < 0 || layer >= m->nb) return DORY_ERR_INVALID_ARG;
  if (m->mx) return DORY_ERR_BAD_CONFIG;   // the built-in scratch has no room for MXFP8 operands
  if (!is_aligned(h, 16)) return DORY_ERR_MISALIGNED;
  const size_t hb_bytes = align_up(size_t(n_rows) * m->d * 2);
  const size_t a_bytes = align_up(size_t(n_rows) * m->ff * 2);
  const size_t y_bytes = align_up(size_t(n_rows) * m->d * 4);
  if (hb_bytes + a_bytes + y_bytes > DORY_NOALLOC_SCRATCH_BYTES) return DORY_ERR_SCRATCH_LIMIT;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DORY_ERR_CUDA;
  if (dev != m->device || dev >= kNoallocMaxDevices) return DORY_ERR_INVALID_ARG;
  uint8_t* base = static_cast<uint8_t*>(noalloc_scratch(dev));
  if (!base) return DORY_ERR_CUDA;
  CallCtx c;
  c.m = m; c.kv = nullptr; c.n = n_rows; c.decode = false;
  c.seq = 0; c.pos0 = 0; c.dseq = nullptr; c.dpos = nullptr; c.max_pos = 0; c.k = 1;
  c.s = static_cast<cudaStream_t>(stream);
  memset(&c.w, 0, sizeof(c.w));
  c.w.hb = reinterpret_cast<__nv_bfloat16*>(base);
  c.w.a = reinterpret_cast<__nv_bfloat16*>(base + hb_bytes);
  c.w.y = reinterpret_cast<float*>(base + hb_bytes + a_bytes);
  m->cur_launches = m->cur_sublayers = 0;
  if (launch_f32_to_bf16(h, c.w.hb, size_t(n_rows) * m->d, c.s) != cudaSuccess) return DORY_ERR_CUDA;
  if (mlp_sublayer(c, layer, h, c.w.hb, false, false, nullptr) != cudaSuccess) return DORY_ERR_CUDA;
  return DORY_OK;
}
