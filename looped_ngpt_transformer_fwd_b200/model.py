"""Torch-side plumbing around the C ABI: device buffers, streams and handles.

`DoryModel` owns the caller-side memory the library asks for (packed weights,
KV caches, workspaces) as torch tensors and forwards every call to the C ABI
(`binding`).  No arithmetic of the forward pass happens here.
"""

import ctypes

import numpy as np
import torch

from . import binding as B


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


class KVCache:
    """A KV cache bound to a torch byte buffer."""

    def __init__(self, model, mode, max_seqs, max_ctx, k_max=1):
        self.model = model
        self.mode = mode
        self.max_seqs, self.max_ctx, self.k_max = max_seqs, max_ctx, k_max
        self.nbytes = B.dory_kv_bytes(model.cfg_struct, mode, max_seqs, max_ctx, k_max)
        if self.nbytes == 0:
            raise ValueError("invalid KV cache arguments")
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=model.device)
        self.handle = B.dory_kv_alloc(model.handle, mode, max_seqs, max_ctx, k_max,
                                      _ptr(self.buf), self.nbytes)

    def layout(self, layer, loop, seq, pos, head):
        return B.dory_kv_layout(self.handle, layer, loop, seq, pos, head)

    def entry_view(self, layer, loop, seq, head, which="k"):
        """bf16 view [capacity, head_dim] of one (layer, loop, seq, head) slot ring."""
        cfg = self.model.cfg
        k_off, v_off = self.layout(layer, loop, seq, 0, head)
        off = k_off if which == "k" else v_off
        full = (layer % cfg["full_period"]) == cfg["full_period"] - 1
        cap = self.max_ctx if full else min(cfg["window"], self.max_ctx)
        n = cap * cfg["head_dim"]
        return self.buf[off:off + 2 * n].view(torch.bfloat16).view(cap, cfg["head_dim"])

    def free(self):
        if self.handle:
            B.dory_kv_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


class Vocab:
    """Embedding and output tables bound to a model (dory_vocab_create)."""

    def __init__(self, model, tables):
        self.model = model
        self.size = int(tables["logit_scale"].shape[0])
        self.nbytes = B.dory_vocab_bytes(model.cfg_struct, self.size)
        if self.nbytes == 0:
            raise ValueError("vocabulary size must be a positive multiple of 256")
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=model.device)
        staged = {k: torch.from_numpy(np.ascontiguousarray(v).view(np.int16) if v.dtype == np.uint16
                                      else np.ascontiguousarray(v)).to(model.device)
                  for k, v in tables.items()}
        self.handle = B.dory_vocab_create(model.handle, self.size, _ptr(staged["emb_in"]),
                                          _ptr(staged["emb_out"]), _ptr(staged["logit_scale"]),
                                          _ptr(self.buf), self.nbytes, _stream(None))
        torch.cuda.synchronize(model.device)

    def embed(self, tokens, stream=None):
        """int32 device tokens [n] -> unit-norm bf16 rows [n, d]."""
        out = torch.empty(tokens.shape[0], self.model.cfg["d_model"], dtype=torch.bfloat16,
                          device=self.model.device)
        B.dory_embed(self.handle, _ptr(tokens), tokens.shape[0], _ptr(out), _stream(stream))
        return out

    def logits(self, h, stream=None):
        """bf16 device rows [n, d] -> fp32 logits [n, V]."""
        z = torch.empty(h.shape[0], self.size, dtype=torch.float32, device=self.model.device)
        B.dory_lm_head(self.handle, _ptr(h), h.shape[0], _ptr(z), _stream(stream))
        return z

    def sample(self, z, temperature=0.0, seed=0, steps=None, stream=None):
        """One int32 token per row of z (greedy at temperature 0)."""
        tok = torch.empty(z.shape[0], dtype=torch.int32, device=self.model.device)
        B.dory_sample(self.handle, _ptr(z), z.shape[0], float(temperature), int(seed),
                      _ptr(steps) if steps is not None else None, _ptr(tok), _stream(stream))
        return tok

    def free(self):
        if getattr(self, "handle", None):
            B.dory_vocab_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


class DoryModel:
    """Packed weights on the device plus a library handle.

    weights: callable b -> dict in the synthetic generator's format (bf16
    matrices as uint16 arrays [out, in], float32 vectors).
    """

    def __init__(self, cfg, weights, device="cuda:0", allow_extrapolated_k=False, stream=None,
                 weight_format="bf16"):
        self.cfg = cfg
        self.device = torch.device(device)
        self.weight_format = weight_format
        self.cfg_struct = B.make_config(cfg, allow_extrapolated_k, weight_format)
        nb = cfg["n_in_blocks"] + cfg["n_rec_blocks"] + cfg["n_out_blocks"]
        self.n_blocks = nb
        self.wbytes = B.dory_weight_bytes(self.cfg_struct)
        if self.wbytes == 0:
            raise ValueError("configuration rejected by dory_weight_bytes")
        self.wbuf = torch.empty(self.wbytes, dtype=torch.uint8, device=self.device)
        torch.cuda.set_device(self.device)
        staged = []
        srcs = []
        for b in range(nb):
            w = weights(b)
            dev = {}
            for name, arr in w.items():
                a = np.ascontiguousarray(arr)
                t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
                dev[name] = t.to(self.device, non_blocking=False)
            staged.append(dev)
            srcs.append(B.DoryBlockSrc(*[dev[n].data_ptr() for n in (
                "wq", "wk", "wv", "wg", "wo", "w_gate", "w_up", "w_down",
                "alpha_attn", "alpha_mlp", "s_qk")]))
        self.handle = B.dory_create(self.cfg_struct, _ptr(self.wbuf), self.wbytes, srcs,
                                    _stream(stream))
        torch.cuda.synchronize(self.device)
        del staged
        self._ws = None
        self._ws_tokens = 0

    # ---------------------------------------------------------------- buffers
    def kv_cache(self, mode, max_seqs, max_ctx, k_max=1):
        return KVCache(self, mode, max_seqs, max_ctx, k_max)

    def vocab(self, tables):
        """Bind embedding / output tables (dict: emb_in, emb_out, logit_scale)."""
        return Vocab(self, tables)

    def workspace(self, max_tokens):
        if self._ws is None or self._ws_tokens < max_tokens:
            n = B.dory_workspace_bytes(self.handle, max_tokens)
            self._ws = torch.empty(n, dtype=torch.uint8, device=self.device)
            self._ws_tokens = max_tokens
        return self._ws

    # ---------------------------------------------------------------- calls
    def prefill(self, kv, h_in, k, seq=0, pos0=0, h_out=None, stream=None):
        """h_in: [n, d] bf16 tensor on the device or in (pinned) host memory."""
        n = h_in.shape[0]
        if h_out is None:
            h_out = torch.empty_like(h_in)
        ws = self.workspace(n)
        B.dory_prefill(self.handle, kv.handle, seq, pos0, n, _ptr(h_in), _ptr(h_out), k,
                       _ptr(ws), ws.numel(), _stream(stream))
        return h_out

    def decode(self, kv, h_in, d_seq, d_pos, max_pos, k, h_out=None, stream=None):
        """One decode step; d_seq / d_pos: int32 device tensors [batch]."""
        n = h_in.shape[0]
        if h_out is None:
            h_out = torch.empty_like(h_in)
        ws = self.workspace(n)
        B.dory_decode_step(self.handle, kv.handle, n, _ptr(d_seq), _ptr(d_pos), max_pos,
                           _ptr(h_in), _ptr(h_out), k, _ptr(ws), ws.numel(), _stream(stream))
        return h_out

    def decode_mixed(self, kv, h_in, d_seq, d_pos, d_k, max_pos, k_hi, h_out=None, stream=None):
        """One decode step with a loop count per row; d_seq / d_pos / d_k: int32
        device tensors [batch], k_hi = the largest count."""
        n = h_in.shape[0]
        if h_out is None:
            h_out = torch.empty_like(h_in)
        ws = self.workspace(n)
        B.dory_decode_step_mixed(self.handle, kv.handle, n, _ptr(d_seq), _ptr(d_pos), _ptr(d_k),
                                 k_hi, max_pos, _ptr(h_in), _ptr(h_out), _ptr(ws), ws.numel(),
                                 _stream(stream))
        return h_out

    def attention_sublayer(self, kv, layer, h, loop=1, seq=0, pos0=0, stream=None):
        """In place on h: [n, d] float32 device tensor."""
        ws = self.workspace(h.shape[0])
        B.dory_attention_sublayer(self.handle, kv.handle, layer, loop, seq, pos0, h.shape[0],
                                  _ptr(h), _ptr(ws), ws.numel(), _stream(stream))
        return h

    def mlp_sublayer(self, layer, h, stream=None):
        ws = self.workspace(h.shape[0])
        B.dory_mlp_sublayer(self.handle, layer, h.shape[0], _ptr(h), _ptr(ws), ws.numel(),
                            _stream(stream))
        return h

    def last_loop_backward(self, kv, h, dh_out, k, stream=None):
        """Depth-one truncated back-propagation of one training sequence (rows of
        h = positions 0..n-1, fp32 [n, d] device tensors): returns h_out, dx
        (dL/dx_k) and grads[b][name] for every trained block b (recurrent, then
        output blocks; names as binding.GRAD_TENSORS, shapes of the weights)."""
        n, d = h.shape
        c = self.cfg
        hq, hkv, hd, ff = c["n_q_heads"], c["n_kv_heads"], c["head_dim"], c["d_ff"]
        n_in = c["n_in_blocks"]
        trained = list(range(n_in, self.n_blocks))
        total, offs = B.dory_last_loop_grad_layout(self.handle, len(trained))
        gbuf = torch.empty(total, dtype=torch.uint8, device=self.device)
        ws = torch.empty(B.dory_last_loop_backward_workspace_bytes(self.handle, n),
                         dtype=torch.uint8, device=self.device)
        f32 = dict(dtype=torch.float32, device=self.device)
        h_out = torch.empty(n, d, **f32)
        dx = torch.empty(n, d, **f32)
        B.dory_last_loop_backward(self.handle, kv.handle, n, _ptr(h), _ptr(dh_out), k, _ptr(h_out),
                                  _ptr(dx), _ptr(gbuf), gbuf.numel(), _ptr(ws), ws.numel(),
                                  _stream(stream))
        shapes = dict(wq=(hq * hd, d), wk=(hkv * hd, d), wv=(hkv * hd, d), wg=(hq, d),
                      wo=(d, hq * hd), w_gate=(ff, d), w_up=(ff, d), w_down=(d, ff),
                      alpha_attn=(d,), alpha_mlp=(d,), s_qk=(hd,))
        grads = {}
        for i, b in enumerate(trained):
            grads[b] = {}
            for t, name in enumerate(B.GRAD_TENSORS):
                nel = int(np.prod(shapes[name]))
                grads[b][name] = gbuf[offs[i][t]:offs[i][t] + 4 * nel].view(torch.float32).view(
                    *shapes[name])
        return dict(h_out=h_out, dx=dx, grads=grads, buffer=gbuf)

    def attention_sublayer_backward(self, layer, h, dh_out, stream=None):
        """Gradients of one attention sublayer on a training sequence (rows =
        positions 0..n-1) given its input h and dL/dh_out (fp32 [n, d] device
        tensors): dict of dh, d_wq, d_wk, d_wv, d_wg, d_wo, d_alpha, d_s_qk."""
        n, d = h.shape
        c = self.cfg
        hq, hkv, hd = c["n_q_heads"], c["n_kv_heads"], c["head_dim"]
        ws = torch.empty(B.dory_attention_backward_workspace_bytes(self.handle, n),
                         dtype=torch.uint8, device=self.device)
        f32 = dict(dtype=torch.float32, device=self.device)
        out = dict(dh=torch.empty(n, d, **f32), d_wq=torch.empty(hq * hd, d, **f32),
                   d_wk=torch.empty(hkv * hd, d, **f32), d_wv=torch.empty(hkv * hd, d, **f32),
                   d_wg=torch.empty(hq, d, **f32), d_wo=torch.empty(d, hq * hd, **f32),
                   d_alpha=torch.empty(d, **f32), d_s_qk=torch.empty(hd, **f32))
        B.dory_attention_sublayer_backward(
            self.handle, layer, n, _ptr(h), _ptr(dh_out), _ptr(out["dh"]), _ptr(out["d_wq"]),
            _ptr(out["d_wk"]), _ptr(out["d_wv"]), _ptr(out["d_wg"]), _ptr(out["d_wo"]),
            _ptr(out["d_alpha"]), _ptr(out["d_s_qk"]), _ptr(ws), ws.numel(), _stream(stream))
        return out

    def mlp_sublayer_backward(self, layer, h, dh_out, stream=None):
        """Gradients of one MLP sublayer given its input h and dL/dh_out (fp32
        [n, d] device tensors): dict of dh, d_w_gate, d_w_up, d_w_down, d_alpha."""
        n, d = h.shape
        ff = self.cfg["d_ff"]
        ws = torch.empty(B.dory_mlp_backward_workspace_bytes(self.handle, n), dtype=torch.uint8,
                         device=self.device)
        f32 = dict(dtype=torch.float32, device=self.device)
        out = dict(dh=torch.empty(n, d, **f32), d_w_gate=torch.empty(ff, d, **f32),
                   d_w_up=torch.empty(ff, d, **f32), d_w_down=torch.empty(d, ff, **f32),
                   d_alpha=torch.empty(d, **f32))
        B.dory_mlp_sublayer_backward(self.handle, layer, n, _ptr(h), _ptr(dh_out), _ptr(out["dh"]),
                                     _ptr(out["d_w_gate"]), _ptr(out["d_w_up"]),
                                     _ptr(out["d_w_down"]), _ptr(out["d_alpha"]), _ptr(ws),
                                     ws.numel(), _stream(stream))
        return out

    def mlp_sublayer_noalloc(self, layer, h, stream=None):
        """As mlp_sublayer, but the library supplies the scratch (no workspace)."""
        B.dory_mlp_sublayer_noalloc(self.handle, layer, h.shape[0], _ptr(h), _stream(stream))
        return h

    def mask_probe(self, layer, max_rows):
        """Start recording the attention mask of global block `layer`; returns the
        int32 device tensor [max_rows, n_q_heads, 4] the kernels fill (see
        dory_debug_mask_probe).  mask_probe_off() stops it."""
        rec = torch.empty(max_rows, self.cfg["n_q_heads"], 4, dtype=torch.int32,
                          device=self.device)
        B.dory_debug_mask_probe(self.handle, layer, _ptr(rec), max_rows)
        self._probe = rec
        return rec

    def mask_probe_off(self):
        B.dory_debug_mask_probe(self.handle, 0, None, 0)
        self._probe = None

    def fused_update(self, enable=True):
        """True when the prefill projections apply the nGPT update in their epilogue."""
        return B.dory_debug_fused_update(self.handle, enable) == 0 and enable

    def stream_k(self, enable=True):
        """True when the prefill output / down projections use stream-K tails."""
        return B.dory_debug_stream_k(self.handle, enable) == 0 and enable

    def attention_paths(self):
        return B.dory_debug_attention_paths(self.handle)

    def wait_timeout(self, limit_us, stream=None):
        B.dory_debug_wait_timeout(self.handle, limit_us, _stream(stream))

    def device_status(self, stream=None):
        return B.dory_device_status(self.handle, _stream(stream))

    def last_call_stats(self):
        return B.dory_last_call_stats(self.handle)

    def profile(self, enable=True):
        B.dory_profile_enable(self.handle, enable)

    def profile_read(self):
        """{kind: (total ms, launches)} of the last instrumented call."""
        return {k: B.dory_profile_read(self.handle, k) for k in B.KERNEL_KINDS}

    def close(self):
        if getattr(self, "handle", None):
            B.dory_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def quant_mxfp8(x, stream=None):
    """MXFP8 codes [rows, K] (uint8) and the chunked E8M0 scale bytes of bf16 rows x."""
    rows, K = x.shape
    codes = torch.empty(rows, K, dtype=torch.uint8, device=x.device)
    scales = torch.empty(B.dory_mxfp8_scale_bytes(rows, K), dtype=torch.uint8, device=x.device)
    B.dory_quant_mxfp8(_ptr(x), rows, K, _ptr(codes), _ptr(scales), _stream(stream))
    return codes, scales


def gemm_mxfp8(A, Bm, k_splits=1, stream=None):
    """Q(A) Q(Bm)^T through the block-scaled GEMM (bf16 in, MXFP8 operands, fp32
    out) as its K slices [k_splits, M, N]; the product is their sum."""
    M, K = A.shape
    N = Bm.shape[0]
    ws = torch.empty(B.dory_gemm_mxfp8_workspace_bytes(M, N, K), dtype=torch.uint8, device=A.device)
    C = torch.empty(k_splits, M, N, dtype=torch.float32, device=A.device)
    B.dory_gemm_mxfp8(_ptr(A), _ptr(Bm), _ptr(C), M, N, K, k_splits, _ptr(ws), ws.numel(),
                      _stream(stream))
    return C


def quant_nvfp4(x, g=None, stream=None):
    """NVFP4 packed codes [rows, K/2] (uint8), the chunked E4M3 scale bytes and
    the tensor scale (a 1-element fp32 device tensor) of bf16 rows x; g None
    takes the tensor scale from the data (amax / (6 * 448))."""
    rows, K = x.shape
    codes = torch.empty(rows, K // 2, dtype=torch.uint8, device=x.device)
    scales = torch.empty(B.dory_nvfp4_scale_bytes(rows, K), dtype=torch.uint8, device=x.device)
    d_g = torch.full((1,), float(g) if g is not None else 0.0, dtype=torch.float32,
                     device=x.device)
    B.dory_quant_nvfp4(_ptr(x), rows, K, float(g) if g is not None else 0.0, _ptr(d_g),
                       _ptr(codes), _ptr(scales), _stream(stream))
    return codes, scales, d_g


def gemm_nvfp4(A, Bm, g_a, g_b, k_splits=1, stream=None):
    """Q(A) Q(Bm)^T through the NVFP4 block-scaled GEMM (bf16 in, tensor scales
    g_a and g_b, fp32 out) as its K slices [k_splits, M, N]."""
    M, K = A.shape
    N = Bm.shape[0]
    ws = torch.empty(B.dory_gemm_nvfp4_workspace_bytes(M, N, K), dtype=torch.uint8, device=A.device)
    C = torch.empty(k_splits, M, N, dtype=torch.float32, device=A.device)
    B.dory_gemm_nvfp4(_ptr(A), _ptr(Bm), _ptr(C), M, N, K, float(g_a), float(g_b), k_splits,
                      _ptr(ws), ws.numel(), _stream(stream))
    return C


def gemm_bf16_mn(A, Bm, M, N, K, a_mn, b_mn, stream=None):
    """C[M, N] = op(A) op(Bm)^T through the tcgen05 GEMM with operands read
    MN-major where asked (A stored [K, M] when a_mn, Bm stored [K, N] when b_mn)."""
    C = torch.empty(M, N, dtype=torch.float32, device=A.device)
    B.dory_gemm_bf16_mn(_ptr(A), _ptr(Bm), _ptr(C), M, N, K, int(a_mn), int(b_mn), _stream(stream))
    return C


def gemm_bf16_streamk(A, Bm, ws=None, stream=None):
    """C = A @ Bm^T through the stream-K schedule; `ws` (uint8, device, zeroed
    before its first use) may be passed to keep its launch counter across
    calls.  Returns (C, ws)."""
    M, K = A.shape
    N = Bm.shape[0]
    if ws is None:
        ws = torch.zeros(B.dory_gemm_bf16_streamk_workspace_bytes(N), dtype=torch.uint8,
                         device=A.device)
    C = torch.empty(M, N, dtype=torch.float32, device=A.device)
    B.dory_gemm_bf16_streamk(_ptr(A), _ptr(Bm), _ptr(C), M, N, K, _ptr(ws), ws.numel(),
                             _stream(stream))
    return C, ws


def gemm_bf16(A, Bm, stream=None):
    """C = A @ Bm^T through the library's tcgen05 GEMM (bf16 in, fp32 out)."""
    M, K = A.shape
    N = Bm.shape[0]
    C = torch.empty(M, N, dtype=torch.float32, device=A.device)
    B.dory_gemm_bf16(_ptr(A), _ptr(Bm), _ptr(C), M, N, K, _stream(stream))
    return C
