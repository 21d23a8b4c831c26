"""ctypes binding of libdory.so (the C ABI in include/dory.h).

Argument marshalling only: every step of the forward pass runs in the
library's sm_100a kernels.  PyTorch supplies device memory and streams.  If the
shared library has not been built, importing `lib()` raises ImportError; there
is no fallback implementation.
"""

import ctypes
import os

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libdory.so")

DORY_OK = 0
DORY_KV_PER_LOOP = 0
DORY_KV_LAST_LOOP = 1
MODES = {"per_loop": DORY_KV_PER_LOOP, "last_loop": DORY_KV_LAST_LOOP}

STATUS = {
    0: "DORY_OK", -1: "DORY_ERR_INVALID_ARG", -2: "DORY_ERR_BAD_CONFIG", -3: "DORY_ERR_K_RANGE",
    -4: "DORY_ERR_K_EXCEEDS_KMAX", -5: "DORY_ERR_CTX_OVERFLOW", -6: "DORY_ERR_BUFFER_TOO_SMALL",
    -7: "DORY_ERR_MISALIGNED", -8: "DORY_ERR_CUDA", -9: "DORY_ERR_DEVICE_TIMEOUT",
    -10: "DORY_ERR_UNSUPPORTED_ARCH", -11: "DORY_ERR_DEVICE_BOUNDS", -12: "DORY_ERR_SCRATCH_LIMIT",
}

# every entry point declared in include/dory.h
EXPORTS = (
    "dory_weight_bytes", "dory_create", "dory_kv_bytes", "dory_kv_alloc", "dory_kv_layout",
    "dory_workspace_bytes", "dory_prefill", "dory_decode_step", "dory_decode_step_mixed",
    "dory_device_status",
    "dory_last_call_stats", "dory_error_string", "dory_kv_free", "dory_destroy",
    "dory_attention_sublayer", "dory_mlp_sublayer", "dory_gemm_bf16",
    "dory_profile_enable", "dory_profile_read", "dory_mlp_sublayer_noalloc",
    "dory_debug_mask_probe", "dory_debug_attention_paths", "dory_debug_wait_timeout",
    "dory_debug_fused_update", "dory_quant_mxfp8", "dory_mxfp8_scale_bytes",
    "dory_gemm_mxfp8_workspace_bytes", "dory_gemm_mxfp8", "dory_quant_nvfp4",
    "dory_nvfp4_scale_bytes", "dory_gemm_nvfp4_workspace_bytes", "dory_gemm_nvfp4",
    "dory_gemm_bf16_mn", "dory_mlp_backward_workspace_bytes", "dory_mlp_sublayer_backward",
    "dory_attention_backward_workspace_bytes", "dory_attention_sublayer_backward",
    "dory_last_loop_grad_layout", "dory_last_loop_backward_workspace_bytes",
    "dory_last_loop_backward",
    "dory_vocab_bytes", "dory_vocab_create", "dory_embed", "dory_lm_head", "dory_sample",
    "dory_vocab_free", "dory_gemm_bf16_streamk_workspace_bytes", "dory_gemm_bf16_streamk",
    "dory_debug_stream_k",
)

WEIGHT_FORMATS = {"bf16": 0, "mxfp8": 1, "nvfp4": 2}

ATTENTION_PATHS = ("prefill_tc", "prefill_mma", "decode_tma", "decode_cp")

# size of the library's built-in scratch array (DORY_NOALLOC_SCRATCH_BYTES)
NOALLOC_SCRATCH_BYTES = 8 << 20

KERNEL_KINDS = ("qkvg", "attn", "oproj", "gateup", "down", "row", "kvcommit")


class DoryError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({_errstr(status)})")


class DoryConfig(ctypes.Structure):
    _fields_ = [
        ("d_model", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("d_ff", ctypes.c_int32), ("n_in_blocks", ctypes.c_int32),
        ("n_rec_blocks", ctypes.c_int32), ("n_out_blocks", ctypes.c_int32),
        ("window", ctypes.c_int32), ("full_period", ctypes.c_int32),
        ("rope_base_swa", ctypes.c_double), ("rope_base_full", ctypes.c_double),
        ("softmax_scale", ctypes.c_float), ("gate_scale", ctypes.c_float),
        ("norm_eps", ctypes.c_float), ("allow_extrapolated_k", ctypes.c_int32),
        ("weight_format", ctypes.c_int32),
    ]


class DoryBlockSrc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "wq", "wk", "wv", "wg", "wo", "w_gate", "w_up", "w_down",
        "alpha_attn", "alpha_mlp", "s_qk")]


_LIB = None
P = ctypes.c_void_p
I = ctypes.c_int
SZ = ctypes.c_size_t


def lib():
    """The loaded libdory.so (ImportError when it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "looped_ngpt_transformer_fwd_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        sig = {
            "dory_weight_bytes": (SZ, [P]),
            "dory_create": (I, [P, P, SZ, P, I, P, P]),
            "dory_kv_bytes": (SZ, [P, I, I, I, I]),
            "dory_kv_alloc": (I, [P, I, I, I, I, P, SZ, P]),
            "dory_kv_layout": (I, [P, I, I, I, I, I, P, P]),
            "dory_workspace_bytes": (SZ, [P, I]),
            "dory_prefill": (I, [P, P, I, I, I, P, P, I, P, SZ, P]),
            "dory_decode_step": (I, [P, P, I, P, P, I, P, P, I, P, SZ, P]),
            "dory_decode_step_mixed": (I, [P, P, I, P, P, P, I, I, P, P, P, SZ, P]),
            "dory_device_status": (I, [P, P]),
            "dory_last_call_stats": (I, [P, P, P]),
            "dory_error_string": (ctypes.c_char_p, [I]),
            "dory_kv_free": (None, [P]),
            "dory_destroy": (None, [P]),
            "dory_attention_sublayer": (I, [P, P, I, I, I, I, I, P, P, SZ, P]),
            "dory_mlp_sublayer": (I, [P, I, I, P, P, SZ, P]),
            "dory_gemm_bf16": (I, [P, P, P, I, I, I, P]),
            "dory_gemm_bf16_streamk_workspace_bytes": (SZ, [I]),
            "dory_gemm_bf16_streamk": (I, [P, P, P, I, I, I, P, SZ, P]),
            "dory_debug_stream_k": (I, [P, I]),
            "dory_profile_enable": (I, [P, I]),
            "dory_profile_read": (I, [P, I, P, P]),
            "dory_mlp_sublayer_noalloc": (I, [P, I, I, P, P]),
            "dory_debug_mask_probe": (I, [P, I, P, I]),
            "dory_debug_attention_paths": (I, [P, P]),
            "dory_debug_wait_timeout": (I, [P, ctypes.c_uint32, P]),
            "dory_debug_fused_update": (I, [P, I]),
            "dory_quant_mxfp8": (I, [P, I, I, P, P, P]),
            "dory_mxfp8_scale_bytes": (SZ, [I, I]),
            "dory_gemm_mxfp8_workspace_bytes": (SZ, [I, I, I]),
            "dory_gemm_mxfp8": (I, [P, P, P, I, I, I, I, P, SZ, P]),
            "dory_quant_nvfp4": (I, [P, I, I, ctypes.c_float, P, P, P, P]),
            "dory_nvfp4_scale_bytes": (SZ, [I, I]),
            "dory_gemm_nvfp4_workspace_bytes": (SZ, [I, I, I]),
            "dory_gemm_nvfp4": (I, [P, P, P, I, I, I, ctypes.c_float, ctypes.c_float, I, P, SZ, P]),
            "dory_gemm_bf16_mn": (I, [P, P, P, I, I, I, I, I, P]),
            "dory_mlp_backward_workspace_bytes": (SZ, [P, I]),
            "dory_mlp_sublayer_backward": (I, [P, I, I, P, P, P, P, P, P, P, P, SZ, P]),
            "dory_attention_backward_workspace_bytes": (SZ, [P, I]),
            "dory_last_loop_grad_layout": (SZ, [P, P]),
            "dory_last_loop_backward_workspace_bytes": (SZ, [P, I]),
            "dory_last_loop_backward": (I, [P, P, I, P, P, I, P, P, P, SZ, P, SZ, P]),
            "dory_attention_sublayer_backward": (I, [P, I, I] + [P] * 11 + [SZ, P]),
            "dory_vocab_bytes": (SZ, [P, I]),
            "dory_vocab_create": (I, [P, I, P, P, P, P, SZ, P, P]),
            "dory_embed": (I, [P, P, I, P, P]),
            "dory_lm_head": (I, [P, P, I, P, P]),
            "dory_sample": (I, [P, P, I, ctypes.c_float, ctypes.c_uint32, P, P, P]),
            "dory_vocab_free": (None, [P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def _errstr(status):
    try:
        return lib().dory_error_string(status).decode()
    except ImportError:
        return "?"


def check(status, where):
    if status != DORY_OK:
        raise DoryError(status, where)
    return status


def make_config(cfg, allow_extrapolated_k=False, weight_format="bf16"):
    """dory_config from a config dict (configs/*.json)."""
    return DoryConfig(
        cfg["d_model"], cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"], cfg["d_ff"],
        cfg["n_in_blocks"], cfg["n_rec_blocks"], cfg["n_out_blocks"], cfg["window"],
        cfg["full_period"], float(cfg["rope_base_swa"]), float(cfg["rope_base_full"]),
        float(cfg["softmax_scale"]), float(cfg["gate_scale"]), float(cfg["norm_eps"]),
        1 if allow_extrapolated_k else 0, WEIGHT_FORMATS.get(weight_format, weight_format))


# ----------------------------------------------------------------- thin wrappers
def dory_weight_bytes(cfg_struct):
    return lib().dory_weight_bytes(ctypes.byref(cfg_struct))


def dory_kv_bytes(cfg_struct, mode, max_seqs, max_ctx, k_max):
    return lib().dory_kv_bytes(ctypes.byref(cfg_struct), MODES.get(mode, mode), max_seqs, max_ctx, k_max)


def dory_create(cfg_struct, weight_ptr, weight_bytes, srcs, stream):
    arr = (DoryBlockSrc * len(srcs))(*srcs)
    out = ctypes.c_void_p()
    check(lib().dory_create(ctypes.byref(cfg_struct), weight_ptr, weight_bytes, arr, len(srcs),
                            stream, ctypes.byref(out)), "dory_create")
    return out.value


def dory_kv_alloc(model, mode, max_seqs, max_ctx, k_max, kv_ptr, kv_bytes):
    out = ctypes.c_void_p()
    check(lib().dory_kv_alloc(model, MODES.get(mode, mode), max_seqs, max_ctx, k_max, kv_ptr,
                              kv_bytes, ctypes.byref(out)), "dory_kv_alloc")
    return out.value


def dory_kv_layout(kv, layer, loop, seq, pos, head):
    k_off, v_off = ctypes.c_size_t(), ctypes.c_size_t()
    check(lib().dory_kv_layout(kv, layer, loop, seq, pos, head, ctypes.byref(k_off),
                               ctypes.byref(v_off)), "dory_kv_layout")
    return k_off.value, v_off.value


def dory_workspace_bytes(model, max_tokens):
    return lib().dory_workspace_bytes(model, max_tokens)


def dory_prefill(model, kv, seq, pos0, n_tokens, h_in, h_out, k, ws, ws_bytes, stream):
    return check(lib().dory_prefill(model, kv, seq, pos0, n_tokens, h_in, h_out, k, ws, ws_bytes,
                                    stream), "dory_prefill")


def dory_decode_step(model, kv, batch, d_seq, d_pos, max_pos_hint, h_in, h_out, k, ws, ws_bytes,
                     stream):
    return check(lib().dory_decode_step(model, kv, batch, d_seq, d_pos, max_pos_hint, h_in, h_out,
                                        k, ws, ws_bytes, stream), "dory_decode_step")


def dory_decode_step_mixed(model, kv, batch, d_seq, d_pos, d_k, k_hi, max_pos_hint, h_in, h_out,
                           ws, ws_bytes, stream):
    return check(lib().dory_decode_step_mixed(model, kv, batch, d_seq, d_pos, d_k, k_hi,
                                              max_pos_hint, h_in, h_out, ws, ws_bytes, stream),
                 "dory_decode_step_mixed")


def dory_device_status(model, stream):
    return lib().dory_device_status(model, stream)


def dory_last_call_stats(model):
    a, b = ctypes.c_int(), ctypes.c_int()
    check(lib().dory_last_call_stats(model, ctypes.byref(a), ctypes.byref(b)), "dory_last_call_stats")
    return a.value, b.value


def dory_attention_sublayer(model, kv, layer, loop, seq, pos0, n_rows, h, ws, ws_bytes, stream):
    return check(lib().dory_attention_sublayer(model, kv, layer, loop, seq, pos0, n_rows, h, ws,
                                               ws_bytes, stream), "dory_attention_sublayer")


def dory_mlp_sublayer(model, layer, n_rows, h, ws, ws_bytes, stream):
    return check(lib().dory_mlp_sublayer(model, layer, n_rows, h, ws, ws_bytes, stream),
                 "dory_mlp_sublayer")


def dory_mlp_sublayer_noalloc(model, layer, n_rows, h, stream):
    """dory_mlp_sublayer without a workspace: scratch is the library's static array."""
    return check(lib().dory_mlp_sublayer_noalloc(model, layer, n_rows, h, stream),
                 "dory_mlp_sublayer_noalloc")


def noalloc_max_rows(d_model, d_ff):
    """Largest n_rows dory_mlp_sublayer_noalloc accepts for this shape."""
    def a256(x):
        return (x + 255) // 256 * 256
    n = 0
    while a256(2 * (n + 1) * d_model) + a256(2 * (n + 1) * d_ff) + a256(4 * (n + 1) * d_model) \
            <= NOALLOC_SCRATCH_BYTES:
        n += 1
    return n


def dory_gemm_bf16(A, B, C, M, N, K, stream):
    return check(lib().dory_gemm_bf16(A, B, C, M, N, K, stream), "dory_gemm_bf16")


def dory_gemm_bf16_streamk_workspace_bytes(N):
    return lib().dory_gemm_bf16_streamk_workspace_bytes(N)


def dory_gemm_bf16_streamk(A, B, C, M, N, K, ws, ws_bytes, stream):
    return check(lib().dory_gemm_bf16_streamk(A, B, C, M, N, K, ws, ws_bytes, stream),
                 "dory_gemm_bf16_streamk")


def dory_debug_stream_k(model, enable):
    """Stream-K tails of the prefill projections on or off (default); returns
    the status (DORY_ERR_BAD_CONFIG when the device has more SMs than slots)."""
    return lib().dory_debug_stream_k(model, 1 if enable else 0)


def dory_profile_enable(model, enable):
    return check(lib().dory_profile_enable(model, 1 if enable else 0), "dory_profile_enable")


def dory_profile_read(model, kind):
    """(total ms, launches) of one kernel kind in the last instrumented call."""
    ms, n = ctypes.c_float(), ctypes.c_int()
    kind = KERNEL_KINDS.index(kind) if isinstance(kind, str) else kind
    check(lib().dory_profile_read(model, kind, ctypes.byref(ms), ctypes.byref(n)),
          "dory_profile_read")
    return ms.value, n.value


def dory_debug_mask_probe(model, layer, probe_ptr, max_rows):
    return check(lib().dory_debug_mask_probe(model, layer, probe_ptr, max_rows),
                 "dory_debug_mask_probe")


def dory_debug_attention_paths(model):
    """{kind: launches} of the attention kernels of the most recent call."""
    counts = (ctypes.c_int32 * 4)()
    check(lib().dory_debug_attention_paths(model, counts), "dory_debug_attention_paths")
    return dict(zip(ATTENTION_PATHS, list(counts)))


def dory_debug_wait_timeout(model, limit_us, stream):
    return check(lib().dory_debug_wait_timeout(model, limit_us, stream), "dory_debug_wait_timeout")


def dory_debug_fused_update(model, enable):
    """Fused projection + nGPT update on (default) or off; returns the status
    (DORY_ERR_BAD_CONFIG when the model's d_model has no fused kernel)."""
    return lib().dory_debug_fused_update(model, 1 if enable else 0)


def dory_quant_mxfp8(src, rows, K, codes, scales, stream):
    return check(lib().dory_quant_mxfp8(src, rows, K, codes, scales, stream), "dory_quant_mxfp8")


def dory_mxfp8_scale_bytes(rows, K):
    return lib().dory_mxfp8_scale_bytes(rows, K)


def dory_gemm_mxfp8_workspace_bytes(M, N, K):
    return lib().dory_gemm_mxfp8_workspace_bytes(M, N, K)


def dory_gemm_mxfp8(A, B, C, M, N, K, k_splits, ws, ws_bytes, stream):
    return check(lib().dory_gemm_mxfp8(A, B, C, M, N, K, k_splits, ws, ws_bytes, stream),
                 "dory_gemm_mxfp8")


def dory_gemm_bf16_mn(A, B, C, M, N, K, a_mn, b_mn, stream):
    return check(lib().dory_gemm_bf16_mn(A, B, C, M, N, K, a_mn, b_mn, stream), "dory_gemm_bf16_mn")


def dory_mlp_backward_workspace_bytes(m, n_rows):
    return lib().dory_mlp_backward_workspace_bytes(m, n_rows)


def dory_mlp_sublayer_backward(m, layer, n_rows, h_in, dh_out, dh_in, d_w_gate, d_w_up, d_w_down,
                               d_alpha, ws, ws_bytes, stream):
    return check(lib().dory_mlp_sublayer_backward(m, layer, n_rows, h_in, dh_out, dh_in, d_w_gate,
                                                  d_w_up, d_w_down, d_alpha, ws, ws_bytes, stream),
                 "dory_mlp_sublayer_backward")


def dory_attention_backward_workspace_bytes(m, n_rows):
    return lib().dory_attention_backward_workspace_bytes(m, n_rows)


def dory_attention_sublayer_backward(m, layer, n_rows, h_in, dh_out, dh_in, d_wq, d_wk, d_wv, d_wg,
                                     d_wo, d_alpha, d_s_qk, ws, ws_bytes, stream):
    return check(lib().dory_attention_sublayer_backward(m, layer, n_rows, h_in, dh_out, dh_in, d_wq,
                                                        d_wk, d_wv, d_wg, d_wo, d_alpha, d_s_qk,
                                                        ws, ws_bytes, stream),
                 "dory_attention_sublayer_backward")


GRAD_TENSORS = ("wq", "wk", "wv", "wg", "wo", "w_gate", "w_up", "w_down", "alpha_attn",
                "alpha_mlp", "s_qk")


def dory_last_loop_grad_layout(m, n_trained):
    """(total bytes, [n_trained][11] byte offsets) of the gradient buffer."""
    offs = (ctypes.c_size_t * (n_trained * len(GRAD_TENSORS)))()
    total = lib().dory_last_loop_grad_layout(m, offs)
    return total, [[offs[i * len(GRAD_TENSORS) + t] for t in range(len(GRAD_TENSORS))]
                   for i in range(n_trained)]


def dory_last_loop_backward_workspace_bytes(m, n_rows):
    return lib().dory_last_loop_backward_workspace_bytes(m, n_rows)


def dory_last_loop_backward(m, kv, n_rows, h_in, dh_out, k, h_out, dx, grads, grad_bytes, ws,
                            ws_bytes, stream):
    return check(lib().dory_last_loop_backward(m, kv, n_rows, h_in, dh_out, k, h_out, dx, grads,
                                               grad_bytes, ws, ws_bytes, stream),
                 "dory_last_loop_backward")


def dory_quant_nvfp4(src, rows, K, g, d_g, codes, scales, stream):
    return check(lib().dory_quant_nvfp4(src, rows, K, g, d_g, codes, scales, stream),
                 "dory_quant_nvfp4")


def dory_nvfp4_scale_bytes(rows, K):
    return lib().dory_nvfp4_scale_bytes(rows, K)


def dory_gemm_nvfp4_workspace_bytes(M, N, K):
    return lib().dory_gemm_nvfp4_workspace_bytes(M, N, K)


def dory_gemm_nvfp4(A, B, C, M, N, K, g_a, g_b, k_splits, ws, ws_bytes, stream):
    return check(lib().dory_gemm_nvfp4(A, B, C, M, N, K, g_a, g_b, k_splits, ws, ws_bytes, stream),
                 "dory_gemm_nvfp4")


def dory_vocab_bytes(cfg_struct, vocab):
    return lib().dory_vocab_bytes(ctypes.byref(cfg_struct), vocab)


def dory_vocab_create(model, vocab, emb_in, emb_out, scale, buf, nbytes, stream):
    out = ctypes.c_void_p()
    check(lib().dory_vocab_create(model, vocab, emb_in, emb_out, scale, buf, nbytes, stream,
                                  ctypes.byref(out)), "dory_vocab_create")
    return out.value


def dory_embed(vocab, tokens, n, h_out, stream):
    return check(lib().dory_embed(vocab, tokens, n, h_out, stream), "dory_embed")


def dory_lm_head(vocab, h, n, logits, stream):
    return check(lib().dory_lm_head(vocab, h, n, logits, stream), "dory_lm_head")


def dory_sample(vocab, logits, n, temperature, seed, steps, tokens, stream):
    return check(lib().dory_sample(vocab, logits, n, temperature, seed, steps, tokens, stream),
                 "dory_sample")


def dory_vocab_free(vocab):
    lib().dory_vocab_free(vocab)


def dory_kv_free(kv):
    lib().dory_kv_free(kv)


def dory_destroy(model):
    lib().dory_destroy(model)
