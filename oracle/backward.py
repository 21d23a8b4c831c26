"""Backward pass of the MLP and attention sublayers (oracle side).

TEST INFRASTRUCTURE ONLY, like the rest of `oracle/`: only `tests/`,
`__graft_entry__.smoke()` and the CPU legs of `bench.py` may use it.

"Dory1.0-4B: A Looped Normalized-GPT" (ai.info AI summary), Methodology in
Plain English: back-propagation is truncated to depth one, so only the final
recurrent invocation (and the output block after it) is trained; Future
Directions repeats that the recipe trains only that invocation.  The pages
give no formulas for it: the backward is the derivative of the forward the
same page defines.  This module writes out the chain rule of one MLP sublayer,

    g = h Wg^T,  u = h Wu^T,  a = SiLU(s g) * u,  a_hat = Norm(a),
    y = a_hat Wd^T,  y_hat = Norm(y),  z = h + alpha * (y_hat - h),
    h_out = Norm(z)

(s = gate_scale), in float64 NumPy, in the order of the forward reversed.
Every norm step x -> x / |x| has the derivative
    dx = (dx_hat - x_hat * <x_hat, dx_hat>) / |x|,
and SiLU(x) = x sigma(x) has SiLU'(x) = sigma(x) (1 + x (1 - sigma(x))).
Given dL/dh_out it returns dL/dh, dL/dWg, dL/dWu, dL/dWd and dL/dalpha
(summed over the rows).  The attention sublayer of a training sequence
(positions 0..n-1, every key one of the sequence's own) is written out the same
way: projections, RoPE (an orthogonal rotation: its backward is the rotation
by the opposite angle), the per-head norm times s_qk, masked softmax attention
(dS = P * (dP - rowsum(P * dP))), the per-head sigmoid gate, the norm of the
gated output and the nGPT update.  Pinned by central finite differences and by
the closed form of an output gradient along h_out
(tests/test_oracle_backward.py).
"""

import numpy as np

from .ngpt_oracle import is_full_layer, mask_allows, rope, sigmoid


def _norm_backward(x_hat, x_len, dx_hat):
    """Gradient through x -> x / |x| (rows), given x_hat, |x| and dL/dx_hat."""
    return (dx_hat - x_hat * (x_hat * dx_hat).sum(axis=1, keepdims=True)) / x_len


def mlp_sublayer_forward(cfg, W, h):
    """The sublayer's forward with every intermediate the backward needs."""
    eps, s = cfg["norm_eps"], cfg["gate_scale"]
    g = h @ W["w_gate"].T
    u = h @ W["w_up"].T
    sg = sigmoid(s * g)
    act = s * g * sg                                   # SiLU(s g)
    a = act * u
    a_len = np.sqrt(np.maximum((a * a).sum(axis=1, keepdims=True), eps))
    a_hat = a / a_len
    y = a_hat @ W["w_down"].T
    y_len = np.sqrt(np.maximum((y * y).sum(axis=1, keepdims=True), eps))
    y_hat = y / y_len
    alpha = W["alpha_mlp"][None, :]
    z = h + alpha * (y_hat - h)
    z_len = np.sqrt(np.maximum((z * z).sum(axis=1, keepdims=True), eps))
    h_out = z / z_len
    return dict(g=g, u=u, sg=sg, act=act, a_hat=a_hat, a_len=a_len, y_hat=y_hat, y_len=y_len,
                z_len=z_len, h_out=h_out)


def mlp_sublayer_backward(cfg, W, h, dh_out):
    """dL/d(inputs and parameters) of one MLP sublayer given dL/dh_out.

    W: the block's weights as float64 arrays (w_gate, w_up [d_ff, d], w_down
    [d, d_ff], alpha_mlp [d]); h, dh_out: [rows, d].  Returns a dict with
    dh (rows, d), d_w_gate, d_w_up (d_ff, d), d_w_down (d, d_ff), d_alpha (d,),
    and h_out, the forward's output."""
    h = np.asarray(h, dtype=np.float64)
    dh_out = np.asarray(dh_out, dtype=np.float64)
    s = cfg["gate_scale"]
    f = mlp_sublayer_forward(cfg, W, h)
    alpha = W["alpha_mlp"][None, :]
    # h_out = Norm(z)
    dz = _norm_backward(f["h_out"], f["z_len"], dh_out)
    # z = h + alpha (y_hat - h)
    d_alpha = (dz * (f["y_hat"] - h)).sum(axis=0)
    dh = dz * (1.0 - alpha)
    dy_hat = dz * alpha
    # y_hat = Norm(y), y = a_hat Wd^T
    dy = _norm_backward(f["y_hat"], f["y_len"], dy_hat)
    d_w_down = dy.T @ f["a_hat"]
    da_hat = dy @ W["w_down"]
    # a_hat = Norm(a), a = SiLU(s g) u
    da = _norm_backward(f["a_hat"], f["a_len"], da_hat)
    du = da * f["act"]
    dg = da * f["u"] * s * f["sg"] * (1.0 + s * f["g"] * (1.0 - f["sg"]))
    # g = h Wg^T, u = h Wu^T
    d_w_gate = dg.T @ h
    d_w_up = du.T @ h
    dh = dh + dg @ W["w_gate"] + du @ W["w_up"]
    return dict(dh=dh, d_w_gate=d_w_gate, d_w_up=d_w_up, d_w_down=d_w_down, d_alpha=d_alpha,
                h_out=f["h_out"])



def _rows_norm(x, eps):
    return np.sqrt(np.maximum((x * x).sum(axis=-1, keepdims=True), eps))


def attention_sublayer_forward(cfg, W, h, b):
    """Block b's attention sublayer on a training sequence h [n, d] at positions
    0..n-1 (keys: the sequence's own), with every intermediate the backward
    needs.  The same computation as the oracle's attention sublayer."""
    eps = cfg["norm_eps"]
    n, d = h.shape
    hq, hkv, hd = cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    full = is_full_layer(cfg, b)
    base = cfg["rope_base_full"] if full else cfg["rope_base_swa"]
    pos = np.arange(n)
    rq = rope((h @ W["wq"].T).reshape(n, hq, hd), pos, base)
    rk = rope((h @ W["wk"].T).reshape(n, hkv, hd), pos, base)
    v = (h @ W["wv"].T).reshape(n, hkv, hd)
    gate = sigmoid(h @ W["wg"].T)                                     # [n, hq]
    lq, lk = _rows_norm(rq, eps), _rows_norm(rk, eps)
    uq, uk = rq / lq, rk / lk
    q, k = W["s_qk"] * uq, W["s_qk"] * uk
    group = hq // hkv
    Kq, Vq = np.repeat(k, group, axis=1), np.repeat(v, group, axis=1)
    allowed = mask_allows(pos[:, None], pos[None, :], None if full else cfg["window"])
    s = cfg["softmax_scale"] * np.einsum("ihd,jhd->hij", q, Kq)
    s = np.where(allowed[None], s, -np.inf)
    s = s - s.max(axis=-1, keepdims=True)
    P = np.exp(s)
    P /= P.sum(axis=-1, keepdims=True)
    O = np.einsum("hij,jhd->ihd", P, Vq)                             # before the gate
    o = (O * gate[:, :, None]).reshape(n, hq * hd)
    o_len = _rows_norm(o, eps)
    o_hat = o / o_len
    y = o_hat @ W["wo"].T
    y_len = _rows_norm(y, eps)
    y_hat = y / y_len
    z = h + W["alpha_attn"][None, :] * (y_hat - h)
    z_len = _rows_norm(z, eps)
    return dict(base=base, pos=pos, lq=lq, lk=lk, uq=uq, uk=uk, q=q, Kq=Kq, Vq=Vq, gate=gate,
                P=P, O=O, o_hat=o_hat, o_len=o_len, y_hat=y_hat, y_len=y_len, z_len=z_len,
                h_out=z / z_len)


def attention_sublayer_backward(cfg, W, h, dh_out, b):
    """dL/d(inputs and parameters) of block b's attention sublayer on a training
    sequence, given dL/dh_out.  W: wq, wk, wv [*, d], wg [hq, d], wo [d, hq*hd],
    alpha_attn [d], s_qk [hd] as float64.  Returns dh, d_wq, d_wk, d_wv, d_wg,
    d_wo, d_alpha, d_s_qk and h_out."""
    h = np.asarray(h, dtype=np.float64)
    dh_out = np.asarray(dh_out, dtype=np.float64)
    n, d = h.shape
    hq, hkv, hd = cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    group = hq // hkv
    f = attention_sublayer_forward(cfg, W, h, b)
    alpha = W["alpha_attn"][None, :]
    # nGPT update and output projection
    dz = _norm_backward(f["h_out"], f["z_len"], dh_out)
    d_alpha = (dz * (f["y_hat"] - h)).sum(axis=0)
    dh = dz * (1.0 - alpha)
    dy = _norm_backward(f["y_hat"], f["y_len"], dz * alpha)
    d_wo = dy.T @ f["o_hat"]
    do = _norm_backward(f["o_hat"], f["o_len"], dy @ W["wo"]).reshape(n, hq, hd)
    # gate: o = O * gate, gate = sigmoid(h Wg^T)
    dgate = (do * f["O"]).sum(axis=-1)
    dgl = dgate * f["gate"] * (1.0 - f["gate"])
    dO = do * f["gate"][:, :, None]
    # softmax attention (masked entries have P = 0 and get no gradient)
    P = f["P"]
    dP = np.einsum("ihd,jhd->hij", dO, f["Vq"])
    dVq = np.einsum("hij,ihd->jhd", P, dO)
    dS = P * (dP - (P * dP).sum(axis=-1, keepdims=True))
    scale = cfg["softmax_scale"]
    dq = scale * np.einsum("hij,jhd->ihd", dS, f["Kq"])
    dKq = scale * np.einsum("hij,ihd->jhd", dS, f["q"])
    dk = dKq.reshape(n, hkv, group, hd).sum(axis=2)
    dv = dVq.reshape(n, hkv, group, hd).sum(axis=2)
    # q = s_qk * rq / |rq| (per head), rq = RoPE(q_raw); likewise k
    s_qk = W["s_qk"]
    d_s_qk = (dq * f["uq"]).sum(axis=(0, 1)) + (dk * f["uk"]).sum(axis=(0, 1))
    drq = (s_qk * dq - f["uq"] * (f["uq"] * s_qk * dq).sum(axis=-1, keepdims=True)) / f["lq"]
    drk = (s_qk * dk - f["uk"] * (f["uk"] * s_qk * dk).sum(axis=-1, keepdims=True)) / f["lk"]
    dq_raw = rope(drq, -f["pos"], f["base"]).reshape(n, hq * hd)     # the inverse rotation
    dk_raw = rope(drk, -f["pos"], f["base"]).reshape(n, hkv * hd)
    dv_raw = dv.reshape(n, hkv * hd)
    d_wq, d_wk, d_wv, d_wg = dq_raw.T @ h, dk_raw.T @ h, dv_raw.T @ h, dgl.T @ h
    dh = dh + dq_raw @ W["wq"] + dk_raw @ W["wk"] + dv_raw @ W["wv"] + dgl @ W["wg"]
    return dict(dh=dh, d_wq=d_wq, d_wk=d_wk, d_wv=d_wv, d_wg=d_wg, d_wo=d_wo, d_alpha=d_alpha,
                d_s_qk=d_s_qk, h_out=f["h_out"])


# --------------------------------------------------------------- the stack

TENSORS = ("wq", "wk", "wv", "wg", "wo", "w_gate", "w_up", "w_down", "alpha_attn", "alpha_mlp",
           "s_qk")


def _block_weights(provider, b):
    from synthetic.bf16 import bf16_bits_to_f32
    raw = provider(b)
    return {k: (bf16_bits_to_f32(v).astype(np.float64) if v.dtype == np.uint16
                else np.asarray(v, dtype=np.float64)) for k, v in raw.items()}


def _block_forward(cfg, W, h, b):
    h = attention_sublayer_forward(cfg, W, h, b)["h_out"]
    return mlp_sublayer_forward(cfg, W, h)["h_out"]


def trained_part_forward(cfg, provider, x_k):
    """The part of the stack that depth-one truncated back-propagation trains:
    the final recurrent invocation on its input x_k, then the output block.
    Returns the output and the input of every sublayer on the way."""
    n_in, n_rec, n_out = cfg["n_in_blocks"], cfg["n_rec_blocks"], cfg["n_out_blocks"]
    h = np.asarray(x_k, dtype=np.float64)
    saved = []
    for b in range(n_in, n_in + n_rec + n_out):
        W = _block_weights(provider, b)
        saved.append(("att", b, h))
        h = attention_sublayer_forward(cfg, W, h, b)["h_out"]
        saved.append(("mlp", b, h))
        h = mlp_sublayer_forward(cfg, W, h)["h_out"]
    return h, saved


def last_loop_input(cfg, provider, h_in, k):
    """x_k, the input of the final recurrent invocation of a training sequence
    (positions 0..n-1): e = InputBlock(h_in), x_1 = e, x_{j+1} =
    Norm(RecurrentBlock(x_j) + e) ("Dory1.0-4B: A Looped Normalized-GPT",
    Methodology in Plain English: the input block's output is re-injected
    before every pass)."""
    n_in, n_rec = cfg["n_in_blocks"], cfg["n_rec_blocks"]
    h = np.asarray(h_in, dtype=np.float64)
    for b in range(n_in):
        h = _block_forward(cfg, _block_weights(provider, b), h, b)
    e = h
    x = e
    for _ in range(k - 1):
        y = x
        for b in range(n_in, n_in + n_rec):
            y = _block_forward(cfg, _block_weights(provider, b), y, b)
        s = y + e
        x = s / np.sqrt(np.maximum((s * s).sum(axis=1, keepdims=True), cfg["norm_eps"]))
    return x


def last_loop_backward(cfg, provider, h_in, dh_out, k):
    """Depth-one truncated back-propagation through a training sequence's stack
    ("Dory1.0-4B: A Looped Normalized-GPT", Methodology in Plain English: only
    the final recurrent invocation is trained): the loops before the last are
    run forward only, their output x_k is a constant, and dL/dh_out flows back
    through the output block and the final recurrent invocation.  Returns
    h_out, dx (dL/dx_k) and per trained block b a dict of gradients named like
    TENSORS."""
    x_k = last_loop_input(cfg, provider, h_in, k)
    h_out, saved = trained_part_forward(cfg, provider, x_k)
    dh = np.asarray(dh_out, dtype=np.float64)
    grads = {}
    for kind, b, h in reversed(saved):
        W = _block_weights(provider, b)
        gb = grads.setdefault(b, {})
        if kind == "mlp":
            g = mlp_sublayer_backward(cfg, W, h, dh)
            gb.update(w_gate=g["d_w_gate"], w_up=g["d_w_up"], w_down=g["d_w_down"],
                      alpha_mlp=g["d_alpha"])
        else:
            g = attention_sublayer_backward(cfg, W, h, dh, b)
            gb.update(wq=g["d_wq"], wk=g["d_wk"], wv=g["d_wv"], wg=g["d_wg"], wo=g["d_wo"],
                      alpha_attn=g["d_alpha"], s_qk=g["d_s_qk"])
        dh = g["dh"]
    return dict(h_out=h_out, dx=dh, x_k=x_k, grads=grads)
