"""Backward pass of the MLP sublayer (oracle side).

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
(summed over the rows).  Pinned by central finite differences and by the
closed form of an output gradient along h_out (tests/test_oracle_backward.py).
"""

import numpy as np

from .ngpt_oracle import sigmoid


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

