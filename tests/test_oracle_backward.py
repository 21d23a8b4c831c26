"""Pins of the oracle's MLP-sublayer backward (oracle/backward.py).

Truncated back-propagation of depth one trains only the final recurrent
invocation ("Dory1.0-4B: A Looped Normalized-GPT", Methodology in Plain
English); its sublayers' gradients are derivatives of the forward.  Pinned
against things other than the chain rule it writes out:
  * central finite differences of L = <dh_out, h_out> in every input and
    parameter (float64, step 1e-6);
  * the forward it differentiates is the oracle's MLP sublayer;
  * an output gradient along h_out changes nothing (h_out is a unit vector, so
    L cannot move with its length): every gradient vanishes;
  * gate_scale enters SiLU's argument (a different gate_scale changes dWg).
"""

import numpy as np
import pytest

from oracle import Oracle, weights_from_generator
from oracle.backward import mlp_sublayer_backward, mlp_sublayer_forward
from synthetic import load_config, hidden_in
from synthetic.bf16 import bf16_bits_to_f32


def _setup(seed=3, rows=5, **over):
    cfg = load_config("tiny", **over)
    prov = weights_from_generator(cfg, seed, "random")
    raw = prov(1)
    W = {k: (bf16_bits_to_f32(v).astype(np.float64) if v.dtype == np.uint16
             else np.asarray(v, dtype=np.float64)) for k, v in raw.items()}
    h = bf16_bits_to_f32(hidden_in(cfg, seed + 1, rows)).astype(np.float64)
    rng = np.random.default_rng(seed + 2)
    dh_out = rng.standard_normal(h.shape)
    return cfg, prov, W, h, dh_out


def _loss(cfg, W, h, dh_out):
    return float((mlp_sublayer_forward(cfg, W, h)["h_out"] * dh_out).sum())


def test_forward_is_the_oracle_mlp_sublayer():
    cfg, prov, W, h, _ = _setup()
    ref = Oracle(cfg, prov).mlp_sublayer(1, h)
    assert np.allclose(mlp_sublayer_forward(cfg, W, h)["h_out"], ref, rtol=0, atol=1e-14)


@pytest.mark.parametrize("name", ["h", "w_gate", "w_up", "w_down", "alpha_mlp"])
def test_gradients_match_central_differences(name):
    cfg, _, W, h, dh_out = _setup(d_model=128, n_q_heads=2, d_ff=256)
    g = mlp_sublayer_backward(cfg, W, h, dh_out)
    grad = {"h": g["dh"], "w_gate": g["d_w_gate"], "w_up": g["d_w_up"], "w_down": g["d_w_down"],
            "alpha_mlp": g["d_alpha"]}[name]
    rng = np.random.default_rng(7)
    eps = 1e-6
    target = h if name == "h" else W[name]
    idx = [tuple(rng.integers(0, n) for n in target.shape) for _ in range(12)]
    for ix in idx:
        old = target[ix]
        target[ix] = old + eps
        lp = _loss(cfg, W, h, dh_out)
        target[ix] = old - eps
        lm = _loss(cfg, W, h, dh_out)
        target[ix] = old
        fd = (lp - lm) / (2 * eps)
        assert abs(fd - grad[ix]) <= 1e-6 * max(1.0, abs(fd)), (name, ix, fd, grad[ix])


def test_gradient_along_the_output_vanishes():
    cfg, _, W, h, _ = _setup()
    h_out = mlp_sublayer_forward(cfg, W, h)["h_out"]
    g = mlp_sublayer_backward(cfg, W, h, 3.0 * h_out)
    for k in ("dh", "d_w_gate", "d_w_up", "d_w_down", "d_alpha"):
        assert np.abs(g[k]).max() < 1e-12, k


def test_gate_scale_reaches_the_gate_gradient():
    cfg, _, W, h, dh_out = _setup()
    g1 = mlp_sublayer_backward(cfg, W, h, dh_out)["d_w_gate"]
    g2 = mlp_sublayer_backward(dict(cfg, gate_scale=2.0), W, h, dh_out)["d_w_gate"]
    assert np.abs(g1 - g2).max() > 1e-3 * np.abs(g1).max()


# ------------------------------------------------------------------ attention

def _att_setup(seed=11, rows=9, layer=1, **over):
    over = dict(dict(d_model=64, n_q_heads=4, n_kv_heads=2, head_dim=16, d_ff=128, window=4), **over)
    cfg = load_config("tiny", **over)
    prov = weights_from_generator(cfg, seed, "random")
    raw = prov(layer)
    W = {k: (bf16_bits_to_f32(v).astype(np.float64) if v.dtype == np.uint16
             else np.asarray(v, dtype=np.float64)) for k, v in raw.items()}
    h = bf16_bits_to_f32(hidden_in(cfg, seed + 1, rows)).astype(np.float64)
    dh_out = np.random.default_rng(seed + 2).standard_normal(h.shape)
    return cfg, prov, W, h, dh_out


@pytest.mark.parametrize("layer", [0, 1])   # sliding window (W = 4), full
def test_attention_forward_is_the_oracle_sublayer(layer):
    from oracle import KVCache
    from oracle.backward import attention_sublayer_forward
    cfg, prov, W, h, _ = _att_setup(layer=layer)
    ref = Oracle(cfg, prov).attention_sublayer(layer, h, 0, 0, 1, KVCache(cfg, "last_loop"))
    assert np.allclose(attention_sublayer_forward(cfg, W, h, layer)["h_out"], ref, rtol=0, atol=1e-13)


@pytest.mark.parametrize("layer", [0, 1])
@pytest.mark.parametrize("name", ["h", "wq", "wk", "wv", "wg", "wo", "alpha_attn", "s_qk"])
def test_attention_gradients_match_central_differences(layer, name):
    from oracle.backward import attention_sublayer_backward, attention_sublayer_forward
    cfg, _, W, h, dh_out = _att_setup(layer=layer)
    g = attention_sublayer_backward(cfg, W, h, dh_out, layer)
    key = {"h": "dh", "alpha_attn": "d_alpha", "s_qk": "d_s_qk"}.get(name, "d_" + name)
    grad = g[key]
    target = h if name == "h" else W[name]
    loss = lambda: float((attention_sublayer_forward(cfg, W, h, layer)["h_out"] * dh_out).sum())
    rng = np.random.default_rng(13)
    eps = 1e-6
    for _ in range(10):
        ix = tuple(rng.integers(0, n) for n in target.shape)
        old = target[ix]
        target[ix] = old + eps
        lp = loss()
        target[ix] = old - eps
        lm = loss()
        target[ix] = old
        fd = (lp - lm) / (2 * eps)
        assert abs(fd - grad[ix]) <= 1e-6 * max(1.0, abs(fd)), (name, ix, fd, grad[ix])


def test_attention_gradient_along_the_output_vanishes():
    from oracle.backward import attention_sublayer_backward, attention_sublayer_forward
    cfg, _, W, h, _ = _att_setup()
    h_out = attention_sublayer_forward(cfg, W, h, 1)["h_out"]
    g = attention_sublayer_backward(cfg, W, h, -2.0 * h_out, 1)
    for k in ("dh", "d_wq", "d_wk", "d_wv", "d_wg", "d_wo", "d_alpha", "d_s_qk"):
        assert np.abs(g[k]).max() < 1e-12, k


# ------------------------------------------------------------------ the stack

def _stack_setup(seed=21, rows=10):
    cfg = load_config("tiny", d_model=64, n_q_heads=4, n_kv_heads=2, head_dim=16, d_ff=128,
                      window=4, n_in_blocks=1, n_rec_blocks=2, n_out_blocks=1)
    prov = weights_from_generator(cfg, seed, "random")
    h = bf16_bits_to_f32(hidden_in(cfg, seed + 1, rows)).astype(np.float64)
    dh_out = np.random.default_rng(seed + 2).standard_normal(h.shape)
    return cfg, prov, h, dh_out


def test_stack_forward_is_the_oracle_stack():
    from oracle import KVCache
    from oracle.backward import last_loop_backward
    cfg, prov, h, dh_out = _stack_setup()
    got = last_loop_backward(cfg, prov, h, dh_out, 3)["h_out"]
    ref = Oracle(cfg, prov).forward(h, 0, 3, KVCache(cfg, "last_loop", k_max=3))
    assert np.allclose(got, ref, rtol=0, atol=1e-12)


def test_last_loop_gradients_match_truncated_differences():
    """Finite differences of L = <dh_out, output> with the final invocation's
    input x_k held fixed (the truncation): for x_k itself and for a parameter
    of every trained block (the shared recurrent weights change only the final
    invocation here)."""
    from oracle.backward import last_loop_backward, trained_part_forward
    cfg, prov, h, dh_out = _stack_setup()
    res = last_loop_backward(cfg, prov, h, dh_out, 2)
    x_k = res["x_k"]
    rng = np.random.default_rng(9)
    eps = 1e-6

    def loss(p, xk):
        return float((trained_part_forward(cfg, p, xk)[0] * dh_out).sum())
    for _ in range(6):
        ix = tuple(rng.integers(0, n) for n in x_k.shape)
        xp, xm = x_k.copy(), x_k.copy()
        xp[ix] += eps
        xm[ix] -= eps
        fd = (loss(prov, xp) - loss(prov, xm)) / (2 * eps)
        assert abs(fd - res["dx"][ix]) <= 1e-6 * max(1.0, abs(fd))
    for b in res["grads"]:
        for name in ("wq", "w_down", "alpha_attn", "s_qk"):
            base = prov(b)[name]
            ix = tuple(rng.integers(0, n) for n in base.shape)

            def bumped(delta):
                def p(bb):
                    w = dict(prov(bb))
                    if bb == b:
                        arr = (bf16_bits_to_f32(w[name]).astype(np.float64) if w[name].dtype == np.uint16
                               else np.asarray(w[name], dtype=np.float64)).copy()
                        arr[ix] += delta
                        w[name] = arr
                    return w
                return p
            fd = (loss(bumped(eps), x_k) - loss(bumped(-eps), x_k)) / (2 * eps)
            assert abs(fd - res["grads"][b][name][ix]) <= 1e-6 * max(1.0, abs(fd)), (b, name)
