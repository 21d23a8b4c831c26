"""Plain float64 NumPy oracle of the looped nGPT forward pass (prefill and decode).

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
CPU-baseline legs of bench.py, never by the product path.

Sources (web pages on Dory1.0-4B; cited by title and section):
  [P1] "Dory1.0-4B: A Looped Normalized-GPT" (ai.info AI summary of the paper)
  [P4] "Dory 1.0 4B Benchmarks: How Do 1, 2 and 4 Loops Compare?" (goremy.ai)
  [P5] "NVIDIA Nemotron Labs Dory 1.0 4B: a looped (latent-recurrent) LLM with
       elastic inference compute" (observer.broadside.tech card), which cites
       "nGPT: Normalized Transformer with Representation Learning on the
       Hypersphere" for the backbone.

What the method computes, step by step (each function below cites its step):
  * nGPT backbone: every hidden state lives on the unit sphere; each sublayer
    updates  h <- Norm(h + alpha * (Norm(f(h)) - h))  with learned per-channel
    alpha ([P1] Methodology in Plain English).
  * attention sublayer: grouped-query attention with input-dependent sigmoid
    output gates; sliding-window and full layers interleaved 3:1; RoPE; the
    concatenated gated output is L2-normalised before the output projection
    ([P1] Methodology in Plain English).
  * MLP sublayer: SwiGLU; the activations are L2-normalised before the
    down-projection ([P1] Methodology in Plain English).
  * stack: input block once, shared recurrent block k times with the input
    block's fixed output re-injected before every pass and the recurrent
    output L2-normalised, output block once ([P1] Key Contributions item 1 and
    Methodology; [P4] What is Dory1.0-4B?; [P5] Key ideas).
  * KV caching: per-loop (one cache per loop) or last-loop (one cache per
    recurrent attention layer, each loop overwriting the previous one)
    ([P4] How does looping work at inference time?; [P5] Key ideas).

Readings where the pages are silent (fixed in the committed configs):
  Norm(x) = x / sqrt(max(sum x^2, norm_eps)); RoPE pairs (i, i + hd/2) with
  theta_i = base^(-2i/hd); q and k are RoPE-rotated, L2-normalised per head and
  scaled by s_qk; logits = softmax_scale * q.k with softmax_scale = sqrt(hd);
  the SWA window holds exactly W keys including the query's own position; the
  output gate is one sigmoid per query head; SwiGLU is SiLU(gate_scale * h Wg^T)
  * (h Wu^T); re-injection is x_j = Norm(y_{j-1} + e) with y_0 = e; under
  last-loop caching, the tokens of one call at loop j attend to earlier
  positions' cached entries and to this call's own loop-j entries.

Parity status: the real checkpoint's numerics are unpinned (no weights and no
activations are published); every function here is pinned by closed forms,
invariants and brute-force checks in tests/test_oracle_pins.py.
"""

import numpy as np

from synthetic import bf16_bits_to_f32, block_weights


# --------------------------------------------------------------------------
# elementary operations
# --------------------------------------------------------------------------

def l2norm(x, eps=1e-20, axis=-1):
    """Norm(x) = x / ||x||_2 along `axis` ([P1] Methodology: everything is L2-normalised)."""
    ss = np.sum(x * x, axis=axis, keepdims=True)
    return x / np.sqrt(np.maximum(ss, eps))


def rope(x, positions, base):
    """Rotary position embedding on the last axis ([P1] Methodology: RoPE base per layer type).

    x: [n, heads, hd]; positions: [n] absolute positions.  Dimension i pairs
    with i + hd/2 and is rotated by the angle p * base^(-2i/hd).
    """
    hd = x.shape[-1]
    half = hd // 2
    inv_freq = base ** (-(2.0 * np.arange(half, dtype=np.float64)) / hd)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv_freq[None, :]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def mask_allows(q_pos, k_pos, window=None):
    """Whether the key at position k_pos is visible to the query at q_pos: causal
    (k_pos <= q_pos) and, in a sliding-window layer, among the last `window`
    positions up to and including the query's own ([P1] Methodology in Plain
    English: sliding-window and full-attention layers; the window holds
    exactly W keys).  Works elementwise on arrays; window None = full layer."""
    q_pos = np.asarray(q_pos)
    k_pos = np.asarray(k_pos)
    ok = k_pos <= q_pos
    if window is not None:
        ok = ok & (q_pos - k_pos < window)
    return ok


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def silu(x):
    return x * sigmoid(x)


# --------------------------------------------------------------------------
# stack structure
# --------------------------------------------------------------------------

def is_full_layer(cfg, b):
    """Global block b uses full attention iff b mod P == P-1 (P = 4: three SWA
    blocks then one full block, [P1] Methodology in Plain English)."""
    p = cfg["full_period"]
    return (b % p) == p - 1


def block_role(cfg, b):
    """'input', 'recurrent' or 'output' for global block index b ([P4] What is Dory1.0-4B?)."""
    if b < cfg["n_in_blocks"]:
        return "input"
    if b < cfg["n_in_blocks"] + cfg["n_rec_blocks"]:
        return "recurrent"
    return "output"


def layer_applications(cfg, k):
    """Sublayer applications per token: 2 * (in + k * rec + out) ([P1] Key Contributions 1)."""
    return 2 * (cfg["n_in_blocks"] + k * cfg["n_rec_blocks"] + cfg["n_out_blocks"])


def kv_cache_bytes(cfg, mode, max_seqs, max_ctx, k_max):
    """Device bytes of a bf16 KV cache under `mode` ('per_loop' or 'last_loop').

    One cache per attention layer, except that recurrent layers keep k_max
    caches under per-loop caching ([P4] How does looping work at inference
    time?).  A sliding-window layer stores min(window, max_ctx) positions, a
    full layer max_ctx; each position holds K and V for all KV heads in bf16.
    """
    nb = cfg["n_in_blocks"] + cfg["n_rec_blocks"] + cfg["n_out_blocks"]
    per_pos = 2 * cfg["n_kv_heads"] * cfg["head_dim"] * 2
    total = 0
    for b in range(nb):
        loops = k_max if (mode == "per_loop" and block_role(cfg, b) == "recurrent") else 1
        cap = max_ctx if is_full_layer(cfg, b) else min(cfg["window"], max_ctx)
        total += loops * max_seqs * cap * per_pos
    return total


# --------------------------------------------------------------------------
# weights
# --------------------------------------------------------------------------

def weights_from_generator(cfg, seed, variant="default", cache_blocks=True):
    """Weight provider reading the shared synthetic generator (bf16 values held exactly)."""
    memo = {}

    def provide(b):
        if b in memo:
            return memo[b]
        w = block_weights(cfg, seed, b, variant)
        if cache_blocks:
            memo[b] = w
        return w
    return provide


def _as_float(w, dtype):
    if w.dtype == np.uint16:
        return bf16_bits_to_f32(w).astype(dtype)
    return np.asarray(w, dtype=dtype)


# --------------------------------------------------------------------------
# KV cache
# --------------------------------------------------------------------------

class KVCache:
    """KV cache of the oracle, addressed by (block, loop, sequence, position).

    Entries hold k-hat (post-RoPE, post-norm, post-s_qk) and v.  Positions a
    sequence had before the oracle saw it may come from `prefill`, a callable
    (slot_id, seq, lo, hi) -> (K, V) float arrays [hi-lo, n_kv, hd], held in
    float32 (the filled contents are bf16 values); any other read of a position
    never written raises KeyError.

    Slot ids: block * 16 + loop slot, where the loop slot is (loop - 1) for a
    recurrent block under per-loop caching and 0 otherwise ([P5] Key ideas:
    last-loop mode overwrites the previous loop's entries).
    """

    def __init__(self, cfg, mode, k_max=1, prefill=None, prefilled_len=None):
        if mode not in ("per_loop", "last_loop"):
            raise ValueError(mode)
        self.cfg, self.mode, self.k_max = cfg, mode, k_max
        self.prefill = prefill
        self.prefilled_len = dict(prefilled_len or {})  # seq -> n cached positions
        self._pre = {}      # (slot, seq) -> (lo, K, V) materialised prefilled range
        self._new = {}      # (slot, seq) -> {pos: (k, v)}

    def slot_id(self, b, loop):
        if self.mode == "per_loop" and block_role(self.cfg, b) == "recurrent":
            if not 1 <= loop <= self.k_max:
                raise ValueError(f"loop {loop} outside 1..k_max={self.k_max}")
            return b * 16 + (loop - 1)
        return b * 16

    def slot_ids(self):
        nb = self.cfg["n_in_blocks"] + self.cfg["n_rec_blocks"] + self.cfg["n_out_blocks"]
        out = []
        for b in range(nb):
            loops = (range(1, self.k_max + 1)
                     if self.mode == "per_loop" and block_role(self.cfg, b) == "recurrent" else [1])
            out.extend(self.slot_id(b, j) for j in loops)
        return out

    def write(self, b, loop, seq, pos0, k, v):
        d = self._new.setdefault((self.slot_id(b, loop), seq), {})
        for i in range(k.shape[0]):
            d[pos0 + i] = (k[i], v[i])

    def read(self, b, loop, seq, lo, hi, dtype=np.float64):
        """K, V for positions [lo, hi) of one sequence: arrays [hi-lo, n_kv, hd]."""
        slot = self.slot_id(b, loop)
        npre = self.prefilled_len.get(seq, 0)
        new = self._new.get((slot, seq), {})
        ks, vs = [], []
        p = lo
        if lo < npre:
            # positions written by this oracle override prefilled ones
            top = min(hi, npre)
            pk, pv = self._prefilled(slot, seq, lo, top)
            pk, pv = pk.astype(dtype), pv.astype(dtype)
            for i in range(top - lo):
                if lo + i in new:
                    pk[i], pv[i] = new[lo + i]
            ks.append(pk)
            vs.append(pv)
            p = top
        if p < hi:
            try:
                ks.append(np.stack([new[q][0] for q in range(p, hi)]).astype(dtype))
                vs.append(np.stack([new[q][1] for q in range(p, hi)]).astype(dtype))
            except KeyError as err:
                raise KeyError(f"read of unwritten position {err} (slot {slot}, seq {seq})") from None
        if not ks:
            shape = (0, self.cfg["n_kv_heads"], self.cfg["head_dim"])
            return np.zeros(shape, dtype), np.zeros(shape, dtype)
        return np.concatenate(ks), np.concatenate(vs)

    def _prefilled(self, slot, seq, lo, hi):
        if self.prefill is None:
            raise KeyError(f"position {lo} of seq {seq} was never written")
        got = self._pre.get((slot, seq))
        if got is None or not (got[0] <= lo and hi <= got[0] + got[1].shape[0]):
            npre = self.prefilled_len[seq]
            b = slot // 16
            span_lo = 0 if is_full_layer(self.cfg, b) else max(0, npre - self.cfg["window"])
            span_lo = min(span_lo, lo)
            k, v = self.prefill(slot, seq, span_lo, npre)
            got = (span_lo, np.asarray(k, np.float32), np.asarray(v, np.float32))
            self._pre[(slot, seq)] = got
        off = lo - got[0]
        return got[1][off:off + hi - lo].copy(), got[2][off:off + hi - lo].copy()


# --------------------------------------------------------------------------
# the model
# --------------------------------------------------------------------------

class Oracle:
    """Looped nGPT forward pass in float64.

    weights: callable b -> dict of the block's tensors in the synthetic
    generator's format (matrices as bf16 bits or floats [out, in]; alpha_attn,
    alpha_mlp [d]; s_qk [hd]).
    """

    def __init__(self, cfg, weights, dtype=np.float64, on_state=None, act_quant=None):
        self.cfg = cfg
        self.weights = weights
        self.dt = dtype
        self.on_state = on_state          # optional hook(h) after every sublayer
        # optional x -> Q(x) applied to every projection's input (quantised
        # checkpoints: MXFP8 activations, see oracle.quant.mxfp8_fake_quant)
        self.act_quant = act_quant
        self.sublayer_apps = 0
        self.q_block = 128                # queries per softmax batch (memory only)

    # -- helpers ---------------------------------------------------------
    def _w(self, b, names):
        raw = self.weights(b)
        return {name: _as_float(raw[name], self.dt) for name in names}

    def _act(self, x):
        return x if self.act_quant is None else self.act_quant(x)

    def _norm(self, x, axis=-1):
        return l2norm(x, self.cfg["norm_eps"], axis)

    def _ngpt_update(self, h, y, alpha):
        """h <- Norm(h + alpha * (Norm(y) - h))  ([P1] Methodology, nGPT residual)."""
        h = self._norm(h + alpha[None, :] * (self._norm(y) - h))
        self.sublayer_apps += 1
        if self.on_state is not None:
            self.on_state(h)
        return h

    # -- sublayers -------------------------------------------------------
    def attention_sublayer(self, b, h, pos0, seq, loop, cache):
        """Gated GQA attention sublayer of block b on rows h [n, d] at positions pos0.. .

        [P1] Methodology in Plain English: GQA with sigmoid output gates,
        SWA (window W, RoPE base rope_base_swa) or full attention (rope_base_full),
        L2 norm of the concatenated gated output before the output projection.
        """
        cfg = self.cfg
        W = self._w(b, ("wq", "wk", "wv", "wg", "wo", "alpha_attn", "s_qk"))
        n, d = h.shape
        hq, hkv, hd = cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"]
        full = is_full_layer(cfg, b)
        base = cfg["rope_base_full"] if full else cfg["rope_base_swa"]
        positions = pos0 + np.arange(n)

        hx = self._act(h)                                            # projection input
        q = (hx @ W["wq"].T).reshape(n, hq, hd)
        k = (hx @ W["wk"].T).reshape(n, hkv, hd)
        v = (hx @ W["wv"].T).reshape(n, hkv, hd)
        gate = sigmoid(hx @ W["wg"].T)                               # [n, hq]
        q = W["s_qk"] * self._norm(rope(q, positions, base))
        k = W["s_qk"] * self._norm(rope(k, positions, base))

        cache.write(b, loop, seq, pos0, k, v)
        win = None if full else cfg["window"]
        lo = 0 if full else max(0, pos0 - win + 1)
        K, V = cache.read(b, loop, seq, lo, pos0 + n, self.dt)     # [L, hkv, hd]
        kpos = np.arange(lo, pos0 + n)
        group = hq // hkv
        Kq = np.repeat(K, group, axis=1)                             # [L, hq, hd]
        Vq = np.repeat(V, group, axis=1)

        o = np.empty((n, hq, hd), dtype=self.dt)
        for i0 in range(0, n, self.q_block):
            i1 = min(n, i0 + self.q_block)
            qp = positions[i0:i1]
            s = cfg["softmax_scale"] * np.einsum("ihd,jhd->hij", q[i0:i1], Kq)
            allowed = mask_allows(qp[:, None], kpos[None, :], win)
            s = np.where(allowed[None, :, :], s, -np.inf)
            s = s - s.max(axis=-1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=-1, keepdims=True)
            o[i0:i1] = np.einsum("hij,jhd->ihd", p, Vq)
        o = o * gate[:, :, None]
        o_hat = self._norm(o.reshape(n, hq * hd))
        y = self._act(o_hat) @ W["wo"].T
        return self._ngpt_update(h, y, W["alpha_attn"])

    def mlp_sublayer(self, b, h):
        """SwiGLU sublayer with L2-normalised activations before the down-projection
        ([P1] Methodology in Plain English)."""
        W = self._w(b, ("w_gate", "w_up", "w_down", "alpha_mlp"))
        hx = self._act(h)
        a = silu(self.cfg["gate_scale"] * (hx @ W["w_gate"].T)) * (hx @ W["w_up"].T)
        y = self._act(self._norm(a)) @ W["w_down"].T
        return self._ngpt_update(h, y, W["alpha_mlp"])

    def block(self, b, h, pos0, seq, loop, cache):
        h = self.attention_sublayer(b, h, pos0, seq, loop, cache)
        return self.mlp_sublayer(b, h)

    # -- the stack ---------------------------------------------------------
    def forward(self, h_in, pos0, k, cache, seq=0):
        """One prefill call (chunk) of one sequence: rows h_in [n, d] at positions pos0.. .

        Input block once, recurrent block k times with re-injection of the
        input block's output before every pass, output block once
        ([P1] Key Contributions 1, Methodology; [P4] What is Dory1.0-4B?).
        """
        cfg = self.cfg
        n_in, n_rec = cfg["n_in_blocks"], cfg["n_rec_blocks"]
        nb = n_in + n_rec + cfg["n_out_blocks"]
        x = np.asarray(h_in, dtype=self.dt)
        for b in range(n_in):
            x = self.block(b, x, pos0, seq, 1, cache)
        e = x
        y = e
        for j in range(1, k + 1):
            x = self._norm(y + e)                       # re-injection before the pass
            for b in range(n_in, n_in + n_rec):
                x = self.block(b, x, pos0, seq, j, cache)
            y = x
        x = y
        for b in range(n_in + n_rec, nb):
            x = self.block(b, x, pos0, seq, 1, cache)
        return x

    def decode(self, h_in, seqs, positions, k, cache):
        """One decode step for a batch: row i is sequence seqs[i] at position positions[i].

        Each sequence is independent; a decode step is a one-token call.
        """
        out = np.empty((len(seqs), self.cfg["d_model"]), dtype=self.dt)
        for i, (s, p) in enumerate(zip(seqs, positions)):
            out[i] = self.forward(np.asarray(h_in[i:i + 1]), int(p), k, cache, int(s))[0]
        return out
