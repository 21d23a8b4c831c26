#!/usr/bin/env python
"""Benchmark of the looped nGPT forward pass on B200 through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one pass of the whole hot path over one batch of synthetic input:
a prefill call (input block, k loops of the shared recurrent block with
re-injection, output block, KV cache writes) or one decode step.  Workloads
(4B-class shapes: d_model 3072, 24/8 heads of 128, MLP 9216, blocks 8/20/8,
SWA:full 3:1 with window 4096, bf16 weights and activations):

  prefill_k2   (default) 1 x 4096 tokens, k = 2, last-loop cache
  prefill_k1   1 x 4096 tokens, k = 1
  decode_k2    64 sequences x 32768 cached positions, last-loop cache, k = 2
  decode_k4_last / decode_k4_per   32 / 8 sequences x 131072 positions, k = 4
  prefill_long 262144 tokens in 8192-token chunks, k = 4, last-loop cache
  prefill_k2_mxfp8 / decode_k2_mxfp8, prefill_k2_nvfp4 / decode_k2_nvfp4
               the prefill_k2 / decode_k2 shapes with MXFP8 or NVFP4 weights and
               projection inputs (block-scaled tensor-core GEMMs)
  train_k2     (extra only) one training step of depth-one truncated
               back-propagation, 1 x 4096 tokens, k = 2

N > 1 runs N independent replicas (one per GPU, no collective on the data
path; the harness only uses a barrier and a max-reduction of the timings).
Rank 0 prints one JSON line.  `--impl reference` times the CPU oracle (the
plain float64 NumPy restatement of the method) on a bounded sample of the same
workload.
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS = {
    "prefill_k2": dict(kind="prefill", tokens=4096, k=2, mode="last_loop", seed=1),
    "prefill_k1": dict(kind="prefill", tokens=4096, k=1, mode="last_loop", seed=1),
    "decode_k2": dict(kind="decode", batch=64, ctx=32768, k=2, mode="last_loop", seed=2),
    "decode_k4_last": dict(kind="decode", batch=32, ctx=131072, k=4, mode="last_loop", seed=3),
    "decode_k4_per": dict(kind="decode", batch=8, ctx=131072, k=4, mode="per_loop", seed=3),
    "prefill_long": dict(kind="prefill_chunked", tokens=262144, chunk=8192, k=4, mode="last_loop",
                         seed=4),
    # the released MXFP8 checkpoint format: MXFP8 weights and projection inputs
    "prefill_k2_mxfp8": dict(kind="prefill", tokens=4096, k=2, mode="last_loop", seed=1,
                             fmt="mxfp8"),
    "decode_k2_mxfp8": dict(kind="decode", batch=64, ctx=32768, k=2, mode="last_loop", seed=2,
                            fmt="mxfp8"),
    # the released NVFP4 checkpoint format: NVFP4 weights and projection inputs
    "prefill_k2_nvfp4": dict(kind="prefill", tokens=4096, k=2, mode="last_loop", seed=1,
                             fmt="nvfp4"),
    "decode_k2_nvfp4": dict(kind="decode", batch=64, ctx=32768, k=2, mode="last_loop", seed=2,
                            fmt="nvfp4"),
    # one training step of depth-one truncated back-propagation: the stack's
    # forward, then the backward through the output block and the final
    # recurrent invocation (an extra workload only)
    "train_k2": dict(kind="train", tokens=4096, k=2, mode="last_loop", seed=1),
}

# DRAM traffic (read + write bytes per launch) of the dominant kernels from
# one ncu capture, valid only while the kernel source is unchanged since.
PROFILED = {
    "gateup": {"traffic": 138575360 + 55643648,
               "source": ("looped_ngpt_transformer_fwd_b200/csrc/gemm_tc.cu",
                          "13f70dca9836ca126719cb6bc46bdcb3bb4102ce")},
    # NVFP4 weights and activations: a different kernel instance, its own capture
    "gateup:nvfp4": {"traffic": 39038464 + 25788672,
                     "source": ("looped_ngpt_transformer_fwd_b200/csrc/gemm_tc.cu",
                                "13f70dca9836ca126719cb6bc46bdcb3bb4102ce")},
    # decode attention: measured (read + write) / algorithmic bytes of the
    # full-layer launch, applied to the step's total KV bytes
    "attn": {"ratio": (1075915520 + 5085440) / 1073758208,
             "source": ("looped_ngpt_transformer_fwd_b200/csrc/attn_decode_tma.cu",
                        "ae876dbfaa034702e200369ffd5e61e734159c4b")},
}


def profiled_traffic(kernel, work=None, fmt=None):
    """DRAM bytes of one launch from a committed ncu capture, or None when the
    kernel's source changed since (or no capture of this weight format exists)."""
    import hashlib
    ent = PROFILED.get(kernel if fmt in (None, "bf16") else f"{kernel}:{fmt}")
    if not ent:
        return None
    path, sha = ent["source"]
    try:
        with open(os.path.join(ROOT, path), "rb") as f:
            if hashlib.sha1(f.read()).hexdigest() != sha:
                return None
    except OSError:
        return None
    if "ratio" in ent:
        return ent["ratio"] * work if work is not None else None
    return ent["traffic"]


PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return PEAKS_FALLBACK, "fallback"


# ----------------------------------------------------------------- algorithmic work
def block_gemm_flops(cfg):
    d, hq, hkv, hd, ff = (cfg["d_model"], cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"],
                          cfg["d_ff"])
    n_qkvg = hq * hd + 2 * hkv * hd + hq
    return 2 * d * (n_qkvg + hq * hd + 2 * ff) + 2 * ff * d


def attn_pairs(cfg, b, T, pos0=0):
    """Unmasked (query, key) pairs of block b for queries pos0..pos0+T-1."""
    full = b % cfg["full_period"] == cfg["full_period"] - 1
    q = np.arange(pos0, pos0 + T, dtype=np.int64)
    if full:
        return int((q + 1).sum())
    return int(np.minimum(q + 1, cfg["window"]).sum())


def stack_blocks(cfg, k):
    n_in, n_rec = cfg["n_in_blocks"], cfg["n_rec_blocks"]
    nb = n_in + n_rec + cfg["n_out_blocks"]
    return list(range(n_in)) + [b for _ in range(k) for b in range(n_in, n_in + n_rec)] + \
        list(range(n_in + n_rec, nb))


def prefill_flops(cfg, T, k, pos0=0):
    per_pair = 4 * cfg["head_dim"] * cfg["n_q_heads"]
    blocks = stack_blocks(cfg, k)
    return sum(block_gemm_flops(cfg) * T + per_pair * attn_pairs(cfg, b, T, pos0) for b in blocks)


def train_flops(cfg, T, k):
    """Algorithmic FLOPs of one truncated training step on a T-token sequence:
    the forward of the whole stack, then for every trained block (the final
    recurrent invocation and the output block) its GEMMs three times (the
    recomputed forward, dgrad and wgrad) and its attention three times (the
    recomputed S and P V; dP, dV, dQ and dK), unmasked pairs only."""
    n_in = cfg["n_in_blocks"]
    nb = n_in + cfg["n_rec_blocks"] + cfg["n_out_blocks"]
    per_pair = 4 * cfg["head_dim"] * cfg["n_q_heads"]
    bwd = sum(3 * block_gemm_flops(cfg) * T + 3 * per_pair * attn_pairs(cfg, b, T)
              for b in range(n_in, nb))
    return prefill_flops(cfg, T, k) + bwd


def decode_kv_bytes(cfg, B, pos, k):
    per_pos = 2 * cfg["n_kv_heads"] * cfg["head_dim"] * 2
    tot = 0
    for b in stack_blocks(cfg, k):
        full = b % cfg["full_period"] == cfg["full_period"] - 1
        keys = pos + 1 if full else min(pos + 1, cfg["window"])
        tot += B * keys * per_pos
    return tot


# ----------------------------------------------------------------- clocks
class ClockSampler:
    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-i",
                 str(self.index), "-lms", "200"], stdout=open(self.path, "w"),
                stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) >= 9:
                    rows.append(f)
        finally:
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ----------------------------------------------------------------- our arm
def fill_decode_cache(model, kv, cfg, seed, ctx, mode, k_max, batch):
    """Seeded cache contents for positions [0, ctx) of every sequence (counter hash)."""
    import torch
    from synthetic.kvfill import kv_values_torch
    from synthetic import block_weights
    nb = cfg["n_in_blocks"] + cfg["n_rec_blocks"] + cfg["n_out_blocks"]
    hkv, hd, W = cfg["n_kv_heads"], cfg["head_dim"], cfg["window"]
    for b in range(nb):
        s_qk = block_weights(cfg, seed, b, names=("s_qk",))["s_qk"]
        full = b % cfg["full_period"] == cfg["full_period"] - 1
        rec = cfg["n_in_blocks"] <= b < cfg["n_in_blocks"] + cfg["n_rec_blocks"]
        loops = range(1, k_max + 1) if (mode == "per_loop" and rec) else [1]
        cap = kv.max_ctx if full else min(W, kv.max_ctx)
        if full:
            slots = torch.arange(ctx, device="cuda")
            positions = slots
        else:
            lo = max(0, ctx - W)
            positions = torch.arange(lo, ctx, device="cuda")
            slots = positions % cap
        for loop in loops:
            for s in range(batch):
                for c0 in range(0, positions.numel(), 16384):   # bounded temporaries
                    pc, sc = positions[c0:c0 + 16384], slots[c0:c0 + 16384]
                    kk, vv = kv_values_torch(seed, b * 16 + (loop - 1), s, pc, hkv, hd, s_qk,
                                             "cuda")
                    for h in range(hkv):
                        kv.entry_view(b, loop, s, h, "k")[sc] = kk[:, h]
                        kv.entry_view(b, loop, s, h, "v")[sc] = vv[:, h]
    torch.cuda.synchronize()


def weight_provider(cfg, seed):
    """Seeded synthetic 4B-class weights (block -> dict), each block drawn once."""
    from synthetic import block_weights
    memo = {}

    def provide(b):
        if b not in memo:
            memo[b] = block_weights(cfg, seed, b)
        return memo[b]
    return provide


def run_ours(args, wl, rank, world, device_index, model=None, prov=None, steps=None,
             warmup=None):
    """Time one workload; `model` / `prov` reuse an existing model (same weights)."""
    import torch
    from looped_ngpt_transformer_fwd_b200 import build as libbuild
    from looped_ngpt_transformer_fwd_b200.model import DoryModel
    from synthetic import load_config, hidden_in

    steps = steps or args.steps
    warmup = warmup or args.warmup
    libbuild.build()
    torch.cuda.set_device(device_index)
    cfg = load_config("dory4b", **block_override(args))
    seed = wl["seed"] + 1000 * rank
    if model is None:
        prov = weight_provider(cfg, wl["seed"])
        model = DoryModel(cfg, prov, device=f"cuda:{device_index}",
                          weight_format=wl.get("fmt", "bf16"))
        if args.fused_update:
            model.fused_update(True)
        if args.stream_k:
            model.stream_k(True)
    k, mode = wl["k"], wl["mode"]
    stream = torch.cuda.current_stream()
    res = {}

    if wl["kind"] == "prefill":
        T = wl["tokens"]
        x = torch.from_numpy(hidden_in(cfg, seed, T).view(np.int16)).view(torch.bfloat16).cuda()
        kv = model.kv_cache(mode, 1, T, k_max=k)
        out = torch.empty_like(x)

        def step():
            model.prefill(kv, x, k, h_out=out)
        units_per_step = T
        flops = prefill_flops(cfg, T, k)
        dom = ("gateup", 2.0 * T * 2 * cfg["d_ff"] * cfg["d_model"], "tensor")
        hin_host = x.cpu().pin_memory()
        hout_host = torch.empty_like(hin_host).pin_memory()

        def e2e_step():
            model.prefill(kv, hin_host, k, h_out=hout_host)
        e2e_bytes = (hin_host.numel() * 2, hout_host.numel() * 2)
        workload = f"dory4b prefill 1x{T} k={k} {mode}"
        extra = {"tokens_per_step": T, "k": k, "kv_mode": mode, "flops_per_step": flops}
    elif wl["kind"] == "decode":
        B, ctx = wl["batch"], wl["ctx"]
        max_ctx = ctx + 64
        kv = model.kv_cache(mode, B, max_ctx, k_max=k)
        fill_decode_cache(model, kv, cfg, wl["seed"], ctx, mode, k, B)
        x = torch.from_numpy(hidden_in(cfg, seed, B).view(np.int16)).view(torch.bfloat16).cuda()
        d_seq = torch.arange(B, dtype=torch.int32, device="cuda")
        d_pos = torch.full((B,), ctx, dtype=torch.int32, device="cuda")
        out = torch.empty_like(x)

        def step():
            # every timed step decodes position ctx again (same work each step)
            model.decode(kv, x, d_seq, d_pos, ctx, k, h_out=out)
        units_per_step = B
        kvb = decode_kv_bytes(cfg, B, ctx, k)
        dom = ("attn", float(kvb), "hbm")
        hin_host = x.cpu().pin_memory()
        hout_host = torch.empty_like(hin_host).pin_memory()

        def e2e_step():
            model.decode(kv, hin_host, d_seq, d_pos, ctx, k, h_out=hout_host)
        e2e_bytes = (hin_host.numel() * 2, hout_host.numel() * 2)
        workload = f"dory4b decode B={B} ctx={ctx} k={k} {mode}"
        extra = {"batch": B, "context": ctx, "k": k, "kv_mode": mode, "kv_bytes_read_per_step": kvb,
                 "kv_footprint_bytes": kv.nbytes}
    else:   # chunked long prefill
        T, C = wl["tokens"], wl["chunk"]
        kv = model.kv_cache(mode, 1, T, k_max=k)
        xs = torch.from_numpy(hidden_in(cfg, seed, T).view(np.int16)).view(torch.bfloat16).cuda()
        out = torch.empty(C, cfg["d_model"], dtype=torch.bfloat16, device="cuda")

        def step():
            for c0 in range(0, T, C):
                model.prefill(kv, xs[c0:c0 + C], k, pos0=c0, h_out=out)
        units_per_step = T
        dom = ("attn", float(sum(4 * cfg["head_dim"] * cfg["n_q_heads"] * attn_pairs(cfg, b, T)
                                 for b in stack_blocks(cfg, k))), "tensor")
        e2e_step = None
        e2e_bytes = (0, 0)
        workload = f"dory4b chunked prefill {T} tokens (chunks of {C}) k={k} {mode}"
        extra = {"tokens_per_step": T, "chunk": C, "k": k, "kv_mode": mode}

    # warm-up (captures graphs)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    status = model.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")
    launches_per_step, sublayers = model.last_call_stats()
    if wl["kind"] == "prefill_chunked":
        launches_per_step *= wl["tokens"] // wl["chunk"]

    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device_index) as clk:
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = e0.elapsed_time(e1) / steps
    ms = reduce_max(ms, world)
    clocks = clk.summary()

    # end to end through the C ABI with pinned host buffers
    e2e = None
    if e2e_step is not None:
        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        e0.record(stream)
        for _ in range(steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = reduce_max(e0.elapsed_time(e1) / steps, world)
        e2e = {"value": units_per_step * world / e2e_ms * 1e3,
               "unit": "tokens/s", "h2d_bytes_per_step": e2e_bytes[0],
               "d2h_bytes_per_step": e2e_bytes[1]}

    # per-kernel device time of the dominant kernel (instrumented replays)
    model.profile(True)
    step()
    torch.cuda.synchronize()
    tot = {kk: [0.0, 0] for kk in ("qkvg", "attn", "oproj", "gateup", "down", "row", "kvcommit")}
    if wl["kind"] == "prefill_chunked":
        # one replay of the whole step, reading every chunk's kernels
        reps = 1
        T, C = wl["tokens"], wl["chunk"]
        for c0 in range(0, T, C):
            model.prefill(kv, xs[c0:c0 + C], k, pos0=c0, h_out=out)
            torch.cuda.synchronize()
            for kk, (t, n) in model.profile_read().items():
                tot[kk][0] += t
                tot[kk][1] += n
    else:
        reps = max(1, min(steps, 5))
        for _ in range(reps):
            step()
            torch.cuda.synchronize()
            for kk, (t, n) in model.profile_read().items():
                tot[kk][0] += t
                tot[kk][1] += n
    model.profile(False)
    kernel_ms = {kk: (v[0] / reps, v[1] // reps) for kk, v in tot.items()}
    dom_name, dom_work, bound = dom
    dom_ms, dom_n = kernel_ms[dom_name]
    res.update(ms=ms, units=units_per_step, clocks=clocks, e2e=e2e, launches=launches_per_step,
               sublayers=sublayers, workload=workload, extra=extra, kernel_ms=kernel_ms,
               dom=(dom_name, dom_work, bound, dom_ms, dom_n))
    res["model"] = model
    res["prov"] = prov
    res["cfg"] = cfg
    return res


def run_train(args, wl, model, device_index, steps, warmup, peaks, peak_src):
    """Time the truncated training step (dory_last_loop_backward) on the 4B
    shapes; the roofline is the whole step's algorithmic FLOPs over its device
    time against the sustained bf16 figure."""
    import torch
    from synthetic import hidden_in
    from synthetic.bf16 import bf16_bits_to_f32
    cfg = model.cfg
    T, k = wl["tokens"], wl["k"]
    h = torch.from_numpy(bf16_bits_to_f32(hidden_in(cfg, wl["seed"], T)).astype(np.float32)).cuda()
    g = torch.Generator(device="cuda").manual_seed(wl["seed"])
    dh = torch.randn(T, cfg["d_model"], device="cuda", generator=g) * 0.1
    kv = model.kv_cache(wl["mode"], 1, T, k_max=k)
    stream = torch.cuda.current_stream()
    out = None
    for _ in range(warmup):
        out = model.last_loop_backward(kv, h, dh, k)
    torch.cuda.synchronize()
    if model.device_status() != 0:
        raise RuntimeError("device status after the training warm-up")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device_index) as clk:
        e0.record(stream)
        for _ in range(steps):
            out = model.last_loop_backward(kv, h, dh, k)
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    flops = train_flops(cfg, T, k)
    achieved = flops / (ms / 1e3) / 1e12
    peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    roof = {"bound": "tensor", "kernel": "whole step (stack forward + truncated backward)",
            "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "peak_source": f"{peak_src} (bf16_tflops_sustained)",
            "frac_of_datasheet": achieved / DATASHEET["tensor"], "traffic": None,
            "work_per_launch": flops, "launches_per_step": 1, "device_ms_per_step": ms}
    grad_bytes = int(out["buffer"].numel())
    del out, kv, h, dh
    return {"tokens_per_s": T / ms * 1e3, "ms_per_step": ms, "steps": steps, "warmup": warmup,
            "workload": f"dory4b training step 1x{T} k={k}: stack forward + depth-one truncated "
                        "backward (final recurrent invocation and output block)",
            "e2e_tokens_per_s": None, "roofline": roof, "clocks": clk.summary(),
            "flops_per_step": flops, "tokens_per_step": T, "gradient_bytes": grad_bytes,
            "dtype": "bf16 operands, fp32 accumulation and gradients", "k": k,
            "kv_mode": wl["mode"]}


def block_override(args):
    if not args.blocks:
        return {}
    i, r, o = (int(v) for v in args.blocks.split(","))
    return {"n_in_blocks": i, "n_rec_blocks": r, "n_out_blocks": o}


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def reduce_max(x, world):
    """Max of x over the ranks (the slowest replica sets the step time)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(units_per_step, ms_per_step_local, world):
    """Whole-job throughput of `world` replicas: every rank's units over the
    slowest rank's step time.  Returns (ms_per_step, units per second)."""
    ms = reduce_max(ms_per_step_local, world)
    return ms, units_per_step * world / ms * 1e3


# ----------------------------------------------------------------- CPU oracle
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


_ORACLE_STATE = {}


def oracle_sample(wl, prov=None, n_blocks=4):
    """Time the float64 oracle on a bounded sample of the workload.

    The sample is the first `n_blocks` blocks of the stack (blocks 0-3: three
    sliding-window blocks and one full block) applied to a few rows of the
    workload; every block application of the stack costs the same for these
    rows, so the time is scaled by (block applications of the step) / n_blocks.
    Weight generation and the materialisation of pre-filled cache entries are
    done before the timer.  Returns (units/s, unit, sample description)."""
    from oracle import Oracle, KVCache, weights_from_generator
    from synthetic import load_config, hidden_in, bf16_bits_to_f32, block_weights
    from synthetic.kvfill import kv_values
    cfg = load_config("dory4b")
    key = wl["seed"]
    if key not in _ORACLE_STATE:
        _ORACLE_STATE.clear()
        _ORACLE_STATE[key] = prov or weights_from_generator(cfg, wl["seed"], cache_blocks=True)
    prov = _ORACLE_STATE[key]
    for b in range(n_blocks):
        prov(b)
    orc = Oracle(cfg, prov)
    k, mode = wl["k"], wl["mode"]
    apps = len(stack_blocks(cfg, k))
    if wl["kind"] in ("prefill", "prefill_chunked"):
        n = 32
        h = bf16_bits_to_f32(hidden_in(cfg, wl["seed"], n)).astype(np.float64)
        cache = KVCache(cfg, mode, k_max=k)
        t0 = time.perf_counter()
        x = h
        for b in range(n_blocks):
            x = orc.block(b, x, 0, 0, 1, cache)
        dt = (time.perf_counter() - t0) * apps / n_blocks
        return n / dt, "tokens/s", (f"{n} prompt tokens through blocks 0-{n_blocks - 1}, time "
                                    f"scaled x{apps}/{n_blocks} to the k={k} stack")
    ctx = wl["ctx"]
    s_qk = {b: block_weights(cfg, wl["seed"], b, names=("s_qk",))["s_qk"] for b in range(n_blocks)}

    def pre(slot, seq, lo, hi):
        return kv_values(wl["seed"], slot, seq, np.arange(lo, hi), cfg["n_kv_heads"],
                         cfg["head_dim"], s_qk[slot // 16])
    cache = KVCache(cfg, mode, k_max=k, prefill=pre, prefilled_len={0: ctx})
    h = bf16_bits_to_f32(hidden_in(cfg, wl["seed"], 1)).astype(np.float64)
    for b in range(n_blocks):          # materialise the pre-filled entries
        orc.block(b, h, ctx, 0, 1, cache)
    t0 = time.perf_counter()
    x = h
    for b in range(n_blocks):
        x = orc.block(b, x, ctx, 0, 1, cache)
    dt = (time.perf_counter() - t0) * apps / n_blocks
    return 1 / dt, "tokens/s", (f"1 sequence, decode of position {ctx} through blocks "
                                f"0-{n_blocks - 1}, time scaled x{apps}/{n_blocks} to the k={k} stack")


# ----------------------------------------------------------------- roofline
DATASHEET = {"tensor": 2250.0, "hbm": 8000.0}    # dense bf16 TFLOP/s, HBM3e GB/s (context only)
DATASHEET_LOWP = {"mxfp8": 4500.0, "nvfp4": 9000.0}   # dense fp8 / fp4 TFLOP/s (context only)
# nominal ratio of a low-precision contraction's peak to bf16's (4.5 / 2.25, 9 / 2.25)
LOWP_RATIO = {"mxfp8": 2.0, "nvfp4": 4.0}


def roofline(res, wl, peaks, peak_src):
    """Roofline of the dominant kernel: algorithmic work of its launches in one
    step over their summed device time (events around every launch)."""
    dom_name, dom_work, bound, dom_ms, dom_n = res["dom"]
    if bound == "tensor":
        achieved = dom_work / (dom_ms / 1e3) / 1e12 if dom_ms > 0 else None
        if wl["kind"] != "prefill_chunked" and dom_ms > 0:
            achieved = dom_work / (dom_ms / dom_n / 1e3) / 1e12   # dom_work is per launch
        peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
        unit, key = "TFLOP/s", "bf16_tflops_sustained"
        fmt = wl.get("fmt")
        if fmt in LOWP_RATIO:
            # fp8 / fp4 contraction: the bf16 figure times the nominal ratio of the peaks
            peak, key = LOWP_RATIO[fmt] * peak, f"bf16_tflops_sustained x {LOWP_RATIO[fmt]:g} ({fmt})"
        per_launch = dom_work if wl["kind"] != "prefill_chunked" else dom_work / max(dom_n, 1)
        traffic = profiled_traffic(dom_name, fmt=fmt)
    else:
        achieved = dom_work / (dom_ms / 1e3) / 1e9 if dom_ms > 0 else None
        peak = peaks["hbm_gbs"]
        unit, key = "GB/s", "hbm_gbs"
        per_launch = dom_work / max(dom_n, 1)
        traffic = profiled_traffic(dom_name, per_launch)
    return {"bound": bound, "kernel": dom_name, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": (achieved / peak) if achieved else None,
            "peak_source": f"{peak_src} ({key})",
            "frac_of_datasheet": (achieved / (DATASHEET_LOWP[wl["fmt"]]
                                              if (bound == "tensor" and wl.get("fmt") in DATASHEET_LOWP)
                                              else DATASHEET[bound])) if achieved else None,
            "traffic": traffic, "work_per_launch": per_launch, "launches_per_step": dom_n,
            "device_ms_per_step": dom_ms}


def footprint_check(cfg, wl):
    """The last-loop cache of the workload's shape is the same size for every k
    and equals the one-loop (per-loop, k_max = 1) size."""
    from looped_ngpt_transformer_fwd_b200 import binding as B
    c = B.make_config(cfg)
    B_, ctx = wl["batch"], wl["ctx"] + 64
    one = B.dory_kv_bytes(c, "per_loop", B_, ctx, 1)
    return all(B.dory_kv_bytes(c, "last_loop", B_, ctx, k) == one for k in (1, 2, 3, 4))


DEFAULT_EXTRAS = ["prefill_k1", "decode_k2", "decode_k4_last", "decode_k4_per",
                  "prefill_k2_mxfp8", "decode_k2_mxfp8", "prefill_k2_nvfp4", "decode_k2_nvfp4",
                  "train_k2"]
DTYPES = {"bf16": "bf16",
          "mxfp8": "mxfp8 (E4M3 x E4M3, E8M0 block scales, fp32 accumulation)",
          "nvfp4": "nvfp4 (E2M1 x E2M1, E4M3 block scales of 16, fp32 tensor scales, "
                   "fp32 accumulation)"}


# ----------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="prefill_k2",
                    choices=sorted(n for n, w in WORKLOADS.items() if w["kind"] != "train"))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--blocks", default=None,
                    help="profiling aid: IN,REC,OUT block counts (same kernel shapes, smaller model)")
    ap.add_argument("--batch", type=int, default=None,
                    help="profiling aid: decode batch override (same per-sequence work)")
    ap.add_argument("--fused-update", action="store_true",
                    help="profiling aid: prefill projections with the nGPT update in their epilogue")
    ap.add_argument("--stream-k", action="store_true",
                    help="profiling aid: stream-K tails in the prefill output / down projections")
    ap.add_argument("--extra-workloads", default="auto",
                    help="comma-separated workloads reported under 'workloads' in the same line; "
                         "'auto' = the k = 1 prefill and the three decode workloads when the "
                         "headline workload runs on one GPU; 'none' = off")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    wl = dict(WORKLOADS[args.workload])
    if args.batch and wl["kind"] == "decode":
        wl["batch"] = args.batch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))

    if args.impl == "reference":
        if rank == 0:
            per_step = []
            for _ in range(args.warmup + args.steps):
                v, unit, sample = oracle_sample(wl)
                per_step.append(v)
            v = statistics.median(per_step[args.warmup:])
            line = {"impl": "reference", "metric": f"{'prefill' if 'prefill' in wl['kind'] else 'decode'} tokens/s",
                    "value": v, "unit": unit, "n_gpus": args.gpus, "steps": args.steps,
                    "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
                    "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                    "config": {"workload": args.workload},
                    "cpu_baseline": {"value": v, "unit": unit, "cores": blas_threads(),
                                     "kind": "oracle", "sample": sample},
                    "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0,
                            "d2h_bytes_per_step": 0}}
            print(json.dumps(line), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
        return

    res = run_ours(args, wl, rank, world, local)
    peaks, peak_src = load_peaks()
    roof = roofline(res, wl, peaks, peak_src)
    cpu = None
    if rank == 0 and not args.no_cpu_baseline and not args.blocks and not args.batch:
        v, u, sample = oracle_sample(wl, res["prov"])
        cpu = {"value": v, "unit": u, "cores": blas_threads(), "kind": "oracle", "sample": sample}

    # the other workloads of the metric (k = 1 prefill, decode at k = 2 and 4 in both
    # cache modes) on the same model, fewer steps each, at N = 1
    extras = {}
    models = {res["model"].weight_format: res["model"]}
    names = [] if args.extra_workloads in ("", "none") else (
        DEFAULT_EXTRAS if args.extra_workloads == "auto" else args.extra_workloads.split(","))
    if args.extra_workloads == "auto" and (world > 1 or args.workload != "prefill_k2"
                                           or args.blocks or args.batch):
        names = []
    for name in names:
        xwl = dict(WORKLOADS[name])
        xsteps = min(args.steps, 10)
        fmt = xwl.get("fmt", "bf16")
        if xwl["kind"] == "train":
            import torch
            extras[name] = run_train(args, xwl, res["model"], local, min(xsteps, 5), args.warmup,
                                     peaks, peak_src)
            torch.cuda.empty_cache()
            continue
        if fmt not in models:
            from looped_ngpt_transformer_fwd_b200.model import DoryModel
            models[fmt] = DoryModel(res["cfg"], res["prov"], device=f"cuda:{local}",
                                    weight_format=fmt)
        r = run_ours(args, xwl, rank, world, local, model=models[fmt], prov=res["prov"],
                     steps=xsteps, warmup=args.warmup)
        entry = {"tokens_per_s": r["units"] * world / r["ms"] * 1e3, "ms_per_step": r["ms"],
                 "steps": xsteps, "warmup": args.warmup, "workload": r["workload"],
                 "e2e_tokens_per_s": r["e2e"]["value"] if r["e2e"] else None,
                 "roofline": roofline(r, xwl, peaks, peak_src),
                 "kernel_ms_per_step": {kk: round(v[0], 4) for kk, v in r["kernel_ms"].items()},
                 "gpu_launches": r["launches"] * xsteps, "clocks": r["clocks"],
                 "weights_seed": WORKLOADS[args.workload]["seed"],
                 "dtype": DTYPES[fmt]}
        entry.update({kk: vv for kk, vv in r["extra"].items() if kk not in ("k", "kv_mode")})
        entry["k"], entry["kv_mode"] = xwl["k"], xwl["mode"]
        if xwl["kind"] == "decode":
            entry["last_loop_footprint_equals_k1"] = footprint_check(r["cfg"], xwl)
        extras[name] = entry
        del r
        import torch
        torch.cuda.empty_cache()

    if rank == 0:
        value = res["units"] * world / res["ms"] * 1e3   # res["ms"] is already the max over ranks
        line = {
            "metric": f"{'prefill' if 'prefill' in wl['kind'] else 'decode'} tokens/s",
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": res["ms"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": DTYPES[wl.get("fmt", "bf16")],
            "data": "synthetic (seeded unit-norm inputs, seeded random 4B-class weights)",
            "config": dict({"workload": res["workload"] + (f" blocks={args.blocks}" if args.blocks else ""),
                            "parallelism": f"replicas x{world}",
                            "l2": "per-step working set (7.9 GB of weights) exceeds the 126 MB L2"},
                           **res["extra"]),
            "roofline": roof,
            "kernel_ms_per_step": {kk: round(v[0], 4) for kk, v in res["kernel_ms"].items()},
            "kernel_ms_source": "CUDA events around every kernel of one instrumented replay of the step",
            "cpu_baseline": cpu,
            "e2e": res["e2e"],
            "gpu_launches": res["launches"] * args.steps,
            "clocks": res["clocks"],
            "sublayer_updates_per_call": res["sublayers"],
        }
        if extras:
            line["workloads"] = extras
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
