"""Exact attention masks on the GPU.

Each attention kernel can record, per (row, query head), which keys it gave a
nonzero softmax weight: the first and last such key position, their number
and the sum of their positions (dory_debug_mask_probe).  These tests compare
those records bit for bit with the set of visible keys that the oracle's mask
rule gives (causal; a sliding-window layer sees the last W positions including
the query's own: "Dory1.0-4B: A Looped Normalized-GPT", Methodology in Plain
English), for every attention kernel of the library:
  * tcgen05 prefill attention (head_dim 128, any chunk start and window:
    key tiles across the chunk start or a ring's end are gathered row by row),
  * mma.sync prefill attention (head_dim 64),
  * TMA-fed decode attention (head_dim 128, window a multiple of 64),
  * cp.async decode attention (head_dim 64, or another window),
at windows 1, 4, 100, 128 and 4096, aligned and unaligned chunk starts, and
sliding-window rings that have wrapped.  The kernel that ran is checked with
dory_debug_attention_paths.
"""

import numpy as np
import pytest
import torch

from oracle import mask_allows
from tests.gpu_util import build, inputs

pytestmark = pytest.mark.gpu

SMALL128 = dict(d_model=256, n_q_heads=2, n_kv_heads=1, head_dim=128, d_ff=256,
                n_in_blocks=1, n_rec_blocks=1, n_out_blocks=1, full_period=2,
                softmax_scale=float(np.sqrt(128.0)))
SMALL64 = dict(n_in_blocks=1, n_rec_blocks=1, n_out_blocks=1)


def expected_records(positions, window, n_heads):
    """Brute force over the oracle's mask rule: [rows, heads, 4] int32."""
    out = np.zeros((len(positions), n_heads, 4), np.int64)
    for r, q in enumerate(positions):
        keys = np.arange(0, q + 1)
        vis = keys[mask_allows(q, keys, window)]
        out[r, :] = (vis.min(), vis.max(), len(vis), int(vis.sum()) % (1 << 32))
    out[:, :, 3] = (out[:, :, 3] + (1 << 31)) % (1 << 32) - (1 << 31)   # as int32
    return out.astype(np.int32)


def check(rec, positions, window, n_heads, what):
    got = rec[:len(positions)].cpu().numpy()
    want = expected_records(positions, window, n_heads)
    bad = np.argwhere((got != want).any(-1))
    assert bad.size == 0, (f"{what}: {len(bad)} mismatching (row, head); first "
                           f"row {bad[0][0]} (position {positions[bad[0][0]]}): "
                           f"got {got[tuple(bad[0])]}, want {want[tuple(bad[0])]}")


def run_prefill(model, kv, x, a, b, k=1, seq=0):
    model.prefill(kv, x[a:b], k, seq=seq, pos0=a)
    torch.cuda.synchronize()


def run_decode(model, kv, x, p, k=1, seq=0, max_pos=None):
    d_seq = torch.tensor([seq], dtype=torch.int32, device="cuda")
    d_pos = torch.tensor([p], dtype=torch.int32, device="cuda")
    model.decode(kv, x[p:p + 1], d_seq, d_pos, max_pos if max_pos is not None else kv.max_ctx - 1, k)
    torch.cuda.synchronize()


def expected_paths(cfg, a, decode):
    """Attention kernels a call must use: the library's documented dispatch rule
    applied to every block of the stack."""
    hd, W, nb = cfg["head_dim"], cfg["window"], cfg["n_in_blocks"] + cfg["n_rec_blocks"] + cfg["n_out_blocks"]
    kinds = set()
    for b in range(nb):
        full = b % cfg["full_period"] == cfg["full_period"] - 1
        if decode:
            kinds.add("decode_tma" if hd == 128 and (full or W % 64 == 0) else "decode_cp")
        else:
            kinds.add("prefill_tc" if hd == 128 else "prefill_mma")
    return kinds


def scenario(model, cfg, chunks, decode_positions, max_ctx, layers=(0, 1)):
    """Run the chunks and decode steps once per probed layer; check every record
    and which attention kernels ran."""
    hq, window = cfg["n_q_heads"], cfg["window"]
    n_max = max(b - a for a, b in chunks)
    x, _ = inputs(cfg, 77, max_ctx)
    seen = set()
    for layer in layers:
        full = layer % cfg["full_period"] == cfg["full_period"] - 1
        win = None if full else window
        kv = model.kv_cache("last_loop", 1, max_ctx)
        rec = model.mask_probe(layer, n_max)
        try:
            for a, b in chunks:
                run_prefill(model, kv, x, a, b)
                ran = {k for k, n in model.attention_paths().items() if n > 0}
                assert ran == expected_paths(cfg, a, False), (a, b, ran)
                seen |= ran
                check(rec, list(range(a, b)), win, hq, f"prefill {a}:{b} layer {layer} W={window}")
            for p in decode_positions:
                run_decode(model, kv, x, p)
                ran = {k for k, n in model.attention_paths().items() if n > 0}
                assert ran == expected_paths(cfg, p, True), (p, ran)
                seen |= ran
                check(rec, [p], win, hq, f"decode {p} layer {layer} W={window}")
        finally:
            model.mask_probe_off()
        assert model.device_status() == 0
        kv.free()
    return seen


@pytest.mark.parametrize("window", [128, 4096])
def test_masks_head_dim_128_tensor_core_paths(window):
    """Every chunk runs the tcgen05 prefill kernel (the unaligned ones gather the
    key tile across their start), decode the TMA kernel; with W = 128 the later
    chunks read a wrapped ring."""
    cfg, _, model = build("tiny", seed=3, variant="random", window=window, **SMALL128)
    if window == 128:
        chunks, dec, ctx = [(0, 384), (384, 640), (640, 661), (661, 700)], [700, 701, 765], 800
    else:
        chunks, dec, ctx = [(0, 4608), (4608, 4736), (4736, 4741)], [4741, 4742], 4800
    seen = scenario(model, cfg, chunks, dec, ctx)
    assert {"prefill_tc", "decode_tma"} <= seen
    model.close()


@pytest.mark.parametrize("window", [1, 4, 100])
def test_masks_head_dim_128_other_windows(window):
    """Windows that are not a multiple of 128 nor of 64: prefill stays on the
    tcgen05 kernel (ring tiles that run past the ring's end are gathered), decode
    runs the cp.async kernel; the full layers keep the TMA decode path."""
    cfg, _, model = build("tiny", seed=4, variant="random", window=window, **SMALL128)
    seen = scenario(model, cfg, [(0, 256), (256, 300), (300, 512)], [512, 513], 600)
    assert seen == {"prefill_tc", "decode_tma", "decode_cp"}
    model.close()


@pytest.mark.parametrize("window", [1, 4, 32])
def test_masks_head_dim_64(window):
    """head_dim 64: mma.sync prefill and cp.async decode kernels; rings of 1, 4 and
    32 slots wrap many times."""
    cfg, _, model = build("tiny", seed=5, variant="random", window=window, **SMALL64)
    seen = scenario(model, cfg, [(0, 100), (100, 101), (101, 230)], [230, 231, 232], 256)
    assert seen == {"prefill_mma", "decode_cp"}
    model.close()


def test_probe_records_a_deliberately_narrower_set_as_different():
    """Negative control of the comparison itself: the records of a W = 128 layer
    differ from the brute-force set of W = 127."""
    cfg, _, model = build("tiny", seed=3, variant="random", window=128, **SMALL128)
    x, _ = inputs(cfg, 77, 512)
    kv = model.kv_cache("last_loop", 1, 512)
    rec = model.mask_probe(0, 512)
    run_prefill(model, kv, x, 0, 512)
    model.mask_probe_off()
    got = rec.cpu().numpy()
    assert np.array_equal(got, expected_records(list(range(512)), 128, cfg["n_q_heads"]))
    assert not np.array_equal(got, expected_records(list(range(512)), 127, cfg["n_q_heads"]))
    model.close()
