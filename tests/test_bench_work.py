"""Host logic of bench.py: the algorithmic work behind every roofline figure.

The benchmark divides FLOPs (prefill) or bytes (decode) per step by measured
time, so these counts are pinned here against independent sources: the
shapes of the generated weight matrices, brute-force counts of the masked
(query, key) pairs with the oracle's layer types, and the closed forms the
targets were set from (depth 32 + 40k sublayers, "Dory1.0-4B: A Looped
Normalized-GPT", Key Contributions 1).  No GPU needed.
"""

import numpy as np
import pytest

import bench
from oracle import is_full_layer, layer_applications
from synthetic import load_config
from synthetic.weights import matrix_shapes


def _gemm_flops_from_shapes(cfg):
    # every weight matrix [out, in] is one GEMM per token: 2 * out * in FLOPs
    return sum(2 * o * i for (o, i) in matrix_shapes(cfg).values())


@pytest.mark.parametrize("name", ["tiny", "dory4b"])
def test_block_gemm_flops_match_the_weight_shapes(name):
    cfg = load_config(name)
    assert bench.block_gemm_flops(cfg) == _gemm_flops_from_shapes(cfg)


def test_4b_gemm_flops_per_token_and_block():
    # 2·d·(q + k + v + gates + o + gate/up) + 2·d_ff·d for d = 3072, d_ff = 9216
    assert bench.block_gemm_flops(load_config("dory4b")) == 220_348_416


def _pairs_brute(cfg, b, T, pos0):
    full = is_full_layer(cfg, b)
    n = 0
    for i in range(pos0, pos0 + T):
        for j in range(0, i + 1):
            if full or i - j < cfg["window"]:
                n += 1
    return n


@pytest.mark.parametrize("T,pos0", [(1, 0), (37, 0), (80, 0), (20, 50), (64, 100)])
def test_attention_pairs_match_brute_force(T, pos0):
    cfg = load_config("tiny")            # window 32, full layer every second block
    for b in range(4):
        assert bench.attn_pairs(cfg, b, T, pos0) == _pairs_brute(cfg, b, T, pos0)


@pytest.mark.parametrize("k", [1, 2, 4])
def test_stack_has_the_depth_of_the_closed_form(k):
    cfg = load_config("dory4b")
    blocks = bench.stack_blocks(cfg, k)
    assert 2 * len(blocks) == layer_applications(cfg, k) == 32 + 40 * k
    # the recurrent blocks appear k times, the others once
    assert blocks.count(8) == k and blocks.count(0) == 1 and blocks.count(35) == 1


def test_prefill_flops_of_the_4b_workloads():
    cfg = load_config("dory4b")
    # T = W = 4096: every layer is causal over the whole call
    pairs = 4096 * 4097 // 2
    per_pair = 4 * cfg["head_dim"] * cfg["n_q_heads"]
    for k, blocks in ((1, 36), (2, 56)):
        expect = blocks * (220_348_416 * 4096 + per_pair * pairs)
        assert bench.prefill_flops(cfg, 4096, k) == expect
    assert abs(bench.prefill_flops(cfg, 4096, 1) / 3.62e13 - 1) < 2e-3
    assert abs(bench.prefill_flops(cfg, 4096, 2) / 5.64e13 - 1) < 2e-3


def _kv_bytes_brute(cfg, B, pos, k):
    per_pos = 2 * cfg["n_kv_heads"] * cfg["head_dim"] * 2     # K and V, bf16
    tot = 0
    for b in bench.stack_blocks(cfg, k):
        keys = sum(1 for j in range(pos + 1)
                   if is_full_layer(cfg, b) or pos - j < cfg["window"])
        tot += B * keys * per_pos
    return tot


def test_decode_kv_bytes_match_brute_force():
    cfg = load_config("tiny")
    for pos in (0, 5, 31, 32, 90):
        for k in (1, 3):
            assert bench.decode_kv_bytes(cfg, 3, pos, k) == _kv_bytes_brute(cfg, 3, pos, k)


def test_decode_kv_bytes_of_the_4b_workload():
    cfg = load_config("dory4b")
    # 64 sequences at position 32768, k = 2: 14 full-layer and 42 window-layer
    # applications, 4096 bytes per cached position
    got = bench.decode_kv_bytes(cfg, 64, 32768, 2)
    assert got == 64 * 4096 * (14 * 32769 + 42 * 4096)
    assert abs(got / 165.4e9 - 1) < 5e-3


def test_profiled_traffic_is_dropped_when_the_kernel_source_changes(tmp_path, monkeypatch):
    import hashlib
    src = tmp_path / "kernel.cu"
    src.write_text("// version 1\n")
    sha = hashlib.sha1(src.read_bytes()).hexdigest()
    monkeypatch.setattr(bench, "PROFILED", {
        "k": {"traffic": 123, "source": (str(src), sha)},
        "r": {"ratio": 1.5, "source": (str(src), sha)},
    })
    assert bench.profiled_traffic("k") == 123
    assert bench.profiled_traffic("r", work=10) == 15.0
    assert bench.profiled_traffic("r") is None
    assert bench.profiled_traffic("unknown") is None
    src.write_text("// version 2\n")
    assert bench.profiled_traffic("k") is None
    assert bench.profiled_traffic("r", work=10) is None


def test_profiled_traffic_is_kept_per_weight_format(tmp_path, monkeypatch):
    """A capture of the bf16 kernel never stands in for the block-scaled one:
    the lookup is keyed by format, bf16 (or no format) using the plain key."""
    import hashlib
    src = tmp_path / "kernel.cu"
    src.write_text("// v\n")
    sha = hashlib.sha1(src.read_bytes()).hexdigest()
    monkeypatch.setattr(bench, "PROFILED", {
        "k": {"traffic": 100, "source": (str(src), sha)},
        "k:nvfp4": {"traffic": 40, "source": (str(src), sha)},
    })
    assert bench.profiled_traffic("k") == 100
    assert bench.profiled_traffic("k", fmt="bf16") == 100
    assert bench.profiled_traffic("k", fmt="nvfp4") == 40
    assert bench.profiled_traffic("k", fmt="mxfp8") is None


def test_committed_traffic_captures_match_the_current_sources():
    """Every committed capture names the kernel source it was taken on; the
    ones the bench reports must still match it (else the bench prints null)."""
    import hashlib
    import os
    for name, ent in bench.PROFILED.items():
        path, sha = ent["source"]
        with open(os.path.join(bench.ROOT, path), "rb") as f:
            assert hashlib.sha1(f.read()).hexdigest() == sha, name
