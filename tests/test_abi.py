"""The C ABI on a host without a GPU: the library loads, exports every symbol the
header declares, and its pure-arithmetic calls agree with the oracle."""

import ctypes
import os
import re

import pytest

from oracle import kv_cache_bytes
from synthetic import load_config

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dory.h")


@pytest.fixture(scope="module")
def B():
    from looped_ngpt_transformer_fwd_b200 import build, binding
    build.build()
    binding.lib()
    return binding


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"DORY_API\s+[\w\s\*]*?\b(dory_\w+)\s*\(", text)))


def test_header_declares_what_binding_expects(B):
    assert _declared() == sorted(B.EXPORTS)


def test_library_exports_every_declared_symbol(B):
    lib = ctypes.CDLL(B.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name


@pytest.mark.parametrize("name", ["tiny", "dory4b"])
@pytest.mark.parametrize("mode", ["per_loop", "last_loop"])
def test_kv_bytes_matches_oracle(B, name, mode):
    cfg = load_config(name)
    c = B.make_config(cfg)
    for seqs, ctx, kmax in ((1, 128, 1), (64, 32768, 2), (32, 131072, 4), (3, 17, 3), (8, 4095, 4)):
        assert B.dory_kv_bytes(c, mode, seqs, ctx, kmax) == kv_cache_bytes(cfg, mode, seqs, ctx, kmax)


def test_kv_bytes_last_loop_constant_and_config4_figures(B):
    """Last-loop footprint is the one-loop footprint for every k; the B=32 x 128K
    per-loop cache of the k=4 decode workload is ~451 GB (does not fit one GPU)."""
    c = B.make_config(load_config("dory4b"))
    one = B.dory_kv_bytes(c, "per_loop", 32, 131072, 1)
    assert all(B.dory_kv_bytes(c, "last_loop", 32, 131072, k) == one for k in (1, 2, 3, 4))
    per4 = B.dory_kv_bytes(c, "per_loop", 32, 131072, 4)
    assert abs(per4 / 1e9 - 450.9) < 0.5 and abs(one / 1e9 - 169.1) < 0.5


def test_bad_arguments_are_rejected_without_a_gpu(B):
    cfg = load_config("tiny")
    bad = B.make_config(dict(cfg, head_dim=96, d_model=384))
    assert B.dory_weight_bytes(bad) == 0
    assert B.dory_kv_bytes(B.make_config(cfg), "per_loop", 0, 10, 1) == 0
    assert B.dory_kv_bytes(B.make_config(cfg), 7, 1, 10, 1) == 0
    assert B.lib().dory_error_string(-3).decode() == "loop count k out of range"
    assert B.dory_weight_bytes(B.make_config(cfg)) > 0
