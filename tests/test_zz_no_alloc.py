"""The allocation-free entry point, dory_mlp_sublayer_noalloc.

It exists for callers that cannot allocate device memory (no cudaMalloc in
their context, a fixed memory pool, or a plugin that only receives its input
and output buffers) and so cannot hand the library a workspace.  Its scratch is
a fixed array inside the library.  These tests call it through the C ABI and
check that it produces what the workspace-based dory_mlp_sublayer produces,
bit for bit, on two calls in a row (the second call finds the first call's
leftovers in the shared array), also at the 4B MLP shape's row limit, that it
matches the oracle's MLP sublayer, and that oversized calls are refused.  This file is collected
last so that a failure here never hides the other tests' results; it also
passes on its own in a fresh process.
"""

import numpy as np
import pytest
import torch

from tests.gpu_util import build, inputs, to_np, assert_parity, oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny():
    return build("tiny", seed=5, variant="random")


def test_noalloc_matches_workspace_entry_point_twice(tiny):
    cfg, prov, model = tiny
    _, rows = inputs(cfg, 31, 300)
    calls = [(0, rows[:180]), (5, rows[180:300])]   # different layers and row counts
    for layer, h in calls:
        ref = torch.from_numpy(h.astype(np.float32)).cuda()
        got = ref.clone()
        model.mlp_sublayer(layer, ref)                 # existing entry point (workspace)
        model.mlp_sublayer_noalloc(layer, got)         # built-in scratch
        torch.cuda.synchronize()
        assert model.device_status() == 0
        # same kernels on the same inputs: the results agree bit for bit
        assert torch.equal(got, ref), f"no-alloc vs workspace, layer {layer}"
        assert_parity(to_np(got), oracle(cfg, prov).mlp_sublayer(layer, h), tol_abs=5e-3,
                      tol_cos=0.9999, what=f"no-alloc vs oracle, layer {layer}")


def test_noalloc_rejects_rows_beyond_its_scratch(tiny):
    from looped_ngpt_transformer_fwd_b200 import binding as B
    cfg, prov, model = tiny
    limit = B.noalloc_max_rows(cfg["d_model"], cfg["d_ff"])
    h = torch.zeros(limit + 1, cfg["d_model"], dtype=torch.float32, device="cuda")
    with pytest.raises(B.DoryError) as e:
        model.mlp_sublayer_noalloc(0, h)
    assert e.value.status == -12
    ok = torch.from_numpy(inputs(cfg, 32, limit)[1].astype(np.float32)).cuda()
    ref = ok.clone()
    model.mlp_sublayer_noalloc(0, ok)
    model.mlp_sublayer(0, ref)
    torch.cuda.synchronize()
    assert torch.equal(ok, ref), "at the row limit"


def test_noalloc_at_the_4b_shape_limit():
    """The 4B MLP shape (d_model 3072, d_ff 9216) at the largest row count the
    built-in scratch holds, twice in a row: bit for bit the workspace entry
    point, and the oracle's MLP sublayer within the per-sublayer bar."""
    from looped_ngpt_transformer_fwd_b200 import binding as B
    cfg, prov, model = build("dory4b", seed=6, variant="random",
                             n_in_blocks=1, n_rec_blocks=1, n_out_blocks=1)
    n = B.noalloc_max_rows(cfg["d_model"], cfg["d_ff"])
    assert n >= 200
    _, rows = inputs(cfg, 33, n + 7)
    for layer, h in ((0, rows[:n]), (2, rows[7:n + 7])):
        ref = torch.from_numpy(h.astype(np.float32)).cuda()
        got = ref.clone()
        model.mlp_sublayer_noalloc(layer, got)
        model.mlp_sublayer(layer, ref)
        torch.cuda.synchronize()
        assert model.device_status() == 0
        assert torch.equal(got, ref), f"4B shape, layer {layer}"
        sel = slice(0, n, 37)            # sampled rows (the oracle runs in float64)
        assert_parity(to_np(got)[sel], oracle(cfg, prov).mlp_sublayer(layer, h[sel]),
                      tol_abs=5e-3, tol_cos=0.9999, what=f"4B shape vs oracle, layer {layer}")
    model.close()
