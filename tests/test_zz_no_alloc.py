"""The allocation-free entry point, dory_mlp_sublayer_noalloc.

It exists for callers that cannot allocate device memory (no cudaMalloc in
their context, a fixed memory pool, or a plugin that only receives its input
and output buffers) and so cannot hand the library a workspace.  Its scratch is
a fixed array inside the library.  These tests call it through the C ABI and
check that it produces what the workspace-based dory_mlp_sublayer produces,
on two calls in a row (the second call finds the first call's leftovers in the
shared array), and that oversized calls are refused.  This file is collected
last so that a failure here never hides the other tests' results; it also
passes on its own in a fresh process.
"""

import numpy as np
import pytest
import torch

from tests.gpu_util import build, inputs, to_np, assert_parity

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
        assert_parity(to_np(got), to_np(ref), tol_abs=5e-3, tol_cos=0.9999,
                      what=f"no-alloc vs workspace, layer {layer}")


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
    assert_parity(to_np(ok), to_np(ref), tol_abs=5e-3, tol_cos=0.9999, what="at the row limit")
