"""Stream-K tails of the tensor-core GEMM (the prefill output and down
projections' schedule): a partial last wave of tiles is spread over every CTA
as equal runs of k blocks, a tile split between two CTAs finished by the one
holding its first k blocks.

Checked: the product against the float64 product of the same bf16 operands at
the 4B projection shapes and at ragged ones (M not a multiple of 128, a single
wave, 128-column tiles, two k blocks per tile); results identical from call to
call and with a reused workspace (its launch counter moves every call); the
workspace's status word stays zero; and the whole 4B-shape prefill with the
tails on against the same model with them off.
"""

import ctypes

import numpy as np
import pytest
import torch

from tests.gpu_util import inputs, to_np

pytestmark = pytest.mark.gpu


def _lib():
    from looped_ngpt_transformer_fwd_b200 import build as libbuild
    libbuild.build()


def _tiles(M, N):
    bn = 256 if N % 256 == 0 else 128
    return -(-M // 128) * (N // bn)


# (M, N, K): 4B down (384 tiles, 144 k blocks of 64), 4B output projection
# (384 tiles, 48), ragged M with one and a fraction waves (160 tiles), a
# second wave just begun on 128-column tiles (352 tiles), two k blocks per tile
SHAPES = [(4096, 3072, 9216), (4096, 3072, 3072), (2500, 2048, 1024), (4096, 1408, 512),
          (300, 25600, 128)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_streamk_gemm_matches_fp64_and_repeats_exactly(M, N, K):
    from looped_ngpt_transformer_fwd_b200.model import gemm_bf16, gemm_bf16_streamk
    _lib()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert _tiles(M, N) > sms and _tiles(M, N) % sms != 0     # the tail runs
    g = torch.Generator(device="cuda").manual_seed(M + 3 * N + K)
    A = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
    Bm = torch.randn(N, K, device="cuda", generator=g).to(torch.bfloat16)
    C, ws = gemm_bf16_streamk(A, Bm)
    C2, _ = gemm_bf16_streamk(A, Bm, ws=ws)          # counter moved: same bits
    C3, _ = gemm_bf16_streamk(A, Bm)                 # fresh workspace: same bits
    plain = gemm_bf16(A, Bm)
    torch.cuda.synchronize()
    assert int(ws[-4:].view(torch.int32).item()) == 0   # no wait gave up
    assert torch.equal(C, C2) and torch.equal(C, C3)
    ref = A.double() @ Bm.double().T
    scale = ref.abs().max().item()
    err = (C.double() - ref).abs().max().item()
    assert err <= 1e-4 * scale + 1e-4, err          # the bound of the plain GEMM's test
    # the plain schedule sums each tile's K in one run: fp32 rounding apart
    assert (C - plain).abs().max().item() <= 2e-6 * scale * np.sqrt(K / 64), \
        (C - plain).abs().max().item()


def test_streamk_gemm_rejects_a_short_or_misaligned_workspace():
    from looped_ngpt_transformer_fwd_b200 import binding as B
    from looped_ngpt_transformer_fwd_b200.model import _ptr
    _lib()
    M, N, K = 512, 512, 128
    A = torch.zeros(M, K, dtype=torch.bfloat16, device="cuda")
    Bm = torch.zeros(N, K, dtype=torch.bfloat16, device="cuda")
    C = torch.empty(M, N, dtype=torch.float32, device="cuda")
    need = B.dory_gemm_bf16_streamk_workspace_bytes(N)
    ws = torch.zeros(need + 512, dtype=torch.uint8, device="cuda")
    lib = B.lib()
    assert lib.dory_gemm_bf16_streamk(_ptr(A), _ptr(Bm), _ptr(C), M, N, K, _ptr(ws), need - 1,
                                      None) == -6   # DORY_ERR_BUFFER_TOO_SMALL
    off = ctypes.c_void_p(ws.data_ptr() + 16)
    assert lib.dory_gemm_bf16_streamk(_ptr(A), _ptr(Bm), _ptr(C), M, N, K, off, need,
                                      None) == -7   # DORY_ERR_MISALIGNED


@pytest.mark.parametrize("fmt", ["bf16", "mxfp8", "nvfp4"])
def test_4b_shape_prefill_streamk_on_and_off_agree(fmt):
    """4B block shapes (1 + 1 + 1 blocks, k = 2) on 4096 tokens: the output and
    down projections have 384 tiles, so their last wave runs as stream-K
    tails (block-scaled too: the partial is added before the tensor-scale
    product).  With the tails on and off the stack agrees to fp32 rounding
    (propagated through six nGPT updates; for the block-scaled formats also
    through the requantised stream), and two calls with the tails on are
    bit-identical."""
    from looped_ngpt_transformer_fwd_b200.model import DoryModel
    from oracle import weights_from_generator
    from synthetic import load_config
    _lib()
    cfg = load_config("dory4b", n_in_blocks=1, n_rec_blocks=1, n_out_blocks=1, full_period=2)
    prov = weights_from_generator(cfg, 13, "random")
    model = DoryModel(cfg, prov, weight_format=fmt)
    T, k = 4096, 2
    x, _ = inputs(cfg, 47, T)
    outs = []
    for on in (True, True, False):
        assert model.stream_k(on) == on
        kv = model.kv_cache("last_loop", 1, T, k_max=k)
        outs.append(model.prefill(kv, x, k).float())
        torch.cuda.synchronize()
        assert model.device_status() == 0
        del kv
    assert torch.equal(outs[0], outs[1])
    cos = torch.nn.functional.cosine_similarity(outs[0], outs[2], dim=1).min().item()
    if fmt == "bf16":
        diff = (outs[0] - outs[2]).abs().max().item()
        assert diff <= 2e-3, diff      # bf16 outputs: a rounding flip is 2^-9 of a unit row value
        assert cos >= 0.99999, cos
    else:
        # an fp32 rounding difference can flip an element's code in the next
        # projection's quantised input (a whole grid step of E4M3 / E2M1)
        assert cos >= 0.9995, cos
    model.close()
    torch.cuda.empty_cache()
