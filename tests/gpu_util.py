"""Helpers of the GPU parity tests: building the library-backed model and the
oracle on the same seeded inputs, and the parity metrics."""

import numpy as np
import torch

from oracle import Oracle, KVCache as OracleCache, weights_from_generator
from synthetic import load_config, hidden_in, bf16_bits_to_f32

# Parity bar on output hidden states (bf16 weights/activations, fp32
# accumulation against the float64 oracle): max |diff| <= 3e-2 and per-token
# cosine similarity >= 0.999.
TOL_ABS = 3e-2
TOL_COS = 0.999


def build(cfg_name="tiny", seed=0, variant="random", allow_extrapolated_k=False, **over):
    from looped_ngpt_transformer_fwd_b200 import build as libbuild
    from looped_ngpt_transformer_fwd_b200.model import DoryModel
    libbuild.build()
    cfg = load_config(cfg_name, **over)
    prov = weights_from_generator(cfg, seed, variant)
    model = DoryModel(cfg, prov, allow_extrapolated_k=allow_extrapolated_k)
    return cfg, prov, model


def inputs(cfg, seed, n, row0=0):
    """(bf16 torch tensor on cuda [n, d], float64 numpy rows of the same values)."""
    bits = hidden_in(cfg, seed, n, row0)
    t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    return t, bf16_bits_to_f32(bits).astype(np.float64)


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def metrics(gpu, ref):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    diff = np.abs(gpu - ref).max() if gpu.size else 0.0
    cos = (gpu * ref).sum(-1) / (np.linalg.norm(gpu, axis=-1) * np.linalg.norm(ref, axis=-1))
    return float(diff), float(cos.min()) if cos.size else 1.0


def assert_parity(gpu, ref, tol_abs=TOL_ABS, tol_cos=TOL_COS, what=""):
    diff, cos = metrics(gpu, ref)
    assert diff <= tol_abs and cos >= tol_cos, f"{what}: max|diff|={diff:.3e} min cos={cos:.6f}"
    return diff, cos


def oracle(cfg, prov):
    return Oracle(cfg, prov)


def oracle_cache(cfg, mode, k_max=1, **kw):
    return OracleCache(cfg, mode, k_max=k_max, **kw)
