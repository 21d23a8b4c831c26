"""The shared seeded generators: determinism, bf16 rounding and the counter hash."""

import numpy as np
import torch

from synthetic import f32_to_bf16_bits, bf16_bits_to_f32, hidden_in, load_config
from synthetic.kvfill import lowbias32, kv_values, kv_values_torch


def _lowbias32_ref(x):
    # the published steps with full-width Python integers, reduced mod 2^32
    m = 0xFFFFFFFF
    x ^= x >> 16
    x = (x * 0x7FEB352D) & m
    x ^= x >> 15
    x = (x * 0x846CA68B) & m
    x ^= x >> 16
    return x


def test_lowbias32_matches_published_steps():
    xs = [0, 1, 2, 0xDEADBEEF, 0xFFFFFFFF] + list(np.random.default_rng(0).integers(0, 2**32, 200))
    got = lowbias32(np.array(xs, dtype=np.int64))
    assert [int(v) for v in got] == [_lowbias32_ref(int(v)) for v in xs]
    assert lowbias32(0) == 0


def test_kv_values_numpy_equals_torch():
    s_qk = np.random.default_rng(1).uniform(0.5, 1.5, 64).astype(np.float32)
    k, v = kv_values(7, 35, 3, np.arange(1000, 1300), 2, 64, s_qk)
    kt, vt = kv_values_torch(7, 35, 3, np.arange(1000, 1300), 2, 64, s_qk, "cpu")
    assert np.array_equal(k, kt.float().numpy()) and np.array_equal(v, vt.float().numpy())
    # keys are s_qk times a unit vector (up to the bf16 rounding of the scale)
    nrm = np.linalg.norm(k / s_qk, axis=-1)
    assert np.abs(nrm - 1).max() < 1e-2
    assert set(np.unique(np.abs(v * 128))) <= set(range(0, 129))


def test_bf16_round_trip_and_rne():
    x = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, -0.0, 3.0e38], dtype=np.float32)
    r = bf16_bits_to_f32(f32_to_bf16_bits(x))
    assert r[0] == 1.0 and r[1] == 1.0 and r[2] == 1.0 + 2**-6 and r[3] == 0.0
    t = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(r[:4], t[:4])


def test_hidden_in_prefix_consistent_and_unit():
    cfg = load_config("tiny")
    a = hidden_in(cfg, 5, 300)
    b = hidden_in(cfg, 5, 40, row0=250)
    assert np.array_equal(a[250:290], b)
    n = np.linalg.norm(bf16_bits_to_f32(a).astype(np.float64), axis=1)
    assert np.abs(n - 1).max() < 5e-3
