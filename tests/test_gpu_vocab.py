"""Tokens in and out on the GPU: embedding lookup, LM head, sampling.

Against oracle/vocab.py (the nGPT reading of the model's two ends; the
vocabulary size is a config value): embedding rows within bf16 rounding,
logits within fp32 accumulation error, and every sampled token bit for bit the
oracle's draw from the same fp32 logits (the decision is taken in the same
precision on both sides: the kernel's logits, double-precision keys).
"""

import numpy as np
import pytest
import torch

from oracle import vocab as OV
from tests.gpu_util import build, inputs, to_np, oracle, oracle_cache
from synthetic import vocab_weights
from synthetic.bf16 import bf16_bits_to_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny_vocab():
    cfg, prov, model = build("tiny", seed=31, variant="random")
    tables = vocab_weights(cfg, 31)
    return cfg, prov, model, tables, model.vocab(tables)


def _tables_f64(tables):
    return (bf16_bits_to_f32(tables["emb_in"]).astype(np.float64),
            bf16_bits_to_f32(tables["emb_out"]).astype(np.float64),
            tables["logit_scale"].astype(np.float64))


def test_embedding_rows(tiny_vocab):
    cfg, prov, model, tables, voc = tiny_vocab
    E_in, _, _ = _tables_f64(tables)
    toks = np.random.default_rng(1).integers(0, cfg["vocab_size"], 300).astype(np.int32)
    toks[:3] = [0, cfg["vocab_size"] - 1, 0]
    h = voc.embed(torch.from_numpy(toks).cuda())
    torch.cuda.synchronize()
    ref = OV.embed(E_in, toks)
    assert np.abs(to_np(h) - ref).max() < 5e-4
    assert model.device_status() == 0


def test_embedding_rejects_out_of_range_tokens(tiny_vocab):
    cfg, prov, model, tables, voc = tiny_vocab
    toks = torch.tensor([5, -1, cfg["vocab_size"], 7], dtype=torch.int32, device="cuda")
    h = voc.embed(toks)
    torch.cuda.synchronize()
    assert model.device_status() == -11
    assert torch.count_nonzero(h[1:3].float()) == 0 and torch.count_nonzero(h[0].float()) > 0


def test_lm_head_logits(tiny_vocab):
    cfg, prov, model, tables, voc = tiny_vocab
    _, E_out, s = _tables_f64(tables)
    x, h = inputs(cfg, 91, 37)
    z = voc.logits(x)
    torch.cuda.synchronize()
    ref = OV.lm_head(E_out, s, h)
    err = np.abs(to_np(z) - ref).max()
    assert err <= 1e-4 * np.abs(ref).max() + 1e-4, err


@pytest.mark.parametrize("temperature", [0.0, 0.7, 1.0, 2.5])
def test_sampling_is_the_oracle_draw(tiny_vocab, temperature):
    cfg, prov, model, tables, voc = tiny_vocab
    x, _ = inputs(cfg, 92, 64)
    z = voc.logits(x)
    steps = torch.from_numpy(np.random.default_rng(3).integers(0, 2 ** 31, 64).astype(np.int32)).cuda()
    tok = voc.sample(z, temperature, seed=1234, steps=steps)
    torch.cuda.synchronize()
    T = float(np.float32(temperature))
    want = OV.sample(z.double().cpu().numpy(), T, 1234, steps.cpu().numpy())
    assert np.array_equal(tok.cpu().numpy(), want)
    if temperature > 0:
        # the draw moves with the seed
        other = voc.sample(z, temperature, seed=1235, steps=steps)
        assert not torch.equal(other, tok)


def test_sampling_over_a_large_vocabulary():
    """131072 tokens (the assumed 4B vocabulary) on 8 rows, greedy and T = 1."""
    cfg, prov, model = build("tiny", seed=32, variant="random")
    tables = vocab_weights(cfg, 32, vocab=131072)
    voc = model.vocab(tables)
    x, _ = inputs(cfg, 93, 8)
    z = voc.logits(x)
    steps = torch.arange(8, dtype=torch.int32, device="cuda") * 977
    zz = z.double().cpu().numpy()
    for T in (0.0, 1.0):
        tok = voc.sample(z, T, seed=99, steps=steps)
        torch.cuda.synchronize()
        assert np.array_equal(tok.cpu().numpy(), OV.sample(zz, T, 99, steps.cpu().numpy()))
    voc.free()
    model.close()


def test_tokens_through_the_stack(tiny_vocab):
    """tokens -> embedding -> looped prefill (k = 2) -> LM head of every row ->
    greedy next token, against the oracle chain."""
    cfg, prov, model, tables, voc = tiny_vocab
    E_in, E_out, s = _tables_f64(tables)
    toks = np.random.default_rng(4).integers(0, cfg["vocab_size"], 96).astype(np.int32)
    h_in = voc.embed(torch.from_numpy(toks).cuda())
    kv = model.kv_cache("last_loop", 1, 96, k_max=2)
    h_out = model.prefill(kv, h_in, 2)
    z = voc.logits(h_out)
    tok = voc.sample(z, 0.0)
    torch.cuda.synchronize()
    hin_ref = bf16_bits_to_f32(h_in.cpu().view(torch.int16).numpy().view(np.uint16)).astype(np.float64)
    assert np.abs(hin_ref - OV.embed(E_in, toks)).max() < 5e-4
    ref_h = oracle(cfg, prov).forward(hin_ref, 0, 2, oracle_cache(cfg, "last_loop", k_max=2))
    ref_z = OV.lm_head(E_out, s, ref_h)
    got_z = to_np(z)
    assert np.abs(got_z - ref_z).max() < 0.05 * np.abs(ref_z).max()
    assert np.array_equal(tok.cpu().numpy(), OV.sample(z.double().cpu().numpy(), 0.0, 0, None))
    # the oracle's own greedy choice agrees wherever its top two are not within the error
    top2 = np.sort(ref_z, axis=1)[:, -2:]
    clear = (top2[:, 1] - top2[:, 0]) > 2 * np.abs(got_z - ref_z).max()
    assert clear.sum() > 50
    assert np.array_equal(tok.cpu().numpy()[clear], ref_z.argmax(axis=1)[clear])
