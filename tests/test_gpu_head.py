"""Embedding gather (+ soft-token splice) and LM head on the GPU against the oracle.

The gather is a copy, so it must be bit-exact. The logits must be within rel L2
1e-2 of the oracle. The GPU rounds the normalised row to bf16 before the
product, about 2^-9 relative per element, well inside that bound.
"""
import numpy as np
import pytest
import torch

from gpu_common import host, layer_on_device, positions, q3, rel_l2
from oracle import q3vl_oracle as O
import q3vl_synth as syn

pytestmark = pytest.mark.gpu


def _table(vocab, H, seed):
    g = torch.Generator().manual_seed(seed)
    return (0.02 * torch.randn(vocab, H, generator=g)).to(torch.bfloat16)


def test_embed_gathers_and_splices_bit_exact():
    m = q3()
    cfg = m.config_of(syn.Q2B_LAYER)
    vocab, S = 5000, 777
    table = _table(vocab, cfg.hidden, 1)
    rng = np.random.default_rng(2)
    tokens = rng.integers(0, vocab, S)
    rows = np.concatenate([np.arange(100, 356), rng.choice(np.arange(400, 777), 40, replace=False)])
    soft = torch.randn(len(rows), cfg.hidden, generator=torch.Generator().manual_seed(3)).to(
        torch.bfloat16)
    x = m.embed(cfg, table.cuda(), torch.tensor(tokens, dtype=torch.int32, device="cuda"),
                soft.cuda(), torch.tensor(rows, dtype=torch.int32, device="cuda"))
    m.check_device()
    want = O.embed(table, tokens, rows, soft)
    assert np.array_equal(host(x), want)


def test_embed_reports_bad_tokens_and_overlapping_rows():
    m = q3()
    cfg = m.config_of(syn.Q2B_LAYER)
    table = _table(100, cfg.hidden, 4).cuda()
    tok = torch.tensor([1, 2, 100, 3], dtype=torch.int32, device="cuda")
    x = m.embed(cfg, table, tok)
    code, _ = m.device_status()
    assert code == -2 and not x[2].any() and torch.equal(x[3], table[3])
    tok = torch.tensor([1, 2, 3, 4], dtype=torch.int32, device="cuda")
    soft = torch.zeros(2, cfg.hidden, dtype=torch.bfloat16, device="cuda")
    m.embed(cfg, table, tok, soft, torch.tensor([1, 1], dtype=torch.int32, device="cuda"))
    code, _ = m.device_status()
    assert code == -2
    m.embed(cfg, table, tok)
    m.check_device()


@pytest.mark.parametrize("B,vocab", [(1, 151936), (5, 1000), (33, 4096)],
                         ids=["b1-qwen3vl-vocab", "b5-ragged-vocab", "b33"])
def test_lm_head_matches_oracle(B, vocab):
    m = q3()
    w = syn.Q4B_LAYER
    cfg = m.config_of(w)
    table = _table(vocab, w.hidden, 5)
    g = torch.Generator().manual_seed(6)
    x = torch.randn(B, w.hidden, generator=g).to(torch.bfloat16)
    gain = (1.0 + 0.1 * torch.randn(w.hidden, generator=g)).to(torch.bfloat16)
    logits = m.lm_head(cfg, x.cuda(), gain.cuda(), table.cuda())
    m.check_device()
    want = O.lm_head(O.Config.of(w), x, gain, table)
    got = logits.cpu().numpy().astype(np.float64)
    for b in range(B):
        assert rel_l2(got[b], want[b]) <= 1e-2, b


def test_prompt_to_last_row_logits_through_two_layers():
    # tokens -> embed (image rows spliced) -> 2-layer stack with DeepStack ->
    # final norm + LM head of the last row, against the oracle's same chain
    m = q3()
    w = syn.Q2B_STACK.with_seq(600).with_layers(2)
    cfg = m.config_of(w)
    vocab = 3000
    table = _table(vocab, w.hidden, 7)
    rng = np.random.default_rng(8)
    tokens = rng.integers(0, vocab, w.seq)
    img = np.array(syn.image_rows(w))
    soft = torch.randn(len(img), w.hidden, generator=torch.Generator().manual_seed(9)).to(
        torch.bfloat16)
    pos, ref_pos, _, _ = positions(w)
    raws, packed = [], []
    for l in range(2):
        raw, pk = layer_on_device(w, l)
        raws.append(raw)
        packed.append(pk)
    slabs = syn.deepstack_slabs(w)
    rows_d = torch.tensor(img, dtype=torch.int32, device="cuda")
    x = m.embed(cfg, table.cuda(), torch.tensor(tokens, dtype=torch.int32, device="cuda"),
                soft.cuda(), rows_d)
    m.stack_prefill(cfg, packed, x, pos, None, [s.cuda() for s in slabs], rows_d)
    gain = syn.final_norm(w)
    logits = m.lm_head(cfg, x[-1:], gain.cuda(), table.cuda())
    m.check_device()
    x0 = O.embed(table, tokens, img, soft)
    h = O.stack(O.Config.of(w), raws, x0, ref_pos, slabs, img)
    want = O.lm_head(O.Config.of(w), h[-1:], gain, table)[0]
    assert rel_l2(logits.cpu().numpy()[0].astype(np.float64), want) <= 2e-2
