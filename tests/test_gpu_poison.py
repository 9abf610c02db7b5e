"""Scratch poisoning: every call must write the scratch it reads.

The workspaces of the prefill, the decode and the LM head are filled with 0xFF
bytes (a NaN in bf16 and fp32, -1 in int32) before the call, and the result
must be finite and bit-identical to the same call on a zeroed workspace. A
kernel that read a scratch word it had not written first would pick up a NaN
(or a wrong flag / map entry) and differ. This stands in for a device memory
checker, which is not used on this hardware.
"""
import numpy as np
import pytest
import torch

from gpu_common import host, layer_on_device, positions, q3
import q3vl_synth as syn

pytestmark = pytest.mark.gpu


def _ws(m, cfg, S, fill):
    ws = m.workspace(cfg, S)
    ws.fill_(fill)
    return ws


@pytest.mark.parametrize("w", [
    syn.Q2B_STACK.with_seq(700).with_layers(1),            # image span, DeepStack slab
    syn.Q4B_LAYER.with_seq(1000, images=((300, 20, 24),)),  # QKV bias, stream-K GEMMs
    syn.TINY_FP32.with_seq(77),                             # fp32, ragged
], ids=lambda w: f"{w.name}-S{w.seq}")
def test_layer_prefill_on_poisoned_workspace(w):
    m = q3()
    cfg = m.config_of(w)
    _, packed = layer_on_device(w)
    pos, _, _, _ = positions(w)
    slab = rows = None
    if w.images and w.deepstack_layers:
        slab = syn.deepstack_slabs(w)[0].cuda()
        rows = torch.tensor(syn.image_rows(w), dtype=torch.int32, device="cuda")
    x0 = syn.hidden_input(w).cuda()
    outs = []
    for fill in (0, 0xFF):
        x = x0.clone()
        m.layer_prefill(cfg, packed, x, pos, slab, rows, _ws(m, cfg, w.seq, fill))
        m.check_device()
        outs.append(host(x))
    assert np.all(np.isfinite(outs[1]))
    assert np.array_equal(outs[0], outs[1])


def test_stack_prefill_on_poisoned_workspace():
    # three layers of the 2B stack: DeepStack on all three, the row statistic
    # carried from each down epilogue to the next QKV, and the final norm
    m = q3()
    w = syn.Q2B_STACK.with_seq(640).with_layers(3)
    cfg = m.config_of(w)
    layers = [layer_on_device(w, l)[1] for l in range(w.n_layers)]
    pos, _, _, _ = positions(w)
    slabs = [s.cuda() for s in syn.deepstack_slabs(w)]
    rows = torch.tensor(syn.image_rows(w), dtype=torch.int32, device="cuda")
    gain = syn.final_norm(w).cuda()
    x0 = syn.hidden_input(w).cuda()
    outs = []
    for fill in (0, 0xFF):
        x = x0.clone()
        m.stack_prefill(cfg, layers, x, pos, gain, slabs, rows, _ws(m, cfg, w.seq, fill))
        m.check_device()
        outs.append(host(x))
    assert np.all(np.isfinite(outs[1]))
    assert np.array_equal(outs[0], outs[1])


@pytest.mark.parametrize("B", [1, 5])
def test_decode_on_poisoned_workspace(B):
    m = q3()
    w = syn.Q4B_LAYER.with_seq(300, images=((40, 8, 12),))
    cfg = m.config_of(w)
    _, packed = layer_on_device(w)
    pos, _, _, nxt = positions(w)
    kv = m.KvCache(cfg, n_seq=B, cap=w.seq + 8)
    for b in range(B):
        m.layer_prefill_kv(cfg, packed, syn.hidden_input(w).cuda(), pos, kv, seq=b)
    m.check_device()
    g = torch.Generator().manual_seed(5)
    x_in = torch.randn(B, w.hidden, generator=g).to(torch.bfloat16).cuda()
    seq = torch.arange(B, dtype=torch.int32, device="cuda")
    outs = []
    for fill in (0, 0xFF):
        lens = torch.full((B,), w.seq, dtype=torch.int32, device="cuda")
        p = torch.full((3, B), nxt, dtype=torch.int32, device="cuda")
        ws = m.decode_workspace(cfg, B, kv.cap)
        ws.fill_(fill)
        x = x_in.clone()
        m.layer_decode(cfg, packed, x, p, kv, seq, lens, ws)
        m.check_device()
        outs.append((host(x), host(kv.k[:, w.seq]), host(kv.v[:, w.seq])))
    for a, b in zip(outs[0], outs[1]):
        assert np.all(np.isfinite(b))
        assert np.array_equal(a, b)


def test_lm_head_on_poisoned_workspace():
    m = q3()
    cfg = m.config_of(syn.Q2B_LAYER)
    g = torch.Generator().manual_seed(7)
    vocab, B = 3000, 3
    weight = (0.02 * torch.randn(vocab, cfg.hidden, generator=g)).to(torch.bfloat16).cuda()
    gain = (1 + 0.1 * torch.randn(cfg.hidden, generator=g)).to(torch.bfloat16).cuda()
    xr = torch.randn(B, cfg.hidden, generator=g).to(torch.bfloat16).cuda()
    n = int(m.lib().q3vl_lm_head_workspace_bytes(__import__("ctypes").byref(cfg), B))
    outs = []
    for fill in (0, 0xFF):
        ws = torch.full((n,), fill, dtype=torch.uint8, device="cuda")
        outs.append(host(m.lm_head(cfg, xr, gain, weight, ws=ws)))
        m.check_device()
    assert np.all(np.isfinite(outs[1]))
    assert np.array_equal(outs[0], outs[1])
