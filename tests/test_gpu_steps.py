"""Each step of the layer on the GPU against the oracle, teacher-forced.

Every step is fed the GPU's own output of the step before, so a mismatch
names the stage. Sizes span several tiles in every dimension and a ragged
sequence tail.
"""
import dataclasses

import numpy as np
import pytest

from gpu_common import ROW_TOL_BF16, host, layer_on_device, max_row_rel, positions, q3, rel_l2
from oracle import q3vl_oracle as O
import q3vl_synth as syn

pytestmark = pytest.mark.gpu

ODD_GROUP = dataclasses.replace(syn.Q2B_LAYER, name="odd-group-3", hidden=768, n_heads=6,
                                n_kv_heads=2, intermediate=1536, seq=300)

CASES = [
    syn.TINY_FP32,                       # fp32, 1 tile of rows
    syn.TINY_FP32.with_seq(77),          # fp32, ragged
    syn.Q2B_LAYER.with_seq(300),         # bf16, 3 row tiles, ragged
    syn.Q4B_LAYER.with_seq(700, images=((200, 16, 24),)),  # bias + image, ragged
    ODD_GROUP,                           # bf16, 3 query heads per KV head
]


def _within_output_rounding(w, got, ref):
    """|got - ref| within the rounding of the output dtype (plus accumulation slack)."""
    rel = 2.0 ** -8 if w.dtype == "bf16" else 2.0 ** -22
    bound = rel * np.abs(ref) + (1e-3 if w.dtype == "bf16" else 1e-6) * np.abs(ref).mean()
    bad = np.abs(got - ref) > bound
    return int(bad.sum()) == 0


def _tol(w):
    return 2e-6 if w.dtype == "fp32" else 1e-2


def _row_tol(w):
    return 1e-5 if w.dtype == "fp32" else ROW_TOL_BF16


@pytest.mark.parametrize("w", CASES, ids=lambda w: f"{w.name}-S{w.seq}")
def test_steps(w):
    m = q3()
    cfg = m.config_of(w)
    ocfg = O.Config.of(w)
    raw, packed = layer_on_device(w)
    x = syn.hidden_input(w).cuda()
    pos, ref_pos, _, _ = positions(w)
    tol = _tol(w)
    xh = host(x)

    # P1 cos/sin table
    cs = m.rope_table(cfg, pos)
    ang = O.mrope_angles(ref_pos, w.rope_theta, 128, w.mrope_section)
    assert np.max(np.abs(host(cs[..., 0]) - np.cos(ang))) < 2e-7
    assert np.max(np.abs(host(cs[..., 1]) - np.sin(ang))) < 2e-7

    # P2 row statistic: x * inv_rms is RMSNorm with a unit gain
    inv = m.rms_rowstat(cfg, x)
    assert rel_l2(xh * host(inv)[:, None], O.rms_norm(xh, np.ones(w.hidden), w.rms_eps)) < 1e-6

    # P3+P4 projections, q/k norm, MRoPE
    qkv = m.qkv_proj(cfg, packed, x, inv, cs)
    q, k, v = O.qkv(ocfg, raw, xh, ang)
    S = w.seq
    ref = np.concatenate([q.reshape(S, -1), k.reshape(S, -1), v.reshape(S, -1)], axis=1)
    got = host(qkv)
    Dq, Dkv = w.q_dim, w.kv_dim
    for name, sl in (("q", slice(0, Dq)), ("k", slice(Dq, Dq + Dkv)), ("v", slice(Dq + Dkv, None))):
        assert rel_l2(got[:, sl], ref[:, sl]) < tol, name
        # per head row: every (token, head) vector
        gh, rh = got[:, sl].reshape(-1, 128), ref[:, sl].reshape(-1, 128)
        assert max_row_rel(gh, rh) < _row_tol(w), (name, max_row_rel(gh, rh))

    # P5 attention on the GPU's q, k, v
    o = m.attention(cfg, qkv)
    qg = got[:, :Dq].reshape(S, w.n_heads, 128)
    kg = got[:, Dq:Dq + Dkv].reshape(S, w.n_kv_heads, 128)
    vg = got[:, Dq + Dkv:].reshape(S, w.n_kv_heads, 128)
    o_ref = O.attention(qg, kg, vg).reshape(S, -1)
    assert rel_l2(host(o), o_ref) < tol
    oh, orh = host(o).reshape(-1, 128), o_ref.reshape(-1, 128)
    assert max_row_rel(oh, orh) < _row_tol(w), max_row_rel(oh, orh)

    # P6 o-projection + residual: exact inputs, so the only error is the
    # output's own rounding (half an ulp of bf16 = 2^-8 relative) plus fp32
    # accumulation order
    h = m.o_proj(cfg, packed, o, x)
    h_ref = O.o_residual(raw, host(o), xh)
    assert _within_output_rounding(w, host(h), h_ref)

    # P7 + P8 post-attention norm, gate/up, SiLU * up
    inv2 = m.rms_rowstat(cfg, h)
    act = m.gate_up(cfg, packed, h, inv2)
    a_ref = O.ffn_act(ocfg, raw, host(h))
    assert rel_l2(host(act), a_ref) < tol
    assert max_row_rel(host(act), a_ref) < _row_tol(w), max_row_rel(host(act), a_ref)

    # P9 down + residual
    out = m.down(cfg, packed, act, h)
    out_ref = O.down_residual(raw, host(act), host(h))
    assert _within_output_rounding(w, host(out), out_ref)
    m.check_device()


def test_deepstack_down_epilogue():
    m = q3()
    w = syn.Q2B_LAYER.with_seq(260)
    cfg = m.config_of(w)
    raw, packed = layer_on_device(w)
    import torch
    h = syn.hidden_input(w).cuda()
    act = (torch.randn(w.seq, w.intermediate, generator=torch.Generator().manual_seed(3)) * 0.5
           ).to(torch.bfloat16).cuda()
    rows = torch.tensor([0, 5, 6, 7, 128, 129, 259], dtype=torch.int32, device="cuda")
    slab = (torch.randn(7, w.hidden, generator=torch.Generator().manual_seed(4)) * 0.1
            ).to(torch.bfloat16).cuda()
    dmap = m.deepstack_map(rows, w.seq)
    mh = host(dmap)
    assert [int(mh[r]) for r in (0, 5, 6, 7, 128, 129, 259)] == list(range(7))
    assert int((mh >= 0).sum()) == 7
    out0 = m.down(cfg, packed, act, h)
    out1 = m.down(cfg, packed, act, h, slab, dmap)
    rr = host(rows).astype(int)
    # the slab lands on its rows (within the output's bf16 rounding) ...
    ref = O.down_residual(raw, host(act), host(h))
    ref[rr] += host(slab)
    assert _within_output_rounding(w, host(out1), ref)
    # ... and nowhere else (bit-identical to the call without a slab)
    mask = np.ones(w.seq, bool)
    mask[rr] = False
    assert np.array_equal(host(out1)[mask], host(out0)[mask])
    m.check_device()


def test_deepstack_map_rejects_bad_rows():
    import torch
    m = q3()
    rows = torch.tensor([3, 3], dtype=torch.int32, device="cuda")
    m.deepstack_map(rows, 8)
    code, _ = m.device_status()
    assert code == -2
    rows = torch.tensor([1, 8], dtype=torch.int32, device="cuda")
    m.deepstack_map(rows, 8)
    code, _ = m.device_status()
    assert code == -2
    assert m.device_status() == (0, 0)
