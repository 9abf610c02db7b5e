"""Layer stacks on the GPU: the 2B 28-layer stack with DeepStack and final norm,
and the 32B-shape 50-layer prompt encoder, at full size.

The stack call itself is checked layer by layer, teacher-forced: running it
on the first L layers gives x_L, and x_L must match the oracle's layer L-1
applied to x_{L-1} (the same call on L-1 layers), on sampled rows (the oracle
forms K/V for every row and the rest only for the sampled rows). Layers after
the first take their input row statistic from the previous layer's down
epilogue inside the stack, so this exercises that path. The final norm must
match the oracle's norm of x_L.
"""
import numpy as np
import pytest
import torch

from gpu_common import ROW_TOL_BF16, host, max_row_rel, positions, q3, rel_l2
from oracle import q3vl_oracle as O
import q3vl_synth as syn

pytestmark = pytest.mark.gpu


def _rows(w, n, seed):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, w.seq - 1]
    for s, hm, wm in w.images:
        fixed += [s - 1, s, s + 1, s + hm * wm - 1, s + hm * wm]
    return np.unique(np.clip(np.concatenate([fixed, rng.integers(0, w.seq, n)]), 0, w.seq - 1))


def _check_layer(w, raw, x_in, x_out, pos_ref, rows, slab=None, ds_rows=None):
    ref = O.layer(O.Config.of(w), raw, x_in, pos_ref, slab, ds_rows, rows=rows)
    got = host(x_out)[rows]
    xin = host(x_in)[rows]
    assert np.all(np.isfinite(got))
    e = rel_l2(got, ref[rows])
    assert e <= 1e-2, e
    assert rel_l2(got - xin, ref[rows] - xin) <= 2e-2
    assert max_row_rel(got, ref[rows]) <= ROW_TOL_BF16
    assert max_row_rel(got - xin, ref[rows] - xin) <= 2 * ROW_TOL_BF16


def test_2b_stack28_deepstack_final_norm():
    m = q3()
    w = syn.Q2B_STACK
    cfg = m.config_of(w)
    pos, pos_ref, _, _ = positions(w)
    ds_rows = np.array(syn.image_rows(w))
    rows_d = torch.tensor(ds_rows, dtype=torch.int32, device="cuda")
    slabs = syn.deepstack_slabs(w)
    slabs_d = [s.cuda() for s in slabs]
    raws, packed = [], []
    for l in range(w.n_layers):
        raw = syn.layer_weights(w, l)
        raws.append(raw)
        packed.append(m.pack_layer(cfg, {k: v.cuda() for k, v in raw.items()}))
    gain = syn.final_norm(w)
    x0 = syn.hidden_input(w).cuda()
    ws = m.workspace(cfg, w.seq)
    rows = _rows(w, 16, 0)
    prev = x0.clone()
    for L in range(1, w.n_layers + 1):
        x = x0.clone()
        m.stack_prefill(cfg, packed[:L], x, pos, None, slabs_d, rows_d, ws)
        m.check_device()
        l = L - 1
        _check_layer(w, raws[l], prev.cpu(), x, pos_ref, rows,
                     slabs[l] if l < len(slabs) else None, ds_rows if l < len(slabs) else None)
        prev = x
    xs = x0.clone()
    m.stack_prefill(cfg, packed, xs, pos, gain.cuda(), slabs_d, rows_d, ws)
    m.check_device()
    ref_norm = O.rms_norm(host(prev), host(gain), w.rms_eps)
    assert rel_l2(host(xs), ref_norm) <= 1e-2


@pytest.fixture(scope="module")
def encoder32b():
    """The 50 packed layers of the 32B-shape encoder, drawn on the device (~49 GB)."""
    m = q3()
    w = syn.Q32B_ENC
    cfg = m.config_of(w)
    packed = []
    for l in range(w.n_layers):
        raw = syn.layer_weights(w, l, device="cuda")
        packed.append(m.pack_layer(cfg, raw))
        del raw
    torch.cuda.synchronize()
    yield w, cfg, packed
    del packed
    torch.cuda.empty_cache()


@pytest.mark.parametrize("S", [1064, 8192])
def test_32b_encoder50_no_final_norm(encoder32b, S):
    m = q3()
    w0, cfg, packed = encoder32b
    w = w0.with_seq(S)
    pos, pos_ref, _, _ = positions(w)
    x0 = syn.hidden_input(w).cuda()
    ws = m.workspace(cfg, S)
    rows = _rows(w, 12, 1)
    xs = {}
    for L in (1, w.n_layers - 1, w.n_layers):
        x = x0.clone()
        m.stack_prefill(cfg, packed[:L], x, pos, None, (), None, ws)
        m.check_device()
        assert torch.isfinite(x.float()).all()
        xs[L] = x
    xs[0] = x0
    for l in (0, w.n_layers - 1):
        raw = {k: v.cpu() for k, v in syn.layer_weights(w, l, device="cuda").items()}
        _check_layer(w, raw, xs[l].cpu(), xs[l + 1], pos_ref, rows)
