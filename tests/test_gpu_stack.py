"""Layer stacks on the GPU: the 2B 28-layer stack with DeepStack and final norm,
and the 32B-shape 50-layer prompt encoder, at full size.

Per layer, teacher-forced: layer l's GPU output is compared with the oracle
applied to the GPU's own layer-l input, on sampled rows (the oracle forms K/V
for every row and the rest only for the sampled rows). The stack call must
agree with the layer-by-layer sequence (it differs only in how the input row
statistic of layers after the first is summed: from the previous layer's
down epilogue instead of a separate pass), and its final norm must match the
oracle's.
"""
import numpy as np
import pytest
import torch

from gpu_common import host, positions, q3, rel_l2
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

    # layer by layer, teacher-forced against the oracle
    x = x0.clone()
    rows = _rows(w, 16, 0)
    for l in range(w.n_layers):
        x_in = x.clone()
        slab = slabs_d[l] if l < len(slabs_d) else None
        m.layer_prefill(cfg, packed[l], x, pos, slab, rows_d if slab is not None else None, ws)
        m.check_device()
        _check_layer(w, raws[l], x_in.cpu(), x, pos_ref, rows,
                     slabs[l] if l < len(slabs) else None, ds_rows if l < len(slabs) else None)
    by_layer = x.clone()
    m.final_norm(cfg, by_layer, gain.cuda())

    # the stack call is the same sequence
    xs = x0.clone()
    m.stack_prefill(cfg, packed, xs, pos, gain.cuda(), slabs_d, rows_d, ws)
    m.check_device()
    assert rel_l2(host(xs), host(by_layer)) <= 1e-2
    ref_norm = O.rms_norm(host(x), host(gain), w.rms_eps)
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
    # full 50-layer stack, no final norm: the unnormalised residual stream
    xs = x0.clone()
    m.stack_prefill(cfg, packed, xs, pos, None, (), None, ws)
    m.check_device()
    assert torch.isfinite(xs.float()).all()
    # teacher-forced checks of the first and the last layer
    x = x0.clone()
    for l in range(w.n_layers):
        if l in (0, w.n_layers - 1):
            x_in = x.clone()
            m.layer_prefill(cfg, packed[l], x, pos, None, None, ws)
            raw = {k: v.cpu() for k, v in syn.layer_weights(w, l, device="cuda").items()}
            _check_layer(w, raw, x_in.cpu(), x, pos_ref, rows)
        else:
            m.layer_prefill(cfg, packed[l], x, pos, None, None, ws)
    m.check_device()
    assert rel_l2(host(xs), host(x)) <= 1e-2
