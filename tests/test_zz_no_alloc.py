"""q3vl_layer_prefill_noalloc, the entry point for callers that cannot allocate.

Some callers cannot call cudaMalloc at all: a plug-in inside a framework that
has reserved the GPU's memory for its own pool, a C caller without a device
allocator, or a path that must not pay cudaMalloc's device-wide
synchronisation. This entry point runs the same layer with a scratch array
built into the library. It runs the same deterministic kernels as the
workspace entry point, so its output must be bit-identical to that entry
point's output on the same inputs.

The calls go through the C ABI (ctypes). Before the compared calls the shared
scratch is dirtied on purpose by calls on other data: another sequence length,
another input and, for the image workload, a call with a DeepStack slab before
one without. A call that read scratch it had not written first would then see
the previous call's values and differ from the workspace entry point.
"""
import ctypes

import numpy as np
import pytest
import torch

from gpu_common import host, layer_on_device, positions, q3
import q3vl_synth as syn

pytestmark = pytest.mark.gpu


def _noalloc(m, cfg, packed, x, pos, slab, rows):
    n_img = 0 if rows is None else rows.numel()
    ptr = (lambda t: None if t is None else ctypes.c_void_p(t.data_ptr()))
    rc = m.lib().q3vl_layer_prefill_noalloc(
        ctypes.byref(cfg), ctypes.byref(packed.views), ptr(x), x.shape[0], ptr(pos), ptr(slab),
        ptr(rows), n_img, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc


def _inputs(w):
    pos, _, _, _ = positions(w)
    slab = rows = None
    if w.images and w.deepstack_layers:
        slab = syn.deepstack_slabs(w)[0].cuda()
        rows = torch.tensor(syn.image_rows(w), dtype=torch.int32, device="cuda")
    return pos, slab, rows


def _workspace_result(m, cfg, packed, x0, pos, slab, rows):
    """The workspace entry point's output, on a workspace filled with NaN bytes."""
    ws = m.workspace(cfg, x0.shape[0])
    ws.fill_(0xFF)
    x = x0.clone()
    m.layer_prefill(cfg, packed, x, pos, slab, rows, ws)
    m.check_device()
    return host(x)


def _dirty(m, cfg, packed, w, other_seq):
    """noalloc calls on other data: another length and input, a slab call first."""
    wd = w.with_seq(other_seq, images=tuple(im for im in w.images
                                            if im[0] + im[1] * im[2] <= other_seq))
    pos, slab, rows = _inputs(wd)
    xh = syn.hidden_input(wd)
    x = (3.0 * xh.float()).to(xh.dtype).cuda()
    assert _noalloc(m, cfg, packed, x, pos, slab, rows) == 0, m.lib().q3vl_last_error()
    m.check_device()


@pytest.mark.parametrize("w,other_seq", [
    (syn.Q2B_STACK.with_seq(1024).with_layers(1), 1400),  # 2B shape, image span + DeepStack
    (syn.TINY_FP32, 300),                                 # fp32
], ids=lambda v: f"{v.name}-S{v.seq}" if hasattr(v, "name") else str(v))
def test_noalloc_bit_identical_to_workspace_entry_point(w, other_seq):
    m = q3()
    cfg = m.config_of(w)
    _, packed = layer_on_device(w)
    pos, slab, rows = _inputs(w)
    x0 = syn.hidden_input(w).cuda()
    want = _workspace_result(m, cfg, packed, x0, pos, slab, rows)
    _dirty(m, cfg, packed, w, other_seq)
    for call in range(2):   # two calls in a row, the second on the first one's scratch
        x = x0.clone()
        assert _noalloc(m, cfg, packed, x, pos, slab, rows) == 0, m.lib().q3vl_last_error()
        m.check_device()
        got = host(x)
        assert np.all(np.isfinite(got))
        assert np.array_equal(got, want), (call, float(np.max(np.abs(got - want))))
    if slab is not None:
        # after calls with a slab, a call without one: no DeepStack row may leak in
        want_plain = _workspace_result(m, cfg, packed, x0, pos, None, None)
        x = x0.clone()
        assert _noalloc(m, cfg, packed, x, pos, None, None) == 0, m.lib().q3vl_last_error()
        m.check_device()
        assert np.array_equal(host(x), want_plain)
        assert not np.array_equal(want_plain, want)


def test_noalloc_refuses_layers_above_its_scratch():
    m = q3()
    w = syn.Q2B_LAYER.with_seq(2048)   # needs ~76 MiB of scratch
    cfg = m.config_of(w)
    _, packed = layer_on_device(w.with_seq(8))
    x = torch.zeros((w.seq, w.hidden), dtype=torch.bfloat16, device="cuda")
    pos = torch.zeros((3, w.seq), dtype=torch.int32, device="cuda")
    rc = _noalloc(m, cfg, packed, x, pos, None, None)
    assert rc == -5
    assert b"scratch" in m.lib().q3vl_last_error()
