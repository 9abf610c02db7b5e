"""q3vl_layer_prefill_noalloc, the entry point for callers that cannot allocate.

Some callers cannot call cudaMalloc at all (a plug-in inside a framework that
has reserved the GPU's memory for its own pool, a C caller without a device
allocator, a path that must not pay cudaMalloc's device-wide sync). This
entry point runs the same layer with a scratch array built into the library.
Here it is called through the C ABI (ctypes) twice in a row, and each output
must match the workspace entry point's output within the parity tolerance
of the layer tests. The second call starts from the scratch contents the
first call left behind.
"""
import ctypes

import numpy as np
import pytest
import torch

from gpu_common import host, layer_on_device, positions, q3, rel_l2, tolerance
import q3vl_synth as syn

pytestmark = pytest.mark.gpu


def _noalloc(m, cfg, packed, x, pos, slab, rows):
    n_img = 0 if rows is None else rows.numel()
    ptr = (lambda t: None if t is None else ctypes.c_void_p(t.data_ptr()))
    rc = m.lib().q3vl_layer_prefill_noalloc(
        ctypes.byref(cfg), ctypes.byref(packed.views), ptr(x), x.shape[0], ptr(pos), ptr(slab),
        ptr(rows), n_img, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc


@pytest.mark.parametrize("w", [
    syn.Q2B_STACK.with_seq(1024).with_layers(1),   # 2B shape, image span + DeepStack slab
    syn.TINY_FP32,                                 # fp32
], ids=lambda w: f"{w.name}-S{w.seq}")
def test_noalloc_matches_workspace_entry_point_twice(w):
    m = q3()
    cfg = m.config_of(w)
    _, packed = layer_on_device(w)
    pos, _, _, _ = positions(w)
    slab = rows = None
    if w.images and w.deepstack_layers:
        slab = syn.deepstack_slabs(w)[0].cuda()
        rows = torch.tensor(syn.image_rows(w), dtype=torch.int32, device="cuda")
    x0 = syn.hidden_input(w).cuda()
    ref = x0.clone()
    m.layer_prefill(cfg, packed, ref, pos, slab, rows)
    m.check_device()
    want = host(ref)
    tol, mabs = tolerance(w)
    for call in range(2):
        x = x0.clone()
        assert _noalloc(m, cfg, packed, x, pos, slab, rows) == 0, m.lib().q3vl_last_error()
        m.check_device()
        got = host(x)
        assert np.all(np.isfinite(got))
        assert rel_l2(got, want) <= tol, (call, rel_l2(got, want))
        if mabs is not None:
            assert np.max(np.abs(got - want)) <= mabs


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
