"""The bounds-checked debug build (libq3vl_debug.so, -DQ3VL_DEBUG).

In that build every kernel checks the computed index of each global access it
makes outside TMA and records Q3VL_ERANGE (with a location tag) instead of
making an out-of-range access. A child process loads it (Q3VL_LIBRARY=debug),
runs a layer with bias and an image span, a three-layer stack with DeepStack
and the final norm, a decode step and the LM head, and reports the device
error record after each; every record must be clean, and the outputs must
match the release library's on the same inputs (the checks do not touch the
arithmetic, so within the bf16 rounding of the layer).
"""
import json
import os
import subprocess
import sys
import tempfile

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_workloads(out_dir):
    """Runs the calls on the library this process loaded; writes outputs to out_dir."""
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import qwen3_vl_decoder_b200 as m
    import q3vl_synth as syn
    from gpu_common import layer_on_device, positions
    status = {}
    # a layer: QKV bias, an image span, stream-K GEMMs, both attention heads of a group
    w = syn.Q4B_LAYER.with_seq(1000, images=((300, 20, 24),))
    cfg = m.config_of(w)
    _, packed = layer_on_device(w)
    pos, _, _, nxt = positions(w)
    x = syn.hidden_input(w).cuda()
    m.layer_prefill(cfg, packed, x, pos)
    status["layer"] = m.device_status()
    np.save(os.path.join(out_dir, "layer.npy"), x.float().cpu().numpy())
    # decode one token per sequence against the layer's cache, then the LM head
    kv = m.KvCache(cfg, n_seq=2, cap=w.seq + 4)
    for b in range(2):
        m.layer_prefill_kv(cfg, packed, syn.hidden_input(w).cuda(), pos, kv, seq=b)
    xd = torch.randn(2, w.hidden, generator=torch.Generator().manual_seed(3)).to(
        torch.bfloat16).cuda()
    p = torch.full((3, 2), nxt, dtype=torch.int32, device="cuda")
    lens = torch.full((2,), w.seq, dtype=torch.int32, device="cuda")
    m.layer_decode(cfg, packed, xd, p, kv, torch.arange(2, dtype=torch.int32, device="cuda"), lens)
    status["decode"] = m.device_status()
    np.save(os.path.join(out_dir, "decode.npy"), xd.float().cpu().numpy())
    g = torch.Generator().manual_seed(4)
    table = (0.02 * torch.randn(3000, w.hidden, generator=g)).to(torch.bfloat16).cuda()
    gain = (1 + 0.1 * torch.randn(w.hidden, generator=g)).to(torch.bfloat16).cuda()
    logits = m.lm_head(cfg, xd, gain, table)
    status["lm_head"] = m.device_status()
    np.save(os.path.join(out_dir, "logits.npy"), logits.cpu().numpy())
    # a stack: DeepStack on three layers, row statistics carried between layers, final norm
    ws_ = syn.Q2B_STACK.with_seq(640).with_layers(3)
    cfg2 = m.config_of(ws_)
    layers = [layer_on_device(ws_, l)[1] for l in range(ws_.n_layers)]
    pos2, _, _, _ = positions(ws_)
    slabs = [s.cuda() for s in syn.deepstack_slabs(ws_)]
    rows = torch.tensor(syn.image_rows(ws_), dtype=torch.int32, device="cuda")
    x2 = syn.hidden_input(ws_).cuda()
    m.stack_prefill(cfg2, layers, x2, pos2, syn.final_norm(ws_).cuda(), slabs, rows)
    status["stack"] = m.device_status()
    np.save(os.path.join(out_dir, "stack.npy"), x2.float().cpu().numpy())
    with open(os.path.join(out_dir, "status.json"), "w") as f:
        json.dump(status, f)


def _child(library, out_dir):
    env = dict(os.environ, Q3VL_LIBRARY=library)
    code = (f"import sys; sys.path.insert(0, {os.path.join(ROOT, 'tests')!r}); "
            f"import test_gpu_debug_build as t; t.run_workloads({out_dir!r})")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    with open(os.path.join(out_dir, "status.json")) as f:
        return json.load(f)


def test_debug_build_runs_clean_and_matches_release():
    if not os.path.exists(os.path.join(ROOT, "qwen3_vl_decoder_b200", "libq3vl_debug.so")):
        pytest.fail("libq3vl_debug.so is not built (python -m qwen3_vl_decoder_b200.build --debug)")
    with tempfile.TemporaryDirectory() as dbg, tempfile.TemporaryDirectory() as rel:
        st_dbg = _child("debug", dbg)
        st_rel = _child("release", rel)
        for name, (code, where) in st_dbg.items():
            assert code == 0, f"{name}: device error {code} at location {where} in the debug build"
        assert all(c == 0 for c, _ in st_rel.values()), st_rel
        for name in ("layer", "decode", "logits", "stack"):
            a = np.load(os.path.join(dbg, name + ".npy")).astype(np.float64)
            b = np.load(os.path.join(rel, name + ".npy")).astype(np.float64)
            assert np.all(np.isfinite(a))
            err = np.linalg.norm(a - b) / np.linalg.norm(b)
            assert err <= 1e-3, (name, err)
