"""Shared helpers of the GPU parity tests: device inputs, oracle references, metrics."""
import numpy as np
import torch

from oracle import q3vl_oracle as O
import q3vl_synth as syn


def q3():
    import qwen3_vl_decoder_b200 as m
    return m


def rel_l2(got, want) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))


def max_row_rel(got, want) -> float:
    """Largest relative L2 error of any single row (last axis): a per-row bound
    that a handful of wrong rows cannot hide behind the whole-tensor norm."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    num = np.linalg.norm((got - want).reshape(-1, want.shape[-1]), axis=1)
    den = np.maximum(np.linalg.norm(want.reshape(-1, want.shape[-1]), axis=1), 1e-300)
    return float(np.max(num / den))


ROW_TOL_BF16 = 3e-2


def max_abs(got, want) -> float:
    return float(np.max(np.abs(np.asarray(got, np.float64) - np.asarray(want, np.float64))))


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def positions(w):
    """(GPU positions [3, S] int32 on cuda, oracle positions int64 [3, S])."""
    m = q3()
    tt = torch.tensor(syn.token_types(w), dtype=torch.uint8, device="cuda")
    g = syn.grids(w)
    gd = torch.tensor(g, dtype=torch.int32, device="cuda").reshape(-1, 3) if g else None
    pos, nxt = m.mrope_positions(tt, gd)
    ref, ref_next = O.mrope_positions_tokens(syn.token_types(w), g)
    return pos, ref, nxt, ref_next


def layer_on_device(w, layer=0, zero=()):
    """(raw host weights, packed device layer)."""
    m = q3()
    raw = syn.layer_weights(w, layer, "cpu", zero)
    dev = {k: v.cuda().contiguous() for k, v in raw.items()}
    return raw, m.pack_layer(m.config_of(w), dev)


def tolerance(w):
    """(rel L2 bound, max-abs bound or None) on the layer output."""
    return (1e-5, 1e-4) if w.dtype == "fp32" else (1e-2, None)
