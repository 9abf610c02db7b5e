"""Seeded synthetic inputs for the Qwen3-VL text-decoder prefill.

This module is shared by the CPU oracle and the CUDA path, and therefore
holds none of the method's arithmetic: only workload shapes, prompt layouts
(which tokens are text and which belong to an image grid) and seeded random
draws. Every tensor is drawn from its own ``torch.Generator`` seeded from
``(seed, layer, tensor id)`` so that any single layer can be regenerated on
its own, on the CPU or on the device.

Distributions follow the workload descriptions: weights N(0, 0.02), norm
gains 1 + N(0, 0.1), hidden input N(0, 1), Q/K/V bias N(0, 0.02), DeepStack
slabs N(0, 0.1) on image rows. bf16 workloads round every fp32 draw to the
nearest bf16 (round-to-nearest-even, as ``Tensor.to(torch.bfloat16)`` does).
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence, Tuple

import torch

TENSOR_IDS = {
    "attn_norm": 0, "wq": 1, "wk": 2, "wv": 3, "bq": 4, "bk": 5, "bv": 6,
    "q_norm": 7, "k_norm": 8, "wo": 9, "ffn_norm": 10, "wg": 11, "wu": 12,
    "wd": 13, "final_norm": 14, "x": 15, "slab": 16,
}


@dataclasses.dataclass(frozen=True)
class Workload:
    """One named workload: model shape, sequence layout and seed."""
    name: str
    hidden: int
    n_heads: int
    n_kv_heads: int
    intermediate: int
    seq: int
    n_layers: int
    dtype: str                      # "fp32" or "bf16"
    seed: int
    head_dim: int = 128
    rope_theta: float = 5e6
    rms_eps: float = 1e-6
    mrope_section: Tuple[int, int, int] = (24, 20, 20)
    qkv_bias: bool = False
    final_norm: bool = False
    # image spans as (first token index, merged grid rows, merged grid cols)
    images: Tuple[Tuple[int, int, int], ...] = ()
    deepstack_layers: int = 0       # DeepStack slabs added after layers 0..n-1

    @property
    def q_dim(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    def with_seq(self, seq: int, images=None) -> "Workload":
        return dataclasses.replace(self, seq=seq,
                                   images=self.images if images is None else tuple(images))

    def with_layers(self, n_layers: int) -> "Workload":
        return dataclasses.replace(self, n_layers=n_layers)


# The five workloads of the benchmark plan.
TINY_FP32 = Workload("tiny-fp32-layer", 512, 4, 2, 1536, 128, 1, "fp32", 0)
Q2B_LAYER = Workload("qwen3vl-2b-layer-s1024", 2048, 16, 8, 6144, 1024, 1, "bf16", 1)
Q2B_STACK = Workload("qwen3vl-2b-stack28-s2048", 2048, 16, 8, 6144, 2048, 28, "bf16", 2,
                     final_norm=True, images=((100, 16, 16),), deepstack_layers=3)
Q4B_LAYER = Workload("qwen3vl-4b-layer-s4096", 2560, 32, 8, 9728, 4096, 1, "bf16", 3,
                     qkv_bias=True, images=((512, 32, 24),))
Q32B_ENC = Workload("qwen3vl-32b-encoder50-s8192", 5120, 64, 8, 25600, 8192, 50, "bf16", 4)
Q32B_ENC_1064 = dataclasses.replace(Q32B_ENC, name="qwen3vl-32b-encoder50-s1064", seq=1064)

WORKLOADS = {w.name: w for w in (TINY_FP32, Q2B_LAYER, Q2B_STACK, Q4B_LAYER, Q32B_ENC,
                                  Q32B_ENC_1064)}

# Decode after a prompt: the 4B shape with its 36 layers, the prompt being the
# 4B layer workload's (512 text, a 32x24 image, 2816 text = 4096 rows).
Q4B_DECODE = Workload("qwen3vl-4b-stack36-decode-ctx4096", 2560, 32, 8, 9728, 4096, 36, "bf16",
                      3, qkv_bias=True, images=((512, 32, 24),))


def token_types(w: Workload) -> List[int]:
    """Per-token type: 0 = text, 1 = image placeholder (merged grid token)."""
    tt = [0] * w.seq
    for start, hm, wm in w.images:
        for i in range(start, start + hm * wm):
            tt[i] = 1
    return tt


def grids(w: Workload) -> List[Tuple[int, int, int]]:
    """The images' merged grids (t, rows, cols) in prompt order."""
    return [(1, hm, wm) for _, hm, wm in w.images]


def spans(w: Workload) -> List[Tuple[int, int, int, int]]:
    """Image spans as (start, length, merged rows, merged cols)."""
    return [(s, hm * wm, hm, wm) for s, hm, wm in w.images]


def image_rows(w: Workload) -> List[int]:
    """Token indices of image rows, in span order."""
    rows: List[int] = []
    for s, hm, wm in w.images:
        rows.extend(range(s, s + hm * wm))
    return rows


def _gen(seed: int, layer: int, tid: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + layer * 1_009 + tid * 7) & 0x7FFF_FFFF_FFFF)
    return g


def _draw(shape, seed, layer, name, device, mean=0.0, std=1.0) -> torch.Tensor:
    g = _gen(seed, layer, TENSOR_IDS[name], device)
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    return t.mul_(std).add_(mean)


def _cast(t: torch.Tensor, dtype: str) -> torch.Tensor:
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def layer_weights(w: Workload, layer: int, device="cpu", zero: Sequence[str] = ()) -> dict:
    """Raw (unpacked) weights of one layer in torch-Linear [out, in] layout.

    ``zero`` names tensors to replace by zeros (used by invariant tests).
    """
    H, Dq, Dkv, I, hd = w.hidden, w.q_dim, w.kv_dim, w.intermediate, w.head_dim
    shapes = {
        "attn_norm": ((H,), 1.0, 0.1), "wq": ((Dq, H), 0.0, 0.02),
        "wk": ((Dkv, H), 0.0, 0.02), "wv": ((Dkv, H), 0.0, 0.02),
        "q_norm": ((hd,), 1.0, 0.1), "k_norm": ((hd,), 1.0, 0.1),
        "wo": ((H, Dq), 0.0, 0.02), "ffn_norm": ((H,), 1.0, 0.1),
        "wg": ((I, H), 0.0, 0.02), "wu": ((I, H), 0.0, 0.02), "wd": ((H, I), 0.0, 0.02),
    }
    if w.qkv_bias:
        shapes.update({"bq": ((Dq,), 0.0, 0.02), "bk": ((Dkv,), 0.0, 0.02),
                       "bv": ((Dkv,), 0.0, 0.02)})
    out = {}
    for name, (shape, mean, std) in shapes.items():
        if name in zero:
            t = torch.zeros(*shape, device=device, dtype=torch.float32)
        else:
            t = _draw(shape, w.seed, layer, name, device, mean, std)
        out[name] = _cast(t, w.dtype)
    return out


def final_norm(w: Workload, device="cpu") -> Optional[torch.Tensor]:
    if not w.final_norm:
        return None
    return _cast(_draw((w.hidden,), w.seed, 0, "final_norm", device, 1.0, 0.1), w.dtype)


def hidden_input(w: Workload, device="cpu") -> torch.Tensor:
    """The layer / stack input x [S, H], N(0, 1)."""
    return _cast(_draw((w.seq, w.hidden), w.seed, 0, "x", device), w.dtype)


def deepstack_slabs(w: Workload, device="cpu") -> List[torch.Tensor]:
    """Compact DeepStack slabs, one [n_image_rows, H] tensor per injected layer."""
    n = len(image_rows(w))
    if n == 0 or w.deepstack_layers == 0:
        return []
    return [_cast(_draw((n, w.hidden), w.seed, l, "slab", device, 0.0, 0.1), w.dtype)
            for l in range(w.deepstack_layers)]
