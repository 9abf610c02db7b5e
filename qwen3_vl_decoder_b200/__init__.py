"""qwen3_vl_decoder_b200: the Qwen3-VL text decoder on B200 (sm_100a).

The full-sequence causal prefill of a layer or a stack, a KV cache written by
the prefill with one-token decode against it, and the steps either side: the
token-embedding gather with the soft-token splice, and the final norm + LM head.

A thin torch-facing binding of libq3vl's C ABI (include/q3vl.h). torch only
provides device memory and the current stream; every step runs in the
library's CUDA kernels, and there is no other implementation to fall back
to: without the built library, the first call raises ImportError.
"""
from __future__ import annotations

import ctypes
from typing import Dict, List, Optional, Sequence

import torch

from . import _abi
from ._abi import Config, KvCache as KvCacheStruct, Layer, RawWeights  # noqa: F401

_lib_handle: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """The loaded libq3vl (loaded on first use; raises ImportError if not built)."""
    global _lib_handle
    if _lib_handle is None:
        _lib_handle = _abi.load()
    return _lib_handle

RAW_NAMES = ("attn_norm", "wq", "wk", "wv", "bq", "bk", "bv", "q_norm", "k_norm", "wo",
             "ffn_norm", "wg", "wu", "wd")


class Q3VLError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{_abi.STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


def version() -> str:
    return lib().q3vl_version().decode()


def _check(rc: int) -> None:
    if rc != _abi.OK:
        raise Q3VLError(rc, lib().q3vl_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def config(hidden, n_heads, n_kv_heads, intermediate, dtype="bf16", qkv_bias=False,
           head_dim=128, rope_theta=5e6, rms_eps=1e-6, mrope_section=(24, 20, 20)) -> Config:
    c = Config()
    c.hidden, c.n_heads, c.n_kv_heads, c.head_dim = hidden, n_heads, n_kv_heads, head_dim
    c.intermediate = intermediate
    c.dtype = _abi.DTYPE_BF16 if dtype == "bf16" else _abi.DTYPE_FP32
    c.has_qkv_bias = int(bool(qkv_bias))
    c.mrope_section[:] = list(mrope_section)
    c.rope_theta, c.rms_eps = float(rope_theta), float(rms_eps)
    return c


def config_of(w) -> Config:
    """Config of a q3vl_synth.Workload (or any object with the same fields)."""
    return config(w.hidden, w.n_heads, w.n_kv_heads, w.intermediate, w.dtype, w.qkv_bias,
                  w.head_dim, w.rope_theta, w.rms_eps, w.mrope_section)


def torch_dtype(cfg: Config) -> torch.dtype:
    return torch.bfloat16 if cfg.dtype == _abi.DTYPE_BF16 else torch.float32


class PackedLayer:
    """A packed layer: the device buffer plus the views the library reads."""

    def __init__(self, buf: torch.Tensor, views: Layer):
        self.buf = buf
        self.views = views


def packed_layer_bytes(cfg: Config) -> int:
    return int(lib().q3vl_packed_layer_bytes(ctypes.byref(cfg)))


def pack_layer(cfg: Config, raw: Dict[str, torch.Tensor], stream=None) -> PackedLayer:
    """Packs raw layer weights (device tensors in the config dtype)."""
    n = packed_layer_bytes(cfg)
    if n == 0:
        _check(_abi.EINVAL)
    dev = raw["wq"].device
    buf = torch.empty(n, dtype=torch.uint8, device=dev)
    rw = RawWeights()
    for name in RAW_NAMES:
        t = raw.get(name)
        if t is not None:
            assert t.is_contiguous() and t.dtype == torch_dtype(cfg), name
        setattr(rw, name, None if t is None else t.data_ptr())
    views = Layer()
    _check(lib().q3vl_pack_layer(ctypes.byref(cfg), ctypes.byref(rw), _ptr(buf), n,
                                ctypes.byref(views), _stream(stream)))
    return PackedLayer(buf, views)


def mrope_positions(token_types: torch.Tensor, grids: Optional[torch.Tensor], stream=None,
                    check: bool = True):
    """P0: (t, h, w) positions [3, S] int32 and the next position.

    token_types: device uint8 [S] (0 text, 1 image); grids: device int32
    [n, 3] (t, merged rows, merged cols) or None. With ``check`` the call
    synchronises and raises on a grid/run mismatch.
    """
    S = token_types.numel()
    dev = token_types.device
    pos = torch.empty((3, S), dtype=torch.int32, device=dev)
    info = torch.empty(2, dtype=torch.int32, device=dev)
    n = 0 if grids is None else grids.shape[0]
    _check(lib().q3vl_mrope_positions(_ptr(token_types), S, _ptr(grids) if n else None, n,
                                     _ptr(pos), _ptr(info), _stream(stream)))
    if not check:
        return pos, info
    st, nxt = (int(v) for v in info.cpu())
    if st != _abi.OK:
        raise Q3VLError(st, "image placeholders and grids disagree")
    return pos, nxt


def workspace_bytes(cfg: Config, S: int) -> int:
    return int(lib().q3vl_workspace_bytes(ctypes.byref(cfg), S))


def workspace(cfg: Config, S: int, device="cuda") -> torch.Tensor:
    n = workspace_bytes(cfg, S)
    if n == 0:
        _check(_abi.EINVAL)
    return torch.empty(n, dtype=torch.uint8, device=device)


def layer_prefill(cfg: Config, layer: PackedLayer, x: torch.Tensor, pos: torch.Tensor,
                  ds_slab: Optional[torch.Tensor] = None, ds_rows: Optional[torch.Tensor] = None,
                  ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One decoder layer in place on x [S, H]; returns x."""
    S = x.shape[0]
    ws = workspace(cfg, S, x.device) if ws is None else ws
    n_img = 0 if ds_rows is None else ds_rows.numel()
    _check(lib().q3vl_layer_prefill(ctypes.byref(cfg), ctypes.byref(layer.views), _ptr(x), S,
                                   _ptr(pos), _ptr(ds_slab), _ptr(ds_rows), n_img, _ptr(ws),
                                   ws.numel(), _stream(stream)))
    return x


def layer_prefill_noalloc(cfg: Config, layer: PackedLayer, x: torch.Tensor, pos: torch.Tensor,
                          ds_slab: Optional[torch.Tensor] = None,
                          ds_rows: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """layer_prefill with the library's built-in 64 MiB scratch instead of a workspace,
    for callers that cannot allocate device memory; calls must not overlap."""
    n_img = 0 if ds_rows is None else ds_rows.numel()
    _check(lib().q3vl_layer_prefill_noalloc(ctypes.byref(cfg), ctypes.byref(layer.views), _ptr(x),
                                            x.shape[0], _ptr(pos), _ptr(ds_slab), _ptr(ds_rows),
                                            n_img, _stream(stream)))
    return x


def stack_prefill(cfg: Config, layers: Sequence[PackedLayer], x: torch.Tensor, pos: torch.Tensor,
                  final_norm: Optional[torch.Tensor] = None,
                  ds_slabs: Sequence[torch.Tensor] = (), ds_rows: Optional[torch.Tensor] = None,
                  ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """n layers, DeepStack, optional final norm, in place on x; returns x."""
    S = x.shape[0]
    ws = workspace(cfg, S, x.device) if ws is None else ws
    arr = (Layer * len(layers))(*[l.views for l in layers])
    slabs = (ctypes.c_void_p * max(1, len(ds_slabs)))(*[s.data_ptr() for s in ds_slabs])
    n_img = 0 if ds_rows is None else ds_rows.numel()
    _check(lib().q3vl_stack_prefill(ctypes.byref(cfg), len(layers), arr, _ptr(final_norm), _ptr(x),
                                   S, _ptr(pos), slabs if ds_slabs else None, len(ds_slabs),
                                   _ptr(ds_rows), n_img, _ptr(ws), ws.numel(), _stream(stream)))
    return x


# ---------------------------------------------------------------------------
# KV cache and one-token decode (bf16)
# ---------------------------------------------------------------------------
class KvCache:
    """One layer's cache: k and v bf16 [n_seq, cap, nkv*128] on the device (K after the
    per-head norm and MRoPE, as the prefill forms it)."""

    def __init__(self, cfg: Config, n_seq: int, cap: int, device="cuda"):
        dkv = cfg.n_kv_heads * cfg.head_dim
        self.k = torch.zeros((n_seq, cap, dkv), dtype=torch.bfloat16, device=device)
        self.v = torch.zeros_like(self.k)
        self.struct = KvCacheStruct(self.k.data_ptr(), self.v.data_ptr(), cap, n_seq)

    @property
    def cap(self) -> int:
        return int(self.struct.cap)


def kv_caches(cfg: Config, n_layers: int, n_seq: int, cap: int, device="cuda") -> List[KvCache]:
    return [KvCache(cfg, n_seq, cap, device) for _ in range(n_layers)]


def _kv_array(kvs: Sequence[KvCache]):
    return (KvCacheStruct * len(kvs))(*[kv.struct for kv in kvs])


def layer_prefill_kv(cfg: Config, layer: PackedLayer, x: torch.Tensor, pos: torch.Tensor,
                     kv: KvCache, seq: int = 0, ds_slab: Optional[torch.Tensor] = None,
                     ds_rows: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """layer_prefill that also writes rows 0..S-1 of cache slot `seq`."""
    S = x.shape[0]
    ws = workspace(cfg, S, x.device) if ws is None else ws
    n_img = 0 if ds_rows is None else ds_rows.numel()
    _check(lib().q3vl_layer_prefill_kv(ctypes.byref(cfg), ctypes.byref(layer.views), _ptr(x), S,
                                      _ptr(pos), _ptr(ds_slab), _ptr(ds_rows), n_img,
                                      ctypes.byref(kv.struct), seq, _ptr(ws), ws.numel(),
                                      _stream(stream)))
    return x


def stack_prefill_kv(cfg: Config, layers: Sequence[PackedLayer], x: torch.Tensor,
                     pos: torch.Tensor, kvs: Sequence[KvCache], seq: int = 0,
                     final_norm: Optional[torch.Tensor] = None,
                     ds_slabs: Sequence[torch.Tensor] = (), ds_rows: Optional[torch.Tensor] = None,
                     ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """stack_prefill that also writes each layer's rows 0..S-1 of cache slot `seq`."""
    S = x.shape[0]
    ws = workspace(cfg, S, x.device) if ws is None else ws
    arr = (Layer * len(layers))(*[l.views for l in layers])
    slabs = (ctypes.c_void_p * max(1, len(ds_slabs)))(*[s.data_ptr() for s in ds_slabs])
    n_img = 0 if ds_rows is None else ds_rows.numel()
    _check(lib().q3vl_stack_prefill_kv(ctypes.byref(cfg), len(layers), arr, _ptr(final_norm),
                                      _ptr(x), S, _ptr(pos), slabs if ds_slabs else None,
                                      len(ds_slabs), _ptr(ds_rows), n_img, _kv_array(kvs), seq,
                                      _ptr(ws), ws.numel(), _stream(stream)))
    return x


def decode_workspace_bytes(cfg: Config, B: int, cap: int) -> int:
    return int(lib().q3vl_decode_workspace_bytes(ctypes.byref(cfg), B, cap))


def decode_workspace(cfg: Config, B: int, cap: int, device="cuda") -> torch.Tensor:
    n = decode_workspace_bytes(cfg, B, cap)
    if n == 0:
        _check(_abi.EINVAL)
    return torch.empty(n, dtype=torch.uint8, device=device)


def layer_decode(cfg: Config, layer: PackedLayer, x: torch.Tensor, pos: torch.Tensor,
                 kv: KvCache, seq: torch.Tensor, lens: torch.Tensor,
                 ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One new token per sequence (x [B, H] in place): token b's K/V go to row lens[b] of
    slot seq[b], and it attends to rows 0..lens[b] of that slot."""
    B = x.shape[0]
    ws = decode_workspace(cfg, B, kv.cap, x.device) if ws is None else ws
    _check(lib().q3vl_layer_decode(ctypes.byref(cfg), ctypes.byref(layer.views), _ptr(x), B,
                                  _ptr(pos), ctypes.byref(kv.struct), _ptr(seq), _ptr(lens),
                                  _ptr(ws), ws.numel(), _stream(stream)))
    return x


def stack_decode(cfg: Config, layers: Sequence[PackedLayer], x: torch.Tensor, pos: torch.Tensor,
                 kvs: Sequence[KvCache], seq: torch.Tensor, lens: torch.Tensor,
                 final_norm: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    """layer_decode through every layer, then the optional final norm; x in place."""
    B = x.shape[0]
    cap = max(kv.cap for kv in kvs)
    ws = decode_workspace(cfg, B, cap, x.device) if ws is None else ws
    arr = (Layer * len(layers))(*[l.views for l in layers])
    _check(lib().q3vl_stack_decode(ctypes.byref(cfg), len(layers), arr, _ptr(final_norm), _ptr(x),
                                  B, _ptr(pos), _kv_array(kvs), _ptr(seq), _ptr(lens), _ptr(ws),
                                  ws.numel(), _stream(stream)))
    return x


def decode_advance(pos: torch.Tensor, lens: torch.Tensor, stream=None) -> None:
    """lens += 1 and every position axis += 1 (the next text token), on the device."""
    _check(lib().q3vl_decode_advance(lens.numel(), _ptr(pos), _ptr(lens), _stream(stream)))


# ---------------------------------------------------------------------------
# Embedding gather (+ soft-token splice) and LM head
# ---------------------------------------------------------------------------
def embed(cfg: Config, table: torch.Tensor, tokens: torch.Tensor,
          soft: Optional[torch.Tensor] = None, soft_rows: Optional[torch.Tensor] = None,
          x: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """x[p] = table[tokens[p]], then x[soft_rows[k]] = soft[k]; returns x [S, H]."""
    S = tokens.numel()
    x = torch.empty((S, cfg.hidden), dtype=table.dtype, device=table.device) if x is None else x
    n_soft = 0 if soft_rows is None else soft_rows.numel()
    ws = torch.empty(max(1, 4 * S), dtype=torch.uint8, device=table.device) if n_soft else None
    _check(lib().q3vl_embed(ctypes.byref(cfg), _ptr(table), table.shape[0], _ptr(tokens), S,
                           _ptr(soft), _ptr(soft_rows), n_soft, _ptr(x), _ptr(ws),
                           0 if ws is None else ws.numel(), _stream(stream)))
    return x


def lm_head(cfg: Config, x_rows: torch.Tensor, final_norm: Optional[torch.Tensor],
            weight: torch.Tensor, logits: Optional[torch.Tensor] = None,
            ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """logits [B, vocab] fp32 = RMSNorm(x_rows, final_norm) weight^T (weight: [vocab, H])."""
    B, vocab = x_rows.shape[0], weight.shape[0]
    if logits is None:
        logits = torch.empty((B, vocab), dtype=torch.float32, device=x_rows.device)
    if ws is None:
        n = int(lib().q3vl_lm_head_workspace_bytes(ctypes.byref(cfg), B))
        if n == 0:
            _check(_abi.EINVAL)
        ws = torch.empty(n, dtype=torch.uint8, device=x_rows.device)
    _check(lib().q3vl_lm_head(ctypes.byref(cfg), _ptr(x_rows), B, _ptr(final_norm), _ptr(weight),
                             vocab, _ptr(logits), _ptr(ws), ws.numel(), _stream(stream)))
    return logits


# ---------------------------------------------------------------------------
# Step-level calls
# ---------------------------------------------------------------------------
def rope_table(cfg: Config, pos: torch.Tensor, stream=None) -> torch.Tensor:
    S = pos.shape[1]
    cs = torch.empty((S, 64, 2), dtype=torch.float32, device=pos.device)
    _check(lib().q3vl_rope_table(ctypes.byref(cfg), _ptr(pos), S, _ptr(cs), _stream(stream)))
    return cs


def rms_rowstat(cfg: Config, x: torch.Tensor, stream=None) -> torch.Tensor:
    S, width = x.shape
    inv = torch.empty(S, dtype=torch.float32, device=x.device)
    _check(lib().q3vl_rms_rowstat(ctypes.byref(cfg), _ptr(x), S, width, _ptr(inv),
                                 _stream(stream)))
    return inv


def _qkv_dim(cfg: Config) -> int:
    return (cfg.n_heads + 2 * cfg.n_kv_heads) * cfg.head_dim


def qkv_proj(cfg, layer: PackedLayer, x, inv_rms, cos_sin, ws=None, stream=None) -> torch.Tensor:
    S = x.shape[0]
    ws = workspace(cfg, S, x.device) if ws is None else ws
    qkv = torch.empty((S, _qkv_dim(cfg)), dtype=x.dtype, device=x.device)
    _check(lib().q3vl_qkv_proj(ctypes.byref(cfg), ctypes.byref(layer.views), _ptr(x), S,
                              _ptr(inv_rms), _ptr(cos_sin), _ptr(qkv), _ptr(ws), ws.numel(),
                              _stream(stream)))
    return qkv


def attention(cfg, qkv, stream=None) -> torch.Tensor:
    S = qkv.shape[0]
    o = torch.empty((S, cfg.n_heads * cfg.head_dim), dtype=qkv.dtype, device=qkv.device)
    _check(lib().q3vl_attention(ctypes.byref(cfg), _ptr(qkv), S, _ptr(o), _stream(stream)))
    return o


def o_proj(cfg, layer: PackedLayer, o, x, ws=None, stream=None) -> torch.Tensor:
    S = o.shape[0]
    ws = workspace(cfg, S, o.device) if ws is None else ws
    h = torch.empty((S, cfg.hidden), dtype=o.dtype, device=o.device)
    _check(lib().q3vl_o_proj(ctypes.byref(cfg), ctypes.byref(layer.views), _ptr(o), _ptr(x), S,
                            _ptr(h), _ptr(ws), ws.numel(), _stream(stream)))
    return h


def gate_up(cfg, layer: PackedLayer, h, inv_rms2, ws=None, stream=None) -> torch.Tensor:
    S = h.shape[0]
    ws = workspace(cfg, S, h.device) if ws is None else ws
    act = torch.empty((S, cfg.intermediate), dtype=h.dtype, device=h.device)
    _check(lib().q3vl_gate_up(ctypes.byref(cfg), ctypes.byref(layer.views), _ptr(h), S,
                             _ptr(inv_rms2), _ptr(act), _ptr(ws), ws.numel(), _stream(stream)))
    return act


def down(cfg, layer: PackedLayer, act, h, ds_slab=None, ds_map=None, ws=None,
         stream=None) -> torch.Tensor:
    S = act.shape[0]
    ws = workspace(cfg, S, act.device) if ws is None else ws
    out = torch.empty((S, cfg.hidden), dtype=act.dtype, device=act.device)
    _check(lib().q3vl_down(ctypes.byref(cfg), ctypes.byref(layer.views), _ptr(act), _ptr(h), S,
                          _ptr(ds_slab), _ptr(ds_map), _ptr(out), _ptr(ws), ws.numel(),
                          _stream(stream)))
    return out


def deepstack_map(ds_rows: torch.Tensor, S: int, stream=None) -> torch.Tensor:
    m = torch.empty(S, dtype=torch.int32, device=ds_rows.device)
    _check(lib().q3vl_deepstack_map(_ptr(ds_rows), ds_rows.numel(), S, _ptr(m), _stream(stream)))
    return m


def final_norm(cfg, x, gain, stream=None) -> torch.Tensor:
    _check(lib().q3vl_final_norm(ctypes.byref(cfg), _ptr(x), x.shape[0], _ptr(gain),
                                _stream(stream)))
    return x


def device_status(stream=None):
    """Synchronises and returns (code, where) of the device error record, clearing it."""
    code, where = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(lib().q3vl_device_status(_stream(stream), ctypes.byref(code), ctypes.byref(where)))
    return code.value, where.value


def check_device(stream=None) -> None:
    code, where = device_status(stream)
    if code != _abi.OK:
        raise Q3VLError(code, f"device-side error at location {where}")


def selftest_wait_timeout(timeout_us: int, stream=None) -> None:
    _check(lib().q3vl_selftest_wait_timeout(timeout_us, _stream(stream)))


def set_stage_events(events) -> None:
    """Records the 9 stage-boundary events in each following layer_prefill call
    (torch.cuda.Event(enable_timing=True) objects); None stops recording."""
    if events is None:
        _check(lib().q3vl_set_stage_events(None, 0))
        return
    for e in events:
        if e.cuda_event == 0:
            e.record()  # torch creates the CUDA event on first record
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    _check(lib().q3vl_set_stage_events(arr, len(events)))


def launch_count() -> int:
    """Kernels enqueued by the library so far in this process."""
    return int(lib().q3vl_launch_count())
