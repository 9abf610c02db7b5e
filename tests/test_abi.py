"""The C-ABI library loads and exports every symbol the header declares (no GPU).

Only host-side paths are exercised here: size queries and argument
validation, which return before any CUDA call.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "q3vl.h")


@pytest.fixture(scope="module")
def lib():
    from qwen3_vl_decoder_b200 import build
    build.build()
    from qwen3_vl_decoder_b200 import _abi
    return _abi.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(q3vl_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_three_north_calls():
    names = declared_functions()
    for n in ("q3vl_mrope_positions", "q3vl_layer_prefill", "q3vl_stack_prefill"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_binding_covers_every_declared_symbol():
    from qwen3_vl_decoder_b200 import _abi
    assert set(declared_functions()) == set(_abi.SIGNATURES)


def _cfg(**kw):
    from qwen3_vl_decoder_b200 import config
    base = dict(hidden=2560, n_heads=32, n_kv_heads=8, intermediate=9728, dtype="bf16",
                qkv_bias=True)
    base.update(kw)
    return config(**base)


def test_sizes(lib):
    c = _cfg()
    H, Dq, Dkv, I = 2560, 4096, 1024, 9728
    packed = lib.q3vl_packed_layer_bytes(ctypes.byref(c))
    assert packed >= 2 * ((Dq + 2 * Dkv) * H + H * Dq + 2 * I * H + H * I)
    S = 4096
    ws = lib.q3vl_workspace_bytes(ctypes.byref(c), S)
    sk = 148 * (128 * 256 * 4 + 4)   # stream-K partial tiles and flags (148 SMs)
    rowsq = 2 * S * (H // 128) * 4      # per-row sums of squares of h and x' (fused P7, P2)
    need = 2 * S * ((Dq + 2 * Dkv) + Dq + H + I) + S * (64 * 8 + 12) + sk + rowsq
    assert need <= ws <= need + 16 * 256
    assert lib.q3vl_workspace_bytes(ctypes.byref(c), 0) == 0
    assert lib.q3vl_packed_layer_bytes(ctypes.byref(_cfg(head_dim=64))) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=64), -8), (dict(hidden=100), -1), (dict(n_heads=6, n_kv_heads=4), -1),
    (dict(intermediate=100), -1), (dict(mrope_section=(16, 24, 24)), -8),
])
def test_bad_config_rejected(lib, kw, code):
    c = _cfg(**kw)
    rc = lib.q3vl_rope_table(ctypes.byref(c), ctypes.c_void_p(16), 8, ctypes.c_void_p(16), None)
    assert rc == code
    assert lib.q3vl_last_error()


def test_empty_sequence_rejected(lib):
    c = _cfg()
    from qwen3_vl_decoder_b200 import _abi
    lay = _abi.Layer(*[256] * 7)
    rc = lib.q3vl_layer_prefill(ctypes.byref(c), ctypes.byref(lay), ctypes.c_void_p(256), 0,
                                ctypes.c_void_p(256), None, None, 0, ctypes.c_void_p(256),
                                1 << 40, None)
    assert rc == -1 and b"empty" in lib.q3vl_last_error()


def test_small_workspace_rejected(lib):
    c = _cfg()
    from qwen3_vl_decoder_b200 import _abi
    lay = _abi.Layer(*[256] * 7)
    rc = lib.q3vl_layer_prefill(ctypes.byref(c), ctypes.byref(lay), ctypes.c_void_p(256), 16,
                                ctypes.c_void_p(256), None, None, 0, ctypes.c_void_p(256), 1024,
                                None)
    assert rc == -5


def test_deepstack_contract(lib):
    c = _cfg()
    from qwen3_vl_decoder_b200 import _abi
    lay = (_abi.Layer * 1)(_abi.Layer(*[256] * 7))
    big = 1 << 40
    slabs = (ctypes.c_void_p * 2)(256, 256)
    # fewer than three slabs
    rc = lib.q3vl_stack_prefill(ctypes.byref(c), 1, lay, None, ctypes.c_void_p(256), 16,
                                ctypes.c_void_p(256), slabs, 2, ctypes.c_void_p(256), 4,
                                ctypes.c_void_p(256), big, None)
    assert rc == -4
    slabs3 = (ctypes.c_void_p * 3)(256, 256, 256)
    # slabs without image rows
    rc = lib.q3vl_stack_prefill(ctypes.byref(c), 1, lay, None, ctypes.c_void_p(256), 16,
                                ctypes.c_void_p(256), slabs3, 3, None, 0,
                                ctypes.c_void_p(256), big, None)
    assert rc == -4
    # a layer with a slab but no rows
    rc = lib.q3vl_layer_prefill(ctypes.byref(c), lay, ctypes.c_void_p(256), 16,
                                ctypes.c_void_p(256), ctypes.c_void_p(256), None, 0,
                                ctypes.c_void_p(256), big, None)
    assert rc == -4


def test_positions_argument_checks(lib):
    rc = lib.q3vl_mrope_positions(ctypes.c_void_p(256), 0, None, 0, ctypes.c_void_p(256),
                                  ctypes.c_void_p(256), None)
    assert rc == -1
    rc = lib.q3vl_mrope_positions(ctypes.c_void_p(256), 8, None, 1, ctypes.c_void_p(256),
                                  ctypes.c_void_p(256), None)
    assert rc == -1


def _kv(cap=64, n_seq=2):
    from qwen3_vl_decoder_b200 import _abi
    return _abi.KvCache(256, 512, cap, n_seq)


def test_decode_workspace_sizes(lib):
    c = _cfg()
    H, Dq, I, nkv, G = 2560, 4096, 9728, 8, 4
    for B, cap in ((1, 4097), (40, 1000)):
        ws = lib.q3vl_decode_workspace_bytes(ctypes.byref(c), B, cap)
        # activations (bf16 q, o, h, act), rope table, attention chunk partials
        # (o[128], m, l per head over the chunk slots, rounded up to 4)
        nc_pad = (-(-cap // 128) + 3) // 4 * 4
        floor = 2 * B * (2 * Dq + H + I) + B * 64 * 8 + B * nkv * G * 130 * nc_pad * 4
        assert floor < ws < floor + 64 * 1024 * 1024
    assert lib.q3vl_decode_workspace_bytes(ctypes.byref(c), 0, 64) == 0
    assert lib.q3vl_decode_workspace_bytes(ctypes.byref(c), 257, 64) == 0
    assert lib.q3vl_decode_workspace_bytes(ctypes.byref(c), 1, 0) == 0
    assert lib.q3vl_decode_workspace_bytes(ctypes.byref(_cfg(dtype="fp32")), 1, 64) == 0
    assert lib.q3vl_decode_workspace_bytes(ctypes.byref(_cfg(n_heads=48, n_kv_heads=3)), 1, 64) == 0


def test_decode_argument_checks(lib):
    from qwen3_vl_decoder_b200 import _abi
    c = _cfg()
    lay = _abi.Layer(*[256] * 7)
    kv = _kv()
    P = ctypes.c_void_p(256)

    def dec(B=2, ws_bytes=1 << 40, kv_=kv, cfg=c):
        return lib.q3vl_layer_decode(ctypes.byref(cfg), ctypes.byref(lay), P, B, P,
                                     ctypes.byref(kv_), P, P, P, ws_bytes, None)
    assert dec(B=0) == -1
    assert dec(B=257) == -1
    assert dec(ws_bytes=1024) == -5
    assert dec(kv_=_kv(cap=0)) == -1
    assert dec(kv_=_kv(cap=131073)) == -8
    assert dec(kv_=_kv(cap=131072, n_seq=1 << 15)) == -1
    assert dec(cfg=_cfg(dtype="fp32")) == -8
    assert lib.q3vl_decode_advance(0, P, P, None) == -1
    # prefill into a cache: S above the capacity, or a slot outside [0, n_seq)
    pk = lambda S, seq: lib.q3vl_layer_prefill_kv(ctypes.byref(c), ctypes.byref(lay), P, S, P,
                                                  None, None, 0, ctypes.byref(kv), seq, P,
                                                  1 << 40, None)
    assert pk(65, 0) == -2
    assert pk(8, 2) == -2
    assert pk(8, -1) == -2


def test_embed_and_lm_head_argument_checks(lib):
    c = _cfg()
    P = ctypes.c_void_p(256)
    assert lib.q3vl_lm_head_workspace_bytes(ctypes.byref(c), 3) == 3 * 2560 * 2
    assert lib.q3vl_lm_head_workspace_bytes(ctypes.byref(c), 0) == 0
    assert lib.q3vl_lm_head_workspace_bytes(ctypes.byref(_cfg(dtype="fp32")), 1) == 0

    def head(cfg=c, B=1, vocab=1000, ws_bytes=1 << 20):
        return lib.q3vl_lm_head(ctypes.byref(cfg), P, B, None, P, vocab, P, P, ws_bytes, None)
    assert head(cfg=_cfg(dtype="fp32")) == -8
    assert head(B=0) == -1 and head(B=257) == -1
    assert head(vocab=0) == -1
    assert head(ws_bytes=100) == -5

    def emb(vocab=10, S=4, n_soft=0, ws=None, ws_bytes=0):
        return lib.q3vl_embed(ctypes.byref(c), P, vocab, P, S, P if n_soft else None,
                              P if n_soft else None, n_soft, P, ws, ws_bytes, None)
    assert emb(vocab=0) == -1
    assert emb(S=0) == -1
    assert emb(n_soft=-1) == -1
    assert emb(n_soft=2) == -5                                   # soft rows need the row map
    assert emb(n_soft=5, ws=P, ws_bytes=1024) == -2              # more soft rows than tokens
