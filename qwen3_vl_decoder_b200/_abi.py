"""ctypes declarations of libq3vl's C ABI (include/q3vl.h).

Argument marshalling only: every computation runs in the library's CUDA
kernels. Loading fails loudly when the shared library is missing.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# Q3VL_LIBRARY=debug selects the bounds-checked debug build (libq3vl_debug.so)
LIB_PATH = os.path.join(_HERE, "libq3vl_debug.so" if os.environ.get("Q3VL_LIBRARY") == "debug"
                        else "libq3vl.so")

OK, EINVAL, ERANGE, EGRID, EDEEPSTACK, EWORKSPACE, ECUDA, ETIMEOUT, EUNSUPPORTED = \
    0, -1, -2, -3, -4, -5, -6, -7, -8
STATUS_NAMES = {OK: "Q3VL_OK", EINVAL: "Q3VL_EINVAL", ERANGE: "Q3VL_ERANGE",
                EGRID: "Q3VL_EGRID", EDEEPSTACK: "Q3VL_EDEEPSTACK",
                EWORKSPACE: "Q3VL_EWORKSPACE", ECUDA: "Q3VL_ECUDA",
                ETIMEOUT: "Q3VL_ETIMEOUT", EUNSUPPORTED: "Q3VL_EUNSUPPORTED"}
DTYPE_FP32, DTYPE_BF16 = 0, 1


class Config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("intermediate", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("has_qkv_bias", ctypes.c_int32), ("mrope_section", ctypes.c_int32 * 3),
                ("rope_theta", ctypes.c_double), ("rms_eps", ctypes.c_double)]


class RawWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "attn_norm", "wq", "wk", "wv", "bq", "bk", "bv", "q_norm", "k_norm", "wo",
        "ffn_norm", "wg", "wu", "wd")]


class Layer(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "w_qkv", "b_qkv", "q_norm", "k_norm", "w_o", "w_gu", "w_down")]


class KvCache(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("cap", ctypes.c_int64),
                ("n_seq", ctypes.c_int32)]


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32
_SZ = ctypes.c_size_t
_CFG = ctypes.POINTER(Config)

# name -> (restype, argtypes); mirrors include/q3vl.h
SIGNATURES = {
    "q3vl_packed_layer_bytes": (_SZ, [_CFG]),
    "q3vl_pack_layer": (ctypes.c_int, [_CFG, ctypes.POINTER(RawWeights), _P, _SZ,
                                       ctypes.POINTER(Layer), _P]),
    "q3vl_layer_views": (ctypes.c_int, [_CFG, _P, ctypes.POINTER(Layer)]),
    "q3vl_mrope_positions": (ctypes.c_int, [_P, _I64, _P, _I32, _P, _P, _P]),
    "q3vl_workspace_bytes": (_SZ, [_CFG, _I64]),
    "q3vl_layer_prefill": (ctypes.c_int, [_CFG, ctypes.POINTER(Layer), _P, _I64, _P, _P, _P, _I32,
                                          _P, _SZ, _P]),
    "q3vl_layer_prefill_noalloc": (ctypes.c_int, [_CFG, ctypes.POINTER(Layer), _P, _I64, _P, _P,
                                                  _P, _I32, _P]),
    "q3vl_stack_prefill": (ctypes.c_int, [_CFG, _I32, ctypes.POINTER(Layer), _P, _P, _I64, _P,
                                          ctypes.POINTER(_P), _I32, _P, _I32, _P, _SZ, _P]),
    "q3vl_rope_table": (ctypes.c_int, [_CFG, _P, _I64, _P, _P]),
    "q3vl_rms_rowstat": (ctypes.c_int, [_CFG, _P, _I64, _I64, _P, _P]),
    "q3vl_qkv_proj": (ctypes.c_int, [_CFG, ctypes.POINTER(Layer), _P, _I64, _P, _P, _P, _P, _SZ,
                                     _P]),
    "q3vl_attention": (ctypes.c_int, [_CFG, _P, _I64, _P, _P]),
    "q3vl_o_proj": (ctypes.c_int, [_CFG, ctypes.POINTER(Layer), _P, _P, _I64, _P, _P, _SZ, _P]),
    "q3vl_gate_up": (ctypes.c_int, [_CFG, ctypes.POINTER(Layer), _P, _I64, _P, _P, _P, _SZ, _P]),
    "q3vl_down": (ctypes.c_int, [_CFG, ctypes.POINTER(Layer), _P, _P, _I64, _P, _P, _P, _P, _SZ,
                                 _P]),
    "q3vl_deepstack_map": (ctypes.c_int, [_P, _I32, _I64, _P, _P]),
    "q3vl_final_norm": (ctypes.c_int, [_CFG, _P, _I64, _P, _P]),
    "q3vl_layer_prefill_kv": (ctypes.c_int, [_CFG, ctypes.POINTER(Layer), _P, _I64, _P, _P, _P,
                                             _I32, ctypes.POINTER(KvCache), _I32, _P, _SZ, _P]),
    "q3vl_stack_prefill_kv": (ctypes.c_int, [_CFG, _I32, ctypes.POINTER(Layer), _P, _P, _I64, _P,
                                             ctypes.POINTER(_P), _I32, _P, _I32,
                                             ctypes.POINTER(KvCache), _I32, _P, _SZ, _P]),
    "q3vl_decode_workspace_bytes": (_SZ, [_CFG, _I32, _I64]),
    "q3vl_layer_decode": (ctypes.c_int, [_CFG, ctypes.POINTER(Layer), _P, _I32, _P,
                                         ctypes.POINTER(KvCache), _P, _P, _P, _SZ, _P]),
    "q3vl_stack_decode": (ctypes.c_int, [_CFG, _I32, ctypes.POINTER(Layer), _P, _P, _I32, _P,
                                         ctypes.POINTER(KvCache), _P, _P, _P, _SZ, _P]),
    "q3vl_decode_advance": (ctypes.c_int, [_I32, _P, _P, _P]),
    "q3vl_embed": (ctypes.c_int, [_CFG, _P, _I64, _P, _I64, _P, _P, _I32, _P, _P, _SZ, _P]),
    "q3vl_lm_head_workspace_bytes": (_SZ, [_CFG, _I32]),
    "q3vl_lm_head": (ctypes.c_int, [_CFG, _P, _I32, _P, _P, _I64, _P, _P, _SZ, _P]),
    "q3vl_device_status": (ctypes.c_int, [_P, ctypes.POINTER(_I32), ctypes.POINTER(_I32)]),
    "q3vl_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_uint32, _P]),
    "q3vl_set_stage_events": (ctypes.c_int, [ctypes.POINTER(_P), _I32]),
    "q3vl_launch_count": (ctypes.c_uint64, []),
    "q3vl_last_error": (ctypes.c_char_p, []),
    "q3vl_version": (ctypes.c_char_p, []),
}


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{os.path.basename(path)} is not built ({path}); run "
                          "`python -m qwen3_vl_decoder_b200.build`"
                          + (" --debug" if path.endswith("_debug.so") else ""))
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib
