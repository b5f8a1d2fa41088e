"""ctypes view of include/krea_attn.h: the library handle and the params struct.

Marshalling only. The shared library is built in-tree (build.py); when it is
missing this module raises instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

LIB_PATH = Path(__file__).resolve().parent / "libkrea_attn.so"

ABI_VERSION = 3
TILE = 128

MODE = {"dense": 0, "tilemix": 1, "scanline": 2}
DTYPE = {"f16": 0, "bf16": 1, "f32": 2}
PATTERN = {"zero": 0, "band": 1, "one": 2}

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_WORKSPACE = -3
ERR_CUDA = -4
ERR_DEVICE_TIMEOUT = -5
ERR_DEVICE_BOUNDS = -6
ERR_NO_DEVICE = -7
ERR_TOO_LARGE = -8

KIND_MASKED = 1
KIND_INT8 = 2


class Params(ctypes.Structure):
    """krea_attn_params_t."""

    _fields_ = [
        ("abi_version", ctypes.c_int32),
        ("batch", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("q_start", ctypes.c_int32),
        ("q_len", ctypes.c_int32),
        ("in_dtype", ctypes.c_int32),
        ("out_dtype", ctypes.c_int32),
        ("q_stride", ctypes.c_int64 * 3),
        ("k_stride", ctypes.c_int64 * 3),
        ("v_stride", ctypes.c_int64 * 3),
        ("gate_stride", ctypes.c_int64 * 3),
        ("out_stride", ctypes.c_int64 * 3),
        ("softmax_scale", ctypes.c_float),
        ("pattern", ctypes.c_int32),
        ("percentage", ctypes.c_float),
        ("band_blocks", ctypes.c_int32),
        ("smooth_k", ctypes.c_int32),
        ("qk_fp32_accumulate", ctypes.c_int32),
        ("window", ctypes.c_int32),
        ("tile_aligned", ctypes.c_int32),
        ("text_pad", ctypes.c_int32),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("status", ctypes.c_void_p),
        ("debug_wait_limit", ctypes.c_int64),
        ("debug_flags", ctypes.c_int32),
        ("lse", ctypes.c_void_p),
        ("overlap_previous", ctypes.c_int32),
    ]


class RopeParams(ctypes.Structure):
    """krea_rope_params_t."""

    _fields_ = [("axes_dim", ctypes.c_int32 * 3), ("theta", ctypes.c_float), ("eps", ctypes.c_float)]


EXCHANGE_MAX_RANKS = 16
IPC_HANDLE_BYTES = 64


class Exchange(ctypes.Structure):
    """krea_exchange_t."""

    _fields_ = [
        ("world", ctypes.c_int32),
        ("rank", ctypes.c_int32),
        ("tokens_per_rank", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
        ("dst", ctypes.c_void_p * EXCHANGE_MAX_RANKS),
        ("dst_stride", ctypes.c_int64 * 3),
    ]


class WsLayout(ctypes.Structure):
    """krea_attn_ws_layout_t."""

    _fields_ = [(n, ctypes.c_size_t) for n in ("kc", "q8", "k8", "sq", "sk", "mu", "part", "total")]


# Every entry point include/krea_attn.h declares, with its ctypes signature.
_P = ctypes.POINTER(Params)
_VP = ctypes.c_void_p
_I = ctypes.c_int
SIGNATURES = {
    "krea_attn_default_params": (None, [_P, _I, _I, _I, _I, _I, _I, _I]),
    "krea_attn_fwd": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _P, _VP]),
    "krea_attn_fwd_noalloc": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _P, _VP]),
    "krea_attn_fwd_rope_q": (_I, [_VP, _VP, _VP, ctypes.POINTER(RopeParams), _VP, _VP, _VP, _VP, _I, _I, _I, _I,
                                  _P, _VP]),
    "krea_attn_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _P]),
    "krea_attn_workspace_layout": (_I, [_I, _I, _I, _I, _P, ctypes.POINTER(WsLayout)]),
    "krea_attn_map_size": (_I, [_I, _I, _I, _I, _P, ctypes.POINTER(ctypes.c_int32),
                                ctypes.POINTER(ctypes.c_int32)]),
    "krea_attn_get_map": (_I, [_I, _I, _I, _I, _P, _VP, _VP, _VP, ctypes.c_int32]),
    "krea_attn_quantize": (_I, [_VP, _VP, _I, _I, _I, _P, _VP]),
    "krea_attn_build_map_device": (_I, [_I, _I, _I, _I, _P, _VP, _VP, _VP, ctypes.c_int32, _VP]),
    "krea_attn_default_rope": (None, [ctypes.POINTER(RopeParams), _I]),
    "krea_attn_bwd_scratch_bytes": (ctypes.c_size_t, [_I, _I, _I, _P]),
    "krea_attn_bwd": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _P, _VP]),
    "krea_attn_rope_positions": (_I, [_I, _I, _I, _VP, ctypes.c_int32]),
    "krea_attn_rope_table": (_I, [_VP, _I, ctypes.POINTER(RopeParams), _VP, _VP]),
    "krea_attn_qk_prologue": (_I, [_VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_int64),
                                   ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(RopeParams), _VP, _VP, _VP]),
    "krea_attn_seq_to_heads": (_I, [_VP, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_int64),
                                    ctypes.POINTER(Exchange), _VP]),
    "krea_attn_heads_to_seq": (_I, [_VP, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_int64),
                                    ctypes.POINTER(Exchange), _VP]),
    "krea_attn_qk_prologue_to_heads": (_I, [_VP, _VP, _VP, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_int64),
                                            ctypes.POINTER(RopeParams), ctypes.POINTER(Exchange), _VP]),
    "krea_attn_ipc_alloc": (_I, [ctypes.c_size_t, ctypes.POINTER(ctypes.c_void_p), _VP]),
    "krea_attn_ipc_free": (_I, [_VP]),
    "krea_attn_ipc_open": (_I, [_VP, ctypes.POINTER(ctypes.c_void_p)]),
    "krea_attn_ipc_close": (_I, [_VP]),
    "krea_attn_clear_cache": (None, []),
    "krea_attn_error_string": (ctypes.c_char_p, [_I]),
    "krea_attn_abi_version": (_I, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise RuntimeError(
                f"{LIB_PATH.name} is not built; run diffusion_transformer_attention_bidirectional_b200/build.py")
        handle = ctypes.CDLL(str(LIB_PATH))
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        if handle.krea_attn_abi_version() != ABI_VERSION:
            raise RuntimeError("libkrea_attn.so ABI version mismatch")
        _lib = handle
    return _lib


class KreaError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        msg = lib().krea_attn_error_string(code).decode()
        super().__init__(f"{what}: {msg} ({code})" if what else f"{msg} ({code})")
        self.code = code


def check(code: int, what: str = "") -> None:
    if code != OK:
        raise KreaError(code, what)
