"""ctypes binding of libedgerock.so (argument marshalling only).

Every function here converts torch CUDA tensors into the raw pointers, sizes
and stream that the C ABI in include/edgerock.h takes, calls it, and raises on
a non-zero return code.  No computation happens in Python, and there is no
fallback: if the library is missing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libedgerock.so")

ER_OK, ER_EINVAL, ER_ECAPACITY, ER_ECUDA, ER_EDEVICE, ER_ETIMEOUT = 0, -1, -2, -3, -4, -5

D, HIDDEN, NH, NG, WIN, BANK, PEND = 256, 2560, 16, 4, 1024, 1024, 256
QKV, OIN = 12288, 4096


class ERError(RuntimeError):
    def __init__(self, fn, code):
        self.code = code
        super().__init__(f"{fn} failed: {code} ({error_string(code)})")


class CState(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("win_k", "win_v", "bank_k", "bank_v", "pend_k",
                                               "pend_v", "bank_score", "pend_score", "bank_pos",
                                               "pend_pos", "meta", "dev_error")] + [
        ("s_max", ctypes.c_int32), ("n_layers", ctypes.c_int32), ("pool", ctypes.c_int32)]


ER_FLAG_RMA_OFF = 1  # the RMA switched off (the pages' ablation)
ER_STATE_POOL = 1    # the pooled anchor layout (a commit that moves no K/V row)


class CWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w_qkv", "w_o", "q_norm_swa", "k_norm_swa",
                                               "q_norm_rma", "k_norm_rma", "w1", "w2",
                                               "w1_split", "w_qkv_score")]


EXPORTS = {
    # name: (restype, argtypes)
    "er_state_bytes": (ctypes.c_size_t, [ctypes.c_int32, ctypes.c_int32]),
    "er_state_carve": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32,
                                      ctypes.c_int32, ctypes.POINTER(CState)]),
    "er_state_bytes_ex": (ctypes.c_size_t, [ctypes.c_int32, ctypes.c_int32, ctypes.c_uint32]),
    "er_state_carve_ex": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32,
                                         ctypes.c_int32, ctypes.c_uint32,
                                         ctypes.POINTER(CState)]),
    "er_state_init": (ctypes.c_int, [ctypes.POINTER(CState), ctypes.c_void_p, ctypes.c_int32,
                                     ctypes.c_void_p]),
    "er_advance": (ctypes.c_int, [ctypes.POINTER(CState), ctypes.c_void_p, ctypes.c_int32,
                                  ctypes.c_int32, ctypes.c_void_p]),
    "er_advance_ex": (ctypes.c_int, [ctypes.POINTER(CState), ctypes.c_void_p, ctypes.c_int32,
                                     ctypes.c_int32, ctypes.c_uint32, ctypes.c_void_p]),
    "er_last_device_error": (ctypes.c_int, [ctypes.POINTER(CState),
                                            ctypes.POINTER(ctypes.c_int32), ctypes.c_void_p]),
    "er_last_call_error": (ctypes.c_int, [ctypes.POINTER(ctypes.c_int32), ctypes.c_void_p]),
    "er_qk_norm_rope": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "er_linear_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int32, ctypes.c_int32,
                                                     ctypes.c_int32]),
    "er_linear": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32,
                                 ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                                 ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                 ctypes.c_void_p]),
    "er_score_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int32]),
    "er_score_split_w1": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "er_wait_selftest": (ctypes.c_int, [ctypes.POINTER(CState), ctypes.c_int32, ctypes.c_void_p]),
    "er_prepare_qkv_score": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                            ctypes.c_void_p]),
    "er_rma_score": (ctypes.c_int, [ctypes.POINTER(CWeights), ctypes.c_void_p, ctypes.c_int32,
                                    ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                    ctypes.c_void_p]),
    "er_rma_score_ex": (ctypes.c_int, [ctypes.POINTER(CWeights), ctypes.c_void_p,
                                       ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p]),
    "er_rma_score_noalloc": (ctypes.c_int, [ctypes.POINTER(CWeights), ctypes.c_void_p,
                                            ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]),
    "er_rma_append_pending": (ctypes.c_int, [ctypes.POINTER(CState), ctypes.c_int32,
                                             ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                             ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                             ctypes.c_void_p]),
    "er_rma_commit": (ctypes.c_int, [ctypes.POINTER(CState), ctypes.c_int32, ctypes.c_void_p,
                                     ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]),
    "er_attend_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int32]),
    "er_swa_rma_attend": (ctypes.c_int, [ctypes.POINTER(CState), ctypes.c_int32, ctypes.c_void_p,
                                         ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_size_t, ctypes.c_void_p]),
    "er_decode_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int32]),
    "er_swa_rma_decode": (ctypes.c_int, [ctypes.POINTER(CState), ctypes.POINTER(CWeights),
                                         ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32,
                                         ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_size_t, ctypes.c_void_p]),
    "er_swa_rma_decode_ex": (ctypes.c_int, [ctypes.POINTER(CState), ctypes.POINTER(CWeights),
                                            ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32,
                                            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                            ctypes.c_size_t, ctypes.c_uint32, ctypes.c_void_p]),
    "er_prefill_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int32]),
    "er_swa_rma_prefill_chunk": (ctypes.c_int, [ctypes.POINTER(CState),
                                                ctypes.POINTER(CWeights), ctypes.c_int32,
                                                ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32,
                                                ctypes.c_void_p, ctypes.c_void_p,
                                                ctypes.c_size_t, ctypes.c_void_p]),
    "er_swa_rma_prefill_chunk_ex": (ctypes.c_int, [ctypes.POINTER(CState),
                                                   ctypes.POINTER(CWeights), ctypes.c_int32,
                                                   ctypes.c_int32, ctypes.c_void_p,
                                                   ctypes.c_int32, ctypes.c_void_p,
                                                   ctypes.c_void_p, ctypes.c_size_t,
                                                   ctypes.c_uint32, ctypes.c_void_p]),
    "er_error_string": (ctypes.c_char_p, [ctypes.c_int]),
    "er_launch_count": (ctypes.c_uint64, []),
    "er_profile_enable": (ctypes.c_int, [ctypes.c_int]),
    "er_profile_read": (ctypes.c_int, [ctypes.POINTER(ctypes.c_double),
                                       ctypes.POINTER(ctypes.c_int64), ctypes.c_int]),
}

_lib = None


def lib():
    """Load libedgerock.so (raises if it has not been built: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m sliding_window_anchor_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in EXPORTS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def error_string(code: int) -> str:
    try:
        return lib().er_error_string(code).decode()
    except Exception:  # pragma: no cover
        return "?"


def check(fn: str, rc: int):
    if rc != ER_OK:
        raise ERError(fn, rc)


def ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def dev_ptr(t: torch.Tensor, dtype=None, name="tensor"):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def stream_handle(stream=None, device=None):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)
