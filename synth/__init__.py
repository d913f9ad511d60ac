"""Seeded, counter-based synthetic inputs shared by the CPU oracle and the CUDA path.

This module holds no arithmetic of the SWA∥RMA layer.  It maps
(seed, stream, element index) to numbers with SplitMix64 (Steele, Lea & Flood,
OOPSLA 2014) and an Irwin-Hall normal built from exact integer arithmetic, so
the host fills (plain C) and the device fills (CUDA) are bit-identical.  A
sub-range of a tensor can be generated on its own by passing the index of its
first element (``index0``); that is how the oracle rebuilds a few sampled
sequences of a state that only exists in full on the GPU.

Every fill returns a torch tensor on the requested device.  torch is only the
container here.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import torch

_DIR = os.path.dirname(os.path.abspath(__file__))
_HOST_SO = os.path.join(_DIR, "libsynth_host.so")
_DEV_SO = os.path.join(_DIR, "libsynth_dev.so")
_lock = threading.Lock()
_host = None
_dev = None

# stream identifiers (mirror synth.h)
W_QKV, W_O, G_Q_SWA, G_K_SWA, G_Q_RMA, G_K_RMA, W1, W2 = 1, 2, 3, 4, 5, 6, 7, 8
WIN_K, WIN_V, BANK_K, BANK_V, BANK_SCORE, BANK_POS = 16, 17, 18, 19, 20, 21
PEND_K, PEND_V, PEND_SCORE, PEND_FILL = 22, 23, 24, 25
X, DUP, MISC = 32, 40, 48


def stream_id(base: int, layer: int = 0, step: int = 0) -> int:
    """Stream of one tensor of one layer at one step."""
    return int(base) | (int(layer) << 32) | (int(step) << 40)


def build(force: bool = False) -> None:
    """Compile the host fill library (gcc) and the device fill library (nvcc, sm_100a)."""
    with _lock:
        src_h = os.path.join(_DIR, "synth_host.c")
        src_d = os.path.join(_DIR, "synth_dev.cu")
        hdr = os.path.join(_DIR, "synth.h")
        newest = max(os.path.getmtime(p) for p in (src_h, hdr))
        if force or not os.path.exists(_HOST_SO) or os.path.getmtime(_HOST_SO) < newest:
            subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC",
                                   "-shared", "-o", _HOST_SO, src_h])
        newest = max(os.path.getmtime(p) for p in (src_d, hdr))
        if force or not os.path.exists(_DEV_SO) or os.path.getmtime(_DEV_SO) < newest:
            subprocess.check_call(["nvcc", "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
                                   "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
                                   "-fmad=false", "-o", _DEV_SO, src_d])


def _load_host():
    global _host
    if _host is None:
        if not os.path.exists(_HOST_SO):
            build()
        lib = ctypes.CDLL(_HOST_SO)
        u64, i64, f32, u32, i32, vp = (ctypes.c_uint64, ctypes.c_int64, ctypes.c_float,
                                       ctypes.c_uint32, ctypes.c_int32, ctypes.c_void_p)
        lib.synth_fill_normal_f32.argtypes = [vp, i64, u64, u64, u64, f32, f32]
        lib.synth_fill_normal_bf16.argtypes = [vp, i64, u64, u64, u64, f32, f32]
        lib.synth_fill_uniform_i32.argtypes = [vp, i64, u64, u64, u64, u32, i32]
        lib.synth_fill_strata_i32.argtypes = [vp, i64, u64, u64, u64, u32, u32]
        lib.synth_fill_normal_dup_f32.argtypes = [vp, i64, u64, u64, u64, u32, u32]
        for f in (lib.synth_fill_normal_f32, lib.synth_fill_normal_bf16,
                  lib.synth_fill_uniform_i32, lib.synth_fill_strata_i32,
                  lib.synth_fill_normal_dup_f32):
            f.restype = None
        _host = lib
    return _host


def _load_dev():
    global _dev
    if _dev is None:
        if not os.path.exists(_DEV_SO):
            raise RuntimeError("synth device library is not built (run synth.build())")
        lib = ctypes.CDLL(_DEV_SO)
        u64, i64, f32, u32, i32, vp = (ctypes.c_uint64, ctypes.c_int64, ctypes.c_float,
                                       ctypes.c_uint32, ctypes.c_int32, ctypes.c_void_p)
        lib.synthd_fill_normal_f32.argtypes = [vp, i64, u64, u64, u64, f32, f32, vp]
        lib.synthd_fill_normal_bf16.argtypes = [vp, i64, u64, u64, u64, f32, f32, vp]
        lib.synthd_fill_uniform_i32.argtypes = [vp, i64, u64, u64, u64, u32, i32, vp]
        lib.synthd_fill_strata_i32.argtypes = [vp, i64, u64, u64, u64, u32, u32, vp]
        lib.synthd_fill_normal_dup_f32.argtypes = [vp, i64, u64, u64, u64, u32, u32, vp]
        for f in (lib.synthd_fill_normal_f32, lib.synthd_fill_normal_bf16,
                  lib.synthd_fill_uniform_i32, lib.synthd_fill_strata_i32,
                  lib.synthd_fill_normal_dup_f32):
            f.restype = ctypes.c_int
        _dev = lib
    return _dev


def _stream_ptr(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _check(rc):
    if rc != 0:
        raise RuntimeError(f"synth device fill failed: cuda error {rc}")


def fill_normal_(t: torch.Tensor, seed: int, stream: int, index0: int = 0,
                 scale: float = 1.0, offset: float = 0.0) -> torch.Tensor:
    """Fill a contiguous float32 or bfloat16 tensor with offset + scale*N(0,1)."""
    assert t.is_contiguous()
    n = t.numel()
    args = (ctypes.c_void_p(t.data_ptr()), n, seed, stream, index0, scale, offset)
    if t.dtype == torch.float32:
        if t.is_cuda:
            _check(_load_dev().synthd_fill_normal_f32(*args, _stream_ptr(t)))
        else:
            _load_host().synth_fill_normal_f32(*args)
    elif t.dtype == torch.bfloat16:
        if t.is_cuda:
            _check(_load_dev().synthd_fill_normal_bf16(*args, _stream_ptr(t)))
        else:
            _load_host().synth_fill_normal_bf16(*args)
    else:
        raise TypeError(t.dtype)
    return t


def fill_uniform_(t: torch.Tensor, seed: int, stream: int, n: int, add: int = 0,
                  index0: int = 0) -> torch.Tensor:
    """Fill a contiguous int32 tensor with add + U{0..n-1}."""
    assert t.is_contiguous() and t.dtype == torch.int32
    args = (ctypes.c_void_p(t.data_ptr()), t.numel(), seed, stream, index0, n, add)
    if t.is_cuda:
        _check(_load_dev().synthd_fill_uniform_i32(*args, _stream_ptr(t)))
    else:
        _load_host().synth_fill_uniform_i32(*args)
    return t


def fill_strata_(t: torch.Tensor, seed: int, stream: int, period: int, width: int,
                 index0: int = 0) -> torch.Tensor:
    """Fill int32 with ((index % period) * width + U{0..width-1}): distinct per period."""
    assert t.is_contiguous() and t.dtype == torch.int32
    args = (ctypes.c_void_p(t.data_ptr()), t.numel(), seed, stream, index0, period, width)
    if t.is_cuda:
        _check(_load_dev().synthd_fill_strata_i32(*args, _stream_ptr(t)))
    else:
        _load_host().synth_fill_strata_i32(*args)
    return t


def fill_normal_dup_(t: torch.Tensor, seed: int, stream: int, group: int, one_in: int,
                     index0: int = 0) -> torch.Tensor:
    """float32 N(0,1) where ~1/one_in of the values copy another value of their group."""
    assert t.is_contiguous() and t.dtype == torch.float32
    args = (ctypes.c_void_p(t.data_ptr()), t.numel(), seed, stream, index0, group, one_in)
    if t.is_cuda:
        _check(_load_dev().synthd_fill_normal_dup_f32(*args, _stream_ptr(t)))
    else:
        _load_host().synth_fill_normal_dup_f32(*args)
    return t


def normal(shape, seed, stream, dtype=torch.float32, device="cpu", index0=0, scale=1.0,
           offset=0.0):
    t = torch.empty(shape, dtype=dtype, device=device)
    return fill_normal_(t, seed, stream, index0, scale, offset)
