"""CPU oracle of the EdgeRock-4B SWA∥RMA layer and RMA commit (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The product
path (``sliding_window_anchor_b200``) never does.

The arithmetic lives in ``oracle.c`` (plain C, float64); this module only
marshals torch CPU tensors into it.  Per-function sources are cited in
``oracle.c``.  ctypes releases the GIL during each call, so several oracle
calls may run in parallel from a thread pool.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import torch

_DIR = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None

D, HIDDEN, NH, NG, WIN, BANK, PEND = 256, 2560, 16, 4, 1024, 1024, 256
QKV = 2 * (NH * D + 2 * NG * D)


def build(force: bool = False) -> None:
    """Compile oracle.c into liboracle.so (gcc, -O2, no FMA contraction)."""
    with _lock:
        src = os.path.join(_DIR, "oracle.c")
        if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
            subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC",
                                   "-shared", "-Wall", "-o", _SO, src, "-lm"])


class _State(ctypes.Structure):
    _fields_ = [("s_max", ctypes.c_int32), ("n_layers", ctypes.c_int32)] + [
        (n, ctypes.c_void_p) for n in ("win_k", "win_v", "bank_k", "bank_v", "pend_k", "pend_v",
                                       "bank_score", "pend_score", "bank_pos", "pend_pos", "meta")]


class _Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w_qkv", "w_o", "g_q_swa", "g_k_swa", "g_q_rma",
                                               "g_k_rma", "w1", "w2")]


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        L.orc_kv_bytes_per_seq.argtypes = [i32]
        L.orc_kv_bytes_per_seq.restype = i64
        L.orc_norm_rope.argtypes = [vp, vp, vp, i64, vp]
        L.orc_linear_bf16.argtypes = [vp, i32, i32, vp, vp]
        L.orc_score.argtypes = [vp, vp, vp, i32, vp]
        L.orc_attend_rows.argtypes = [vp, vp, vp, i32, vp]
        L.orc_commit.argtypes = [vp, i32, i32, vp]
        L.orc_advance.argtypes = [vp, i32, i32, i32]
        L.orc_decode_layer.argtypes = [vp, vp, i32, i32, vp, vp, vp, vp, i32]
        L.orc_prefill_chunk.argtypes = [vp, vp, i32, i32, vp, i32, vp, i32]
        L.orc_prefill_chunk.restype = ctypes.c_int
        L.orc_append_pending.argtypes = [vp, i32, vp, i32, vp, vp, vp, vp]
        L.orc_f64_to_bf16.argtypes = [ctypes.c_double]
        L.orc_f64_to_bf16.restype = ctypes.c_uint16
        for f in (L.orc_norm_rope, L.orc_linear_bf16, L.orc_score, L.orc_attend_rows,
                  L.orc_commit, L.orc_advance, L.orc_decode_layer, L.orc_append_pending):
            f.restype = None
        _lib = L
    return _lib


def _p(t):
    if t is None:
        return None
    assert t.device.type == "cpu" and t.is_contiguous()
    return ctypes.c_void_p(t.data_ptr())


# --------------------------------------------------------------- containers

class OracleWeights:
    """One layer's weights as CPU tensors (BF16 except the FP32 scorer)."""

    def __init__(self, w_qkv, w_o, g_q_swa, g_k_swa, g_q_rma, g_k_rma, w1, w2):
        self.w_qkv, self.w_o = w_qkv.contiguous(), w_o.contiguous()
        self.g_q_swa, self.g_k_swa = g_q_swa.contiguous(), g_k_swa.contiguous()
        self.g_q_rma, self.g_k_rma = g_q_rma.contiguous(), g_k_rma.contiguous()
        self.w1, self.w2 = w1.contiguous(), w2.contiguous()
        self._s = _Weights(*[t.data_ptr() for t in (self.w_qkv, self.w_o, self.g_q_swa,
                                                    self.g_k_swa, self.g_q_rma, self.g_k_rma,
                                                    self.w1, self.w2)])

    def ptr(self):
        return ctypes.byref(self._s)


class OracleState:
    """Fixed-capacity per-sequence state, same [seq][layer][group][slot][256] layout
    as the device state so the two can be compared array by array."""

    def __init__(self, s_max: int, n_layers: int = 8, kv: bool = True):
        """kv=False builds a state with scores, positions and metadata only (no K/V
        rows): enough to rank and place records in a commit."""
        self.s_max, self.n_layers = s_max, n_layers
        g = (s_max, n_layers, NG)
        z = torch.zeros
        kvs = (lambda slots: g + (slots, D)) if kv else (lambda slots: (0,))
        self.win_k = z(kvs(WIN), dtype=torch.bfloat16)
        self.win_v = z(kvs(WIN), dtype=torch.bfloat16)
        self.bank_k = z(kvs(BANK), dtype=torch.bfloat16)
        self.bank_v = z(kvs(BANK), dtype=torch.bfloat16)
        self.pend_k = z(kvs(PEND), dtype=torch.bfloat16)
        self.pend_v = z(kvs(PEND), dtype=torch.bfloat16)
        self.bank_score = z(g + (BANK,), dtype=torch.float32)
        self.pend_score = z(g + (PEND,), dtype=torch.float32)
        self.bank_pos = z(g + (BANK,), dtype=torch.int32)
        self.pend_pos = z(g + (PEND,), dtype=torch.int32)
        self.meta = z((s_max, 4), dtype=torch.int32)
        self._bind()

    ARRAYS = ("win_k", "win_v", "bank_k", "bank_v", "pend_k", "pend_v", "bank_score",
              "pend_score", "bank_pos", "pend_pos", "meta")

    def _bind(self):
        self._s = _State(self.s_max, self.n_layers,
                         *[(getattr(self, n).data_ptr() if getattr(self, n).numel() else None)
                           for n in self.ARRAYS])

    def ptr(self):
        return ctypes.byref(self._s)

    def clone(self) -> "OracleState":
        o = OracleState.__new__(OracleState)
        o.s_max, o.n_layers = self.s_max, self.n_layers
        for n in self.ARRAYS:
            setattr(o, n, getattr(self, n).clone())
        o._bind()
        return o

    # ----------------------------------------------------------- the layer
    def decode_layer(self, w: OracleWeights, layer: int, seq: int, x: torch.Tensor,
                     want_branches: bool = False, rma_off: bool = False):
        out = torch.empty(HIDDEN, dtype=torch.bfloat16)
        o_swa = torch.empty(NH, D, dtype=torch.float64) if want_branches else None
        o_rma = torch.empty(NH, D, dtype=torch.float64) if want_branches else None
        lib().orc_decode_layer(w.ptr(), self.ptr(), layer, seq, _p(x.contiguous()), _p(out),
                               _p(o_swa), _p(o_rma), 1 if rma_off else 0)
        return (out, o_swa, o_rma) if want_branches else out

    def prefill_chunk(self, w: OracleWeights, layer: int, seq: int, x: torch.Tensor,
                      rma_off: bool = False):
        T = x.shape[0]
        out = torch.empty(T, HIDDEN, dtype=torch.bfloat16)
        rc = lib().orc_prefill_chunk(w.ptr(), self.ptr(), layer, seq, _p(x.contiguous()), T,
                                     _p(out), 1 if rma_off else 0)
        if rc != 0:
            raise ValueError("prefill chunk crosses the pending block boundary")
        return out

    def commit(self, layer: int, seq: int, want_kept: bool = False):
        kept = None
        if want_kept:
            nl = self.n_layers if layer < 0 else 1
            kept = torch.empty(nl, NG, BANK, dtype=torch.int32)
        lib().orc_commit(self.ptr(), layer, seq, _p(kept))
        return kept

    def advance(self, seq: int, T: int = 1, rma_off: bool = False):
        lib().orc_advance(self.ptr(), seq, T, 1 if rma_off else 0)

    def append_pending(self, layer, seqs, k, v, s, pos):
        seqs = torch.as_tensor(seqs, dtype=torch.int32).contiguous()
        lib().orc_append_pending(self.ptr(), layer, _p(seqs), seqs.numel(), _p(k.contiguous()),
                                 _p(v.contiguous()), _p(s.contiguous()), _p(pos.contiguous()))


# ------------------------------------------------------------- step functions

def kv_bytes_per_seq(n_layers: int = 8) -> int:
    return int(lib().orc_kv_bytes_per_seq(n_layers))


def norm_rope(x: torch.Tensor, gain: torch.Tensor, pos) -> torch.Tensor:
    """RMS-norm (gain) + partial RoPE of BF16 rows [..., 256] at per-row positions."""
    x = x.contiguous()
    rows = x.numel() // D
    pos = torch.as_tensor(pos, dtype=torch.int32).reshape(-1).contiguous()
    if pos.numel() == 1 and rows > 1:
        pos = pos.expand(rows).contiguous()
    assert pos.numel() == rows
    out = torch.empty_like(x)
    lib().orc_norm_rope(_p(x), _p(gain.contiguous()), _p(pos), rows, _p(out))
    return out


def linear_bf16(W: torch.Tensor, x: torch.Tensor) -> torch.Tensor:
    out_dim, in_dim = W.shape
    y = torch.empty(out_dim, dtype=torch.bfloat16)
    lib().orc_linear_bf16(_p(W.contiguous()), out_dim, in_dim, _p(x.contiguous()), _p(y))
    return y


def score(w1: torch.Tensor, w2: torch.Tensor, x: torch.Tensor) -> torch.Tensor:
    """FP32 scores [n, 4] of BF16 hidden states [n, 2560]."""
    x = x.reshape(-1, HIDDEN).contiguous()
    s = torch.empty(x.shape[0], NG, dtype=torch.float32)
    lib().orc_score(_p(w1.contiguous()), _p(w2.contiguous()), _p(x), x.shape[0], _p(s))
    return s


def attend_rows(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor) -> torch.Tensor:
    """softmax(q·kᵀ/16)·v over n BF16 rows, float64 [256]."""
    o = torch.empty(D, dtype=torch.float64)
    lib().orc_attend_rows(_p(q.contiguous()), _p(k.contiguous()), _p(v.contiguous()),
                          k.shape[0], _p(o))
    return o


def f64_to_bf16_bits(x: float) -> int:
    return int(lib().orc_f64_to_bf16(float(x)))
