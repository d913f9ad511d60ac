"""B200-native SWA∥RMA hot path of EdgeRock-4B: a C-ABI CUDA library plus this binding.

The layer (EdgeRock-4B 开源：72 MiB 固定 KV, §架构：递归、局部窗口与记忆锚点三件套):
a 1024-position sliding-window attention in parallel with Rock Memory Anchors,
16 query heads over 4 KV groups of width 256, q/k RMS-norm with RoPE on 64 of
256 dims (base 1e7), an FP32 2560→256→4 retention scorer, and a per-group
top-1024 commit of every 256 pending candidates (neodrop.ai "内存还会跌吗？…",
§三段记忆，只记值得记的).

Everything below marshals torch CUDA tensors into the C entry points of
libedgerock.so (declared in include/edgerock.h); all steps of the path run
in that library's kernels.  torch provides device memory and streams only.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import (BANK, D, HIDDEN, NG, NH, OIN, PEND, QKV, WIN, ERError, check, dev_ptr,
                   lib, stream_handle)

__all__ = ["State", "LayerWeights", "qk_norm_rope", "rma_score", "rma_append_pending",
           "rma_commit", "swa_rma_attend", "swa_rma_decode", "swa_rma_prefill_chunk",
           "advance", "state_init", "last_device_error", "launch_count", "profile_enable",
           "profile_read", "decode_workspace_bytes", "prefill_workspace_bytes",
           "attend_workspace_bytes", "score_workspace_bytes", "rma_score_noalloc",
           "wait_selftest", "last_call_error", "linear", "linear_workspace_bytes",
           "ERError"]


class State:
    """Fixed-capacity state for s_max sequences, carved by the library from one
    caller-owned device allocation (er_state_bytes / er_state_carve)."""

    ARRAYS = ("win_k", "win_v", "bank_k", "bank_v", "pend_k", "pend_v", "bank_score",
              "pend_score", "bank_pos", "pend_pos", "meta")

    def __init__(self, s_max: int, n_layers: int = 8, device="cuda", pool: bool = False):
        """pool=True: the pooled anchor layout (ER_STATE_POOL): bank_k / bank_v /
        bank_score / bank_pos hold 1280 pool slots per group, pend_pos the groups'
        256-entry slot lists, and there are no pend_k / pend_v / pend_score."""
        L = lib()
        flags = _lib.ER_STATE_POOL if pool else 0
        nbytes = L.er_state_bytes_ex(s_max, n_layers, flags)
        if nbytes == 0:
            raise ValueError("bad state size")
        self.s_max, self.n_layers, self.pool = s_max, n_layers, pool
        self.device = torch.device(device)
        self.blob = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        self.c = _lib.CState()
        check("er_state_carve_ex", L.er_state_carve_ex(ctypes.c_void_p(self.blob.data_ptr()),
                                                       nbytes, s_max, n_layers, flags,
                                                       ctypes.byref(self.c)))
        base = self.blob.data_ptr()
        g = (s_max, n_layers, NG)
        nb = BANK + PEND if pool else BANK
        spec = {
            "win_k": (torch.bfloat16, g + (WIN, D)), "win_v": (torch.bfloat16, g + (WIN, D)),
            "bank_k": (torch.bfloat16, g + (nb, D)), "bank_v": (torch.bfloat16, g + (nb, D)),
            "bank_score": (torch.float32, g + (nb,)), "bank_pos": (torch.int32, g + (nb,)),
            "pend_pos": (torch.int32, g + (PEND,)),
            "meta": (torch.int32, (s_max, 4)), "dev_error": (torch.int32, (4,)),
        }
        if not pool:
            spec.update({"pend_k": (torch.bfloat16, g + (PEND, D)),
                         "pend_v": (torch.bfloat16, g + (PEND, D)),
                         "pend_score": (torch.float32, g + (PEND,))})
        for name, (dt, shape) in spec.items():
            off = getattr(self.c, name) - base
            n = 1
            for s in shape:
                n *= s
            view = self.blob[off:off + n * torch.tensor([], dtype=dt).element_size()]
            setattr(self, name, view.view(dt).view(shape))

    def ptr(self):
        return ctypes.byref(self.c)

    def arrays(self):
        if self.pool:
            raise ValueError("the pooled layout has no pending arrays; see pool_from_plain")
        return {n: getattr(self, n) for n in self.ARRAYS}

    def pool_from_plain(self, plain: "State", rows=None):
        """Fill this pooled state's rows from a state in the plain layout holding the
        same records: pool slots 0..1023 take the bank slots, 1024..1279 the pending
        block (slot list 1024 + j), slots past the counts are free.  Copies only."""
        if not self.pool or plain.pool:
            raise ValueError("pool_from_plain copies a plain state into a pooled one")
        rows = range(min(self.s_max, plain.s_max)) if rows is None else rows
        free = 0x7FFFFFFF
        for r in rows:
            c, p = int(plain.meta[r, 2]), int(plain.meta[r, 1])
            self.win_k[r].copy_(plain.win_k[r])
            self.win_v[r].copy_(plain.win_v[r])
            self.bank_k[r, :, :, :BANK].copy_(plain.bank_k[r])
            self.bank_k[r, :, :, BANK:].copy_(plain.pend_k[r])
            self.bank_v[r, :, :, :BANK].copy_(plain.bank_v[r])
            self.bank_v[r, :, :, BANK:].copy_(plain.pend_v[r])
            self.bank_score[r, :, :, :BANK].copy_(plain.bank_score[r])
            self.bank_score[r, :, :, BANK:].copy_(plain.pend_score[r])
            self.bank_pos[r, :, :, :BANK].copy_(plain.bank_pos[r])
            self.bank_pos[r, :, :, BANK:].copy_(plain.pend_pos[r])
            self.bank_pos[r, :, :, c:BANK] = free
            self.bank_pos[r, :, :, BANK + p:] = free
            self.bank_score[r, :, :, c:BANK] = 0.0
            self.bank_score[r, :, :, BANK + p:] = 0.0
            self.pend_pos[r].copy_(torch.arange(BANK, BANK + PEND, dtype=torch.int32,
                                                device=self.device).expand_as(self.pend_pos[r]))
            self.meta[r].copy_(plain.meta[r])


class LayerWeights:
    """One layer's device weights (BF16 projections and gains, FP32 scorer).

    With prepare=True (the default) one BF16 [13056][2560] buffer is built here
    (er_prepare_qkv_score): W_qkv followed by W1's three BF16 terms.  The layer
    calls then run the q/k/v projection and the scorer's W1 product as one GEMM,
    and w_qkv and w1_split become views of that buffer (one copy on the device).
    prepare=False leaves w1_split and w_qkv_score NULL: the layer calls project
    and score separately, and each scorer call splits W1 again in its workspace."""

    def __init__(self, w_qkv, w_o, q_norm_swa, k_norm_swa, q_norm_rma, k_norm_rma, w1, w2,
                 prepare: bool = True):
        bf, f32 = torch.bfloat16, torch.float32
        self.t = dict(w_qkv=w_qkv, w_o=w_o, q_norm_swa=q_norm_swa, k_norm_swa=k_norm_swa,
                      q_norm_rma=q_norm_rma, k_norm_rma=k_norm_rma, w1=w1, w2=w2)
        shapes = dict(w_qkv=((QKV, HIDDEN), bf), w_o=((HIDDEN, OIN), bf), q_norm_swa=((D,), bf),
                      k_norm_swa=((D,), bf), q_norm_rma=((D,), bf), k_norm_rma=((D,), bf),
                      w1=((256, HIDDEN), f32), w2=((NG, 256), f32))
        for k, (shape, dt) in shapes.items():
            t = self.t[k]
            if tuple(t.shape) != shape or t.dtype != dt:
                raise ValueError(f"{k}: expected {shape} {dt}, got {tuple(t.shape)} {t.dtype}")
            dev_ptr(t, dt, k)
        self.w1_split = None
        self.w_qkv_score = None
        if prepare:
            self.w_qkv_score = torch.empty(QKV + 3 * 256, HIDDEN, dtype=bf, device=w1.device)
            check("er_prepare_qkv_score", lib().er_prepare_qkv_score(
                dev_ptr(w_qkv, bf, "w_qkv"), dev_ptr(w1, f32, "w1"),
                dev_ptr(self.w_qkv_score, bf, "w_qkv_score"), stream_handle(None, w1.device)))
            self.t["w_qkv"] = self.w_qkv_score[:QKV]
            self.w1_split = self.w_qkv_score[QKV:].view(3, 256, HIDDEN)
        opt = lambda t: t.data_ptr() if t is not None else None
        self.c = _lib.CWeights(*[self.t[k].data_ptr() for k in
                                 ("w_qkv", "w_o", "q_norm_swa", "k_norm_swa", "q_norm_rma",
                                  "k_norm_rma", "w1", "w2")],
                               opt(self.w1_split), opt(self.w_qkv_score))

    @classmethod
    def from_dict(cls, d, prepare: bool = True):
        return cls(d["w_qkv"], d["w_o"], d["q_norm_swa"], d["k_norm_swa"], d["q_norm_rma"],
                   d["k_norm_rma"], d["w1"], d["w2"], prepare=prepare)

    def ptr(self):
        return ctypes.byref(self.c)


def _ids(seq_ids, device):
    if isinstance(seq_ids, torch.Tensor) and seq_ids.is_cuda and seq_ids.dtype == torch.int32:
        return seq_ids.contiguous()
    return torch.as_tensor(seq_ids, dtype=torch.int32).to(device).contiguous()


def state_init(st: State, seq_ids, stream=None):
    ids = _ids(seq_ids, st.device)
    check("er_state_init", lib().er_state_init(st.ptr(), dev_ptr(ids), ids.numel(),
                                               stream_handle(stream, st.device)))


def _flags(rma_off: bool) -> int:
    return _lib.ER_FLAG_RMA_OFF if rma_off else 0


def advance(st: State, seq_ids, T: int = 1, stream=None, rma_off: bool = False):
    """End of a step of T tokens; with rma_off only the positions move."""
    ids = _ids(seq_ids, st.device)
    check("er_advance_ex", lib().er_advance_ex(st.ptr(), dev_ptr(ids), ids.numel(), T,
                                               _flags(rma_off), stream_handle(stream, st.device)))


def last_device_error(st: State, stream=None) -> int:
    code = ctypes.c_int32(0)
    rc = lib().er_last_device_error(st.ptr(), ctypes.byref(code), stream_handle(stream, st.device))
    if rc not in (_lib.ER_OK, _lib.ER_EDEVICE):
        raise ERError("er_last_device_error", rc)
    return int(code.value)


def last_call_error(stream=None) -> int:
    """The library's own error word (the calls that take no state), read and cleared."""
    code = ctypes.c_int32(0)
    rc = lib().er_last_call_error(ctypes.byref(code), stream_handle(stream))
    if rc not in (_lib.ER_OK, _lib.ER_EDEVICE):
        raise ERError("er_last_call_error", rc)
    return int(code.value)


def wait_selftest(st, arrive: bool, stream=None):
    """er_wait_selftest: a bounded device wait that completes (arrive=True) or
    runs out (~2 s, ER_ETIMEOUT in the state's error word, or in the library's
    own word when st is None)."""
    check("er_wait_selftest", lib().er_wait_selftest(
        st.ptr() if st is not None else None, 1 if arrive else 0,
        stream_handle(stream, st.device if st is not None else None)))


def qk_norm_rope(x: torch.Tensor, gain: torch.Tensor, pos: torch.Tensor, out=None, stream=None):
    rows = x.numel() // D
    out = torch.empty_like(x) if out is None else out
    check("er_qk_norm_rope", lib().er_qk_norm_rope(
        dev_ptr(x, torch.bfloat16, "x"), dev_ptr(out, torch.bfloat16, "out"), rows,
        dev_ptr(gain, torch.bfloat16, "gain"), dev_ptr(pos, torch.int32, "pos"),
        stream_handle(stream, x.device)))
    return out


def linear_workspace_bytes(T: int, F: int, K: int) -> int:
    return int(lib().er_linear_workspace_bytes(T, F, K))


def linear(x: torch.Tensor, w: torch.Tensor, fp32_out: bool = False, out=None, ws=None,
           stream=None, dev_error=None):
    """y = x · wᵀ on the tensor cores (er_linear): x BF16 [T, K], w BF16 [F, K];
    y BF16 (or FP32 with fp32_out) [T, F]."""
    T, K = x.shape
    F = w.shape[0]
    dt = torch.float32 if fp32_out else torch.bfloat16
    out = torch.empty(T, F, dtype=dt, device=x.device) if out is None else out
    ws = _ws(linear_workspace_bytes(max(T, 1), F, K), x.device, ws)
    err = dev_ptr(dev_error, torch.int32, "dev_error") if dev_error is not None else None
    check("er_linear", lib().er_linear(
        dev_ptr(x, torch.bfloat16, "x"), T, dev_ptr(w, torch.bfloat16, "w"), F, K,
        dev_ptr(out, dt, "out"), 1 if fp32_out else 0, out.stride(0), dev_ptr(ws), ws.numel(),
        err, stream_handle(stream, x.device)))
    return out


def score_workspace_bytes(n: int) -> int:
    return int(lib().er_score_workspace_bytes(n))


def rma_score(w: LayerWeights, x: torch.Tensor, ws=None, stream=None, dev_error=None):
    """FP32 scores [n, 4].  dev_error: an optional device int32 tensor that receives
    a device-side error code (default: the library's own word, last_call_error)."""
    n = x.numel() // HIDDEN
    s = torch.empty(n, NG, dtype=torch.float32, device=x.device)
    ws = _ws(score_workspace_bytes(n), x.device, ws)
    err = dev_ptr(dev_error, torch.int32, "dev_error") if dev_error is not None else None
    check("er_rma_score_ex", lib().er_rma_score_ex(w.ptr(), dev_ptr(x, torch.bfloat16, "x"), n,
                                                   dev_ptr(s), dev_ptr(ws), ws.numel(), err,
                                                   stream_handle(stream, x.device)))
    return s


def rma_score_noalloc(w: LayerWeights, x: torch.Tensor, stream=None):
    """er_rma_score without a workspace: the scratch is a fixed array inside the
    library (at most ER_SCORE_NOALLOC_MAX_TOKENS = 256 tokens per call)."""
    n = x.numel() // HIDDEN
    s = torch.empty(n, NG, dtype=torch.float32, device=x.device)
    check("er_rma_score_noalloc", lib().er_rma_score_noalloc(
        w.ptr(), dev_ptr(x, torch.bfloat16, "x"), n, dev_ptr(s), stream_handle(stream, x.device)))
    return s


def rma_append_pending(st: State, layer: int, seq_ids, k, v, s, pos, stream=None):
    ids = _ids(seq_ids, st.device)
    check("er_rma_append_pending", lib().er_rma_append_pending(
        st.ptr(), layer, dev_ptr(ids), ids.numel(), dev_ptr(k, torch.bfloat16, "k"),
        dev_ptr(v, torch.bfloat16, "v"), dev_ptr(s, torch.float32, "s"),
        dev_ptr(pos, torch.int32, "pos"), stream_handle(stream, st.device)))


def rma_commit(st: State, layer: int, seq_ids, want_kept=False, stream=None):
    ids = _ids(seq_ids, st.device)
    kept = None
    if want_kept:
        nl = st.n_layers if layer < 0 else 1
        kept = torch.empty(ids.numel(), nl, NG, BANK, dtype=torch.int32, device=st.device)
    check("er_rma_commit", lib().er_rma_commit(st.ptr(), layer, dev_ptr(ids), ids.numel(),
                                               dev_ptr(kept) if kept is not None else None,
                                               stream_handle(stream, st.device)))
    return kept


def attend_workspace_bytes(B: int) -> int:
    return int(lib().er_attend_workspace_bytes(B))


def decode_workspace_bytes(B: int) -> int:
    return int(lib().er_decode_workspace_bytes(B))


def prefill_workspace_bytes(T: int) -> int:
    return int(lib().er_prefill_workspace_bytes(T))


def _ws(nbytes, device, ws=None):
    if ws is not None and ws.numel() >= nbytes:
        return ws
    return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)


def swa_rma_attend(st: State, layer: int, seq_ids, q_swa, q_rma, ws=None, stream=None):
    ids = _ids(seq_ids, st.device)
    B = ids.numel()
    o_swa = torch.empty(B, NH, D, dtype=torch.float32, device=st.device)
    o_rma = torch.empty(B, NH, D, dtype=torch.float32, device=st.device)
    nb = attend_workspace_bytes(B)
    ws = _ws(nb, st.device, ws)
    check("er_swa_rma_attend", lib().er_swa_rma_attend(
        st.ptr(), layer, dev_ptr(ids), B, dev_ptr(q_swa, torch.bfloat16, "q_swa"),
        dev_ptr(q_rma, torch.bfloat16, "q_rma"), dev_ptr(o_swa), dev_ptr(o_rma),
        dev_ptr(ws), ws.numel(), stream_handle(stream, st.device)))
    return o_swa, o_rma


def swa_rma_decode(st: State, w: LayerWeights, layer: int, seq_ids, x, out=None, ws=None,
                   stream=None, rma_off: bool = False):
    ids = _ids(seq_ids, st.device)
    B = ids.numel()
    out = torch.empty(B, HIDDEN, dtype=torch.bfloat16, device=st.device) if out is None else out
    ws = _ws(decode_workspace_bytes(B), st.device, ws)
    check("er_swa_rma_decode_ex", lib().er_swa_rma_decode_ex(
        st.ptr(), w.ptr(), layer, dev_ptr(ids), B, dev_ptr(x, torch.bfloat16, "x"),
        dev_ptr(out, torch.bfloat16, "out"), dev_ptr(ws), ws.numel(), _flags(rma_off),
        stream_handle(stream, st.device)))
    return out


def swa_rma_prefill_chunk(st: State, w: LayerWeights, layer: int, seq_id: int, x, out=None,
                          ws=None, stream=None, rma_off: bool = False):
    T = x.shape[0]
    out = torch.empty(T, HIDDEN, dtype=torch.bfloat16, device=st.device) if out is None else out
    ws = _ws(prefill_workspace_bytes(T), st.device, ws)
    check("er_swa_rma_prefill_chunk_ex", lib().er_swa_rma_prefill_chunk_ex(
        st.ptr(), w.ptr(), layer, int(seq_id), dev_ptr(x, torch.bfloat16, "x"), T,
        dev_ptr(out, torch.bfloat16, "out"), dev_ptr(ws), ws.numel(), _flags(rma_off),
        stream_handle(stream, st.device)))
    return out


def launch_count() -> int:
    return int(lib().er_launch_count())


def profile_enable(on: bool = True):
    lib().er_profile_enable(1 if on else 0)


def profile_read(reset: bool = False):
    ms = ctypes.c_double(0)
    n = ctypes.c_int64(0)
    check("er_profile_read", lib().er_profile_read(ctypes.byref(ms), ctypes.byref(n),
                                                   1 if reset else 0))
    return float(ms.value), int(n.value)
