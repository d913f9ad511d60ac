"""The C-ABI library builds, loads and exports every declared symbol (CPU only).

Only host-side logic is exercised here: sizes, carving, argument checks that
return before anything is enqueued.  No kernel is launched.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from sliding_window_anchor_b200 import build, _lib
    build.build()
    return _lib.lib()


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"\b(er_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(L, n), n
    from sliding_window_anchor_b200 import _lib
    assert set(names) == set(_lib.EXPORTS)


def test_state_bytes_and_carve(L):
    from sliding_window_anchor_b200._lib import CState
    n = L.er_state_bytes(2, 8)
    kv = 2 * 75497472
    meta = 2 * 8 * 4 * (1024 + 256) * 8
    assert kv + meta <= n <= kv + meta + 64 * 1024
    assert L.er_state_bytes(0, 8) == 0 and L.er_state_bytes(1, 9) == 0
    st = CState()
    fake = 1 << 40  # carving only computes pointers
    assert L.er_state_carve(ctypes.c_void_p(fake), n, 2, 8, ctypes.byref(st)) == 0
    assert st.win_v - st.win_k == 2 * 8 * 4 * 1024 * 256 * 2
    assert st.pend_v - st.pend_k == 2 * 8 * 4 * 256 * 256 * 2
    for f in ("win_k", "bank_k", "pend_k", "bank_score", "pend_score", "bank_pos", "pend_pos",
              "meta", "dev_error"):
        assert getattr(st, f) % 256 == 0
    assert st.dev_error + 64 * 4 <= fake + n
    # the carved arrays are disjoint, in order, inside the allocation
    g = 2 * 8 * 4
    sizes = {"win_k": g * 1024 * 512, "win_v": g * 1024 * 512, "bank_k": g * 1024 * 512,
             "bank_v": g * 1024 * 512, "pend_k": g * 256 * 512, "pend_v": g * 256 * 512,
             "bank_score": g * 1024 * 4, "pend_score": g * 256 * 4, "bank_pos": g * 1024 * 4,
             "pend_pos": g * 256 * 4, "meta": 2 * 16, "dev_error": 16}
    spans = sorted((getattr(st, f), getattr(st, f) + b) for f, b in sizes.items())
    assert spans[0][0] >= fake and spans[-1][1] <= fake + n
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 <= b0
    assert L.er_state_carve(ctypes.c_void_p(fake), n - 1, 2, 8, ctypes.byref(st)) == -1
    assert L.er_state_carve(ctypes.c_void_p(fake + 8), n, 2, 8, ctypes.byref(st)) == -1


def test_workspace_sizes_monotone(L):
    prev = 0
    for B in (1, 2, 8, 64, 512):
        n = L.er_decode_workspace_bytes(B)
        assert n > prev
        prev = n
    assert L.er_prefill_workspace_bytes(1) > 0 and L.er_prefill_workspace_bytes(0) == 0
    assert L.er_prefill_workspace_bytes(257) == 0
    assert L.er_attend_workspace_bytes(512) < L.er_decode_workspace_bytes(512)


def test_host_validation_rejects_before_enqueue(L):
    from sliding_window_anchor_b200._lib import CState, CWeights
    st = CState()
    n = L.er_state_bytes(4, 8)
    L.er_state_carve(ctypes.c_void_p(1 << 40), n, 4, 8, ctypes.byref(st))
    w = CWeights()
    nul = None
    # null state / weights / pointers, bad layer, bad sizes: all return before any launch
    assert L.er_swa_rma_decode(None, ctypes.byref(w), 0, nul, 1, nul, nul, nul, 0, nul) == -1
    assert L.er_swa_rma_decode(ctypes.byref(st), ctypes.byref(w), 0, nul, 1, nul, nul, nul, 0,
                               nul) == -1
    assert L.er_swa_rma_decode(ctypes.byref(st), ctypes.byref(w), 8, nul, 1, nul, nul, nul, 0,
                               nul) == -1
    assert L.er_swa_rma_decode(ctypes.byref(st), ctypes.byref(w), 0, nul, 5, nul, nul, nul, 0,
                               nul) == -2  # batch above the state's capacity
    assert L.er_swa_rma_prefill_chunk(ctypes.byref(st), ctypes.byref(w), 0, 0, nul, 257, nul,
                                      nul, 0, nul) == -1
    assert L.er_swa_rma_prefill_chunk(ctypes.byref(st), ctypes.byref(w), 0, 4, nul, 16, nul,
                                      nul, 0, nul) == -1
    assert L.er_rma_commit(ctypes.byref(st), 8, nul, 1, nul, nul) == -1
    assert L.er_rma_commit(ctypes.byref(st), -2, nul, 1, nul, nul) == -1
    assert L.er_rma_append_pending(ctypes.byref(st), 0, nul, 1, nul, nul, nul, nul, nul) == -1
    assert L.er_advance(ctypes.byref(st), nul, 1, 0, nul) == -1
    assert L.er_advance(ctypes.byref(st), nul, 1, 257, nul) == -1
    assert L.er_rma_score(None, nul, 1, nul, nul, 0, nul) == -1
    assert L.er_qk_norm_rope(nul, nul, 4, nul, nul, nul) == -1
    # misaligned rows are refused (16-byte vector loads and bulk copies need alignment)
    fake = ctypes.c_void_p((1 << 40) + 2)
    ok = ctypes.c_void_p(1 << 40)
    before = L.er_launch_count()
    assert L.er_qk_norm_rope(fake, ok, 4, ok, ok, nul) == -1
    assert L.er_swa_rma_attend(ctypes.byref(st), 0, ok, 1, fake, ok, ok, ok, ok, 1 << 30,
                               nul) == -1
    assert L.er_launch_count() == before
    # empty work is fine and launches nothing
    before = L.er_launch_count()
    assert L.er_rma_score(ctypes.byref(w), nul, 0, nul, nul, 0, nul) == 0
    assert L.er_qk_norm_rope(nul, nul, 0, nul, nul, nul) == 0
    assert L.er_launch_count() == before
    assert L.er_error_string(-2) == b"capacity exceeded"
    # flags: the RMA switch is the only defined bit; others are refused before anything else
    before = L.er_launch_count()
    assert L.er_swa_rma_decode_ex(ctypes.byref(st), ctypes.byref(w), 0, nul, 0, nul, nul, nul,
                                  0, 1, nul) == 0
    assert L.er_swa_rma_decode_ex(ctypes.byref(st), ctypes.byref(w), 0, nul, 0, nul, nul, nul,
                                  0, 2, nul) == -1
    assert L.er_advance_ex(ctypes.byref(st), nul, 0, 1, 1, nul) == 0
    assert L.er_advance_ex(ctypes.byref(st), nul, 0, 1, 4, nul) == -1
    assert L.er_swa_rma_prefill_chunk_ex(ctypes.byref(st), ctypes.byref(w), 0, 0, nul, 16, nul,
                                         nul, 0, 8, nul) == -1
    assert L.er_launch_count() == before
    # the bounded-wait diagnostic: only arrive 0 or 1 (with a state or, NULL, the
    # library's own word); a state without an error word is refused
    before = L.er_launch_count()
    assert L.er_wait_selftest(None, 2, nul) == -1
    assert L.er_wait_selftest(ctypes.byref(st), 2, nul) == -1
    no_word = CState()
    ctypes.memmove(ctypes.byref(no_word), ctypes.byref(st), ctypes.sizeof(st))
    no_word.dev_error = None
    assert L.er_wait_selftest(ctypes.byref(no_word), 0, nul) == -1
    # the scorer with an explicit error word checks its arguments the same way
    assert L.er_rma_score_ex(None, nul, 1, nul, nul, 0, nul, nul) == -1
    assert L.er_rma_score_ex(ctypes.byref(w), nul, 0, nul, nul, 0, nul, nul) == 0
    assert L.er_last_call_error(None, nul) == -1
    assert L.er_launch_count() == before
    # the projection GEMM: sizes, alignment and workspace are checked before any launch
    before = L.er_launch_count()
    assert L.er_linear_workspace_bytes(1, 300, 2560) == 0
    assert L.er_linear_workspace_bytes(512, 13056, 2560) > 0
    assert L.er_linear(ok, 4, ok, 300, 2560, ok, 0, 300, ok, 1 << 30, nul, nul) == -1
    assert L.er_linear(ok, 4, ok, 2560, 100, ok, 0, 2560, ok, 1 << 30, nul, nul) == -1
    assert L.er_linear(ok, 4, ok, 2560, 2560, ok, 2, 2560, ok, 1 << 30, nul, nul) == -1
    assert L.er_linear(ok, 4, ok, 2560, 2560, ok, 0, 2000, ok, 1 << 30, nul, nul) == -1
    assert L.er_linear(fake, 4, ok, 2560, 2560, ok, 0, 2560, ok, 1 << 30, nul, nul) == -1
    assert L.er_linear(ok, 4, ok, 2560, 2560, ok, 0, 2560, ok, 16, nul, nul) == -2
    assert L.er_linear(nul, 0, nul, 2560, 2560, nul, 0, 2560, nul, 0, nul, nul) == 0
    assert L.er_launch_count() == before
    # the fused q/k/v + W1-term weights: NULL, unaligned or overlapping buffers are refused
    base = 1 << 40
    qkv_bytes = 12288 * 2560 * 2
    before = L.er_launch_count()
    assert L.er_prepare_qkv_score(nul, ok, ok, nul) == -1
    assert L.er_prepare_qkv_score(ok, ok, fake, nul) == -1
    assert L.er_prepare_qkv_score(ctypes.c_void_p(base), ok,
                                  ctypes.c_void_p(base + qkv_bytes - 4096), nul) == -1
    assert L.er_prepare_qkv_score(ctypes.c_void_p(base + qkv_bytes), ok,
                                  ctypes.c_void_p(base + 4096), nul) == -1
    assert L.er_launch_count() == before
