"""The allocation-free scorer, er_rma_score_noalloc, against er_rma_score.

Some callers of this library cannot give it scratch memory: their device
memory belongs to another framework's allocator, or they only receive the
input and output pointers.  For them the library keeps the scorer's scratch
(W1 as three BF16 terms, the partial scores) in a fixed array of its own (at
most 256 tokens per call).  This file checks, through the C ABI:
  - the allocation-free call returns exactly the bits of the workspace call
    (both run the same fixed-order arithmetic), on two calls in a row (the
    second finds the array holding the first call's leftovers), with the W1
    terms made by the call and with terms prepared once (er_score_split_w1);
  - its scores are within the scorer tolerance of the CPU oracle;
  - the library's error word stays clear after each call;
  - a size above the maximum is refused without launching anything.
It is collected last on purpose.
"""
import ctypes

import pytest
import torch

import oracle
import synth
from synth import workloads as wl

pytestmark = pytest.mark.gpu


def _score_bound(w, x, s_ref):
    # the scorer tolerance used throughout: |Δs| <= 1e-4·(|s| + Σ_j |W2_gj|·|h_j|)
    h = torch.nn.functional.silu(x.double().cpu() @ w["w1"].double().cpu().T).abs()
    return 1e-4 * (s_ref.double().cpu().abs() + h @ w["w2"].double().cpu().abs().T)


def test_noalloc_score_matches_workspace_score_twice():
    from sliding_window_anchor_b200 import _lib, build
    build.build()
    L = _lib.lib()
    seed = 4242
    wdev = wl.make_weights(seed, 0, device="cuda")
    wcpu = wl.make_weights(seed, 0)
    ptrs = [wdev[k].data_ptr() for k in ("w_qkv", "w_o", "q_norm_swa", "k_norm_swa",
                                         "q_norm_rma", "k_norm_rma", "w1", "w2")]
    cw = _lib.CWeights(*ptrs)  # no prepared terms: each call splits W1 in its scratch
    terms = torch.empty(3, 256, 2560, dtype=torch.bfloat16, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.er_score_split_w1(ctypes.c_void_p(wdev["w1"].data_ptr()),
                               ctypes.c_void_p(terms.data_ptr()), stream) == 0
    cw_split = _lib.CWeights(*ptrs, terms.data_ptr(), None)  # terms prepared once
    code = ctypes.c_int32(0)
    assert L.er_last_call_error(ctypes.byref(code), stream) in (0, -4)  # start from a clear word
    cap = 256
    for call, (n, weights) in enumerate(((cap, cw), (100, cw), (cap, cw_split))):
        x = synth.normal((n, 2560), seed, synth.MISC + call, torch.bfloat16, "cuda")
        ws = torch.empty(L.er_score_workspace_bytes(n), dtype=torch.uint8, device="cuda")
        s_ref = torch.empty(n, 4, dtype=torch.float32, device="cuda")
        s_new = torch.full((n, 4), float("nan"), dtype=torch.float32, device="cuda")
        assert L.er_rma_score(ctypes.byref(weights), ctypes.c_void_p(x.data_ptr()), n,
                              ctypes.c_void_p(s_ref.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
                              ws.numel(), stream) == 0
        assert L.er_rma_score_noalloc(ctypes.byref(weights), ctypes.c_void_p(x.data_ptr()), n,
                                      ctypes.c_void_p(s_new.data_ptr()), stream) == 0
        torch.cuda.synchronize()
        assert L.er_last_call_error(ctypes.byref(code), stream) == 0 and code.value == 0, call
        # the same kernels in the same order: the same bits
        assert torch.equal(s_new, s_ref), (call, float((s_new - s_ref).abs().max()))
        # and within the scorer tolerance of the CPU oracle
        ref = oracle.score(wcpu["w1"], wcpu["w2"], x.cpu())
        diff = (s_new.double().cpu() - ref.double()).abs()
        assert bool((diff <= _score_bound(wcpu, x, ref)).all()), (call, float(diff.max()))
    # above the fixed maximum: refused, nothing launched
    before = L.er_launch_count()
    x = torch.zeros(cap + 1, 2560, dtype=torch.bfloat16, device="cuda")
    s = torch.empty(cap + 1, 4, dtype=torch.float32, device="cuda")
    assert L.er_rma_score_noalloc(ctypes.byref(cw), ctypes.c_void_p(x.data_ptr()), cap + 1,
                                  ctypes.c_void_p(s.data_ptr()), stream) == -2
    assert L.er_launch_count() == before
