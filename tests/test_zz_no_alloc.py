"""The allocation-free scorer, er_rma_score_noalloc, against er_rma_score.

Some callers of this library cannot give it scratch memory: their device
memory belongs to another framework's allocator, or they only receive the
input and output pointers.  For them the library keeps the scorer's scratch
(W1 as three BF16 terms, the partial scores) in a fixed array of its own (at
most 256 tokens per call).  This
file checks, through the C ABI, that the allocation-free call returns what the
workspace call returns, on two calls in a row (the second finds the array
holding the first call's leftovers), and that a size above the maximum is
refused without launching anything.  It is collected last on purpose.
"""
import ctypes

import pytest
import torch

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
    cw = _lib.CWeights(*[wdev[k].data_ptr() for k in ("w_qkv", "w_o", "q_norm_swa", "k_norm_swa",
                                                      "q_norm_rma", "k_norm_rma", "w1", "w2")])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cap = 256
    for call, n in enumerate((cap, 100)):
        x = synth.normal((n, 2560), seed, synth.MISC + call, torch.bfloat16, "cuda")
        ws = torch.empty(L.er_score_workspace_bytes(n), dtype=torch.uint8, device="cuda")
        s_ref = torch.empty(n, 4, dtype=torch.float32, device="cuda")
        s_new = torch.full((n, 4), float("nan"), dtype=torch.float32, device="cuda")
        assert L.er_rma_score(ctypes.byref(cw), ctypes.c_void_p(x.data_ptr()), n,
                              ctypes.c_void_p(s_ref.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
                              ws.numel(), stream) == 0
        assert L.er_rma_score_noalloc(ctypes.byref(cw), ctypes.c_void_p(x.data_ptr()), n,
                                      ctypes.c_void_p(s_new.data_ptr()), stream) == 0
        torch.cuda.synchronize()
        diff = (s_new.double() - s_ref.double()).abs().cpu()
        assert bool(torch.isfinite(s_new).all())
        assert bool((diff <= _score_bound(wdev, x, s_ref)).all()), (call, float(diff.max()))
    # above the fixed maximum: refused, nothing launched
    before = L.er_launch_count()
    x = torch.zeros(cap + 1, 2560, dtype=torch.bfloat16, device="cuda")
    s = torch.empty(cap + 1, 4, dtype=torch.float32, device="cuda")
    assert L.er_rma_score_noalloc(ctypes.byref(cw), ctypes.c_void_p(x.data_ptr()), cap + 1,
                                  ctypes.c_void_p(s.data_ptr()), stream) == -2
    assert L.er_launch_count() == before
