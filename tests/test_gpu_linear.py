"""GPU parity of the tensor-core projections (er_linear, the a1 / a6 GEMMs).

y = x·wᵀ with BF16 operands and FP32 accumulation, at the layer's shapes
(F = 13056 / 12288 rows of the fused q/k/v (+ W1 terms) weight, K = 2560;
F = 2560, K = 4096 for o_proj) and token counts from one decode token to a
512-sequence batch, ragged counts included (they leave part of a 16-token
group and of a tile empty).  Up to 32 tokens the call runs the weight-
streaming kernel the layer calls use for small batches (1, 2 or 4 tiles of 8
tokens, K split between the warps of a block); above, the tcgen05 GEMM, which
splits the work between CTA pairs so that some tiles are finished from
partial sums of other pairs; every shape below exercises that path at some
token count.

Bars:
  FP32 output: |Δ| <= 2^-17·Σ_k |x_k·w_k| against a float64 matmul (FP32
    accumulation of 2560-4096 exact BF16 products; the bound is ~30x the
    expected rounding of such sums and far below any indexing mistake).
  BF16 output: against the float64 sum rounded once to BF16 (the oracle's
    linear): every element within one BF16 ulp (plus the FP32 accumulation
    bound above, which matters only where the sum nearly cancels), at least
    99% identical.
  Same inputs, same bits (fixed summation order).
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sab():
    from sliding_window_anchor_b200 import build
    build.build()
    import sliding_window_anchor_b200 as m
    return m


def _weights(F, K, seed):
    return synth.normal((F, K), seed, synth.MISC + 7, torch.bfloat16, scale=K ** -0.5)


def _x(T, K, seed):
    return synth.normal((T, K), seed, synth.MISC + 8, torch.bfloat16)


def bf16_exact(a):
    """float64 -> BF16 with one round-to-nearest-even (numpy frexp/rint)."""
    a = np.asarray(a, dtype=np.float64)
    m, e = np.frexp(a)
    y = np.ldexp(np.rint(m * 256.0), e - 8)
    return torch.from_numpy(y.astype(np.float32)).to(torch.bfloat16)


@pytest.mark.parametrize("F,K", [(13056, 2560), (12288, 2560), (2560, 4096)])
@pytest.mark.parametrize("T", [1, 7, 9, 16, 24, 32, 33, 100, 256, 300, 512])
def test_linear_fp32_matches_float64(sab, F, K, T):
    w = _weights(F, K, 11 + F)
    x = _x(T, K, 13 + T)
    got = sab.linear(x.cuda(), w.cuda(), fp32_out=True)
    assert sab.last_call_error() == 0
    ref = x.double() @ w.double().T
    mag = x.double().abs() @ w.double().abs().T
    err = (got.double().cpu() - ref).abs()
    assert bool((err <= 2.0 ** -17 * mag + 1e-30).all()), float((err / mag).max())
    # same inputs, same bits
    again = sab.linear(x.cuda(), w.cuda(), fp32_out=True)
    assert torch.equal(got, again)


@pytest.mark.parametrize("T", [1, 5, 16, 31, 64, 77, 256, 512])
def test_linear_bf16_matches_single_rounding(sab, T):
    F, K = 2560, 4096
    w = _weights(F, K, 5)
    x = _x(T, K, 6 + T)
    got = sab.linear(x.cuda(), w.cuda()).cpu()
    exact = x.double() @ w.double().T
    ref = bf16_exact(exact.numpy())
    # one BF16 ulp of the result, plus the FP32 accumulation error (which decides
    # the rounding only where the sum nearly cancels)
    mag = x.double().abs() @ w.double().abs().T
    ulp = ref.double().abs() * 2.0 ** -7 + 2.0 ** -17 * mag
    diff = (got.double() - ref.double()).abs()
    assert bool((diff <= ulp).all()), float((diff / ulp).max())
    assert float((got == ref).double().mean()) >= 0.99
    if T <= 16:
        # the oracle's own linear (float64 then one BF16 rounding) on a few tokens
        for t in range(min(T, 2)):
            assert torch.equal(oracle.linear_bf16(w, x[t]), ref[t])


@pytest.mark.parametrize("T", [7, 40])
def test_linear_row_stride_and_zero_tokens(sab, T):
    """Output rows with a stride above F (the fused projection's layout) leave the
    columns past F untouched, in both kernels (7 tokens: the weight-streaming one,
    40: the tcgen05 GEMM); T = 0 launches nothing."""
    F, K = 2560, 2560
    w = _weights(F, K, 21)
    x = _x(T, K, 22)
    out = torch.full((T, F + 256), 7.0, dtype=torch.float32, device="cuda")
    sab.linear(x.cuda(), w.cuda(), fp32_out=True, out=out)
    ref = sab.linear(x.cuda(), w.cuda(), fp32_out=True)
    assert torch.equal(out[:, :F], ref)
    assert bool((out[:, F:] == 7.0).all())
    n0 = sab.launch_count()
    empty = torch.empty(0, K, dtype=torch.bfloat16, device="cuda")
    sab.linear(empty, w.cuda())
    assert sab.launch_count() == n0
