"""Shared test helpers: building matching oracle / device weights and states.

The oracle side seeds with oracle.norm_rope, the device side with the
library's er_qk_norm_rope; both draw the same raw numbers from synth.
"""
from __future__ import annotations

import torch

import oracle
import synth
from synth import workloads as wl

D, HIDDEN, NG, NH, WIN, BANK, PEND = 256, 2560, 4, 16, 1024, 1024, 256


def oracle_weights(seed, layer):
    w = wl.make_weights(seed, layer)
    return oracle.OracleWeights(w["w_qkv"], w["w_o"], w["q_norm_swa"], w["k_norm_swa"],
                                w["q_norm_rma"], w["k_norm_rma"], w["w1"], w["w2"]), w


def gpu_weights(seed, layer, prepare=True):
    """Device weights; prepare=True gives the fused q/k/v + W1-term GEMM weights."""
    import sliding_window_anchor_b200 as sab
    w = wl.make_weights(seed, layer, device="cuda")
    return sab.LayerWeights.from_dict(w, prepare=prepare), w


def gpu_normrope(x, gain, pos):
    import sliding_window_anchor_b200 as sab
    return sab.qk_norm_rope(x.contiguous(), gain, pos.to(torch.int32).contiguous())


def seed_gpu_state(st, n_layers, t0, pend_mode, seed, wdicts, plain_keys=False,
                   dup_scores=False):
    return wl.seed_state(st.arrays(), range(st.s_max), n_layers, t0, pend_mode, seed, wdicts,
                         gpu_normrope, device="cuda", plain_keys=plain_keys,
                         dup_scores=dup_scores)


def seed_oracle_state(ost, seqs, n_layers, t0, pend_mode, seed, wdicts, plain_keys=False,
                      dup_scores=False):
    arrays = {n: getattr(ost, n) for n in oracle.OracleState.ARRAYS}
    return wl.seed_state(arrays, seqs, n_layers, t0, pend_mode, seed, wdicts, oracle.norm_rope,
                         device="cpu", plain_keys=plain_keys, dup_scores=dup_scores)


def upload_state(st, ost, rows=None):
    """Copy an oracle state's arrays into device state rows (default: the same rows)."""
    rows = list(range(ost.s_max)) if rows is None else list(rows)
    for n in oracle.OracleState.ARRAYS:
        src = getattr(ost, n)
        dst = getattr(st, n)
        for i, r in enumerate(rows):
            dst[r].copy_(src[i])


def download_row(st, row):
    """One device state row as CPU tensors (dict)."""
    return {n: getattr(st, n)[row].cpu() for n in oracle.OracleState.ARRAYS}


def tol_ok(gpu, ref, atol=1e-2, rtol=1e-2):
    """The stated tolerance for attention/layer outputs: |Δ| <= atol + rtol·|ref|."""
    g = gpu.double().cpu()
    r = ref.double().cpu()
    return bool(((g - r).abs() <= atol + rtol * r.abs()).all())


def max_err(gpu, ref):
    return float((gpu.double().cpu() - ref.double().cpu()).abs().max())


def kept_sets_agree(gpu_row, ost_row, n_layers):
    """Bank position sets per (layer, group) match, up to near-ties at the boundary."""
    for l in range(n_layers):
        for g in range(4):
            c = int(ost_row["meta"][2])
            gp = set(gpu_row["bank_pos"][l, g, :c].tolist())
            op = set(ost_row["bank_pos"][l, g, :c].tolist())
            if gp == op:
                continue
            # records only one side kept must sit at the boundary score within 1e-5 relative
            ob = ost_row["bank_score"][l, g, :c].double()
            smin = float(ob.min())
            for side, pos_set, other, scores, poss in (
                    ("gpu", gp, op, gpu_row["bank_score"][l, g, :c], gpu_row["bank_pos"][l, g, :c]),
                    ("oracle", op, gp, ost_row["bank_score"][l, g, :c], ost_row["bank_pos"][l, g, :c])):
                for pos in pos_set - other:
                    s = float(scores[(poss == pos).nonzero()[0, 0]])
                    assert abs(s - smin) <= 1e-5 * max(abs(smin), 1e-30) + 1e-12, (side, l, g, pos)
    return True
