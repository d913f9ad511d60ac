"""Synthetic workloads of the SWA∥RMA decode / commit / prefill path.

Recipes only: shapes, seeds, which stream feeds which tensor, and the value
distributions.  The one step of the layer's own arithmetic a recipe needs
(RMS-norm + RoPE of seeded keys at their source positions) is passed in as a
callable, so the oracle side seeds with the oracle and the device side with
the device kernel; nothing here computes it.

Recipe (stated once, used by tests and bench):
  weights   w_qkv ~ N(0, 1/2560) BF16, w_o ~ N(0, 1/4096) BF16, RMS gains
            1 + 0.1·N(0,1) BF16, w1 ~ N(0, 1/2560) FP32, w2 ~ N(0, 1/256) FP32
  x         BF16 N(0,1) per (step, layer, sequence)
  window    full at t0: slot s holds position t0-1024 + ((s - t0) mod 1024);
            K = normrope(N(0,1), k_norm_swa, position), V = N(0,1)
  bank      full (1024): positions distinct, stratified below t0-1024
            (slot i in [i·w, (i+1)·w), w = (t0-1024)//1024); K normed and
            rotated at that position, V = N(0,1), score FP32 N(0,1)
  pending   fill f per sequence (0, or U{0..255}); record j < f has position
            t0-f+j, K normed/rotated there, V = N(0,1), score FP32 N(0,1)
  meta      {t0, f, 1024, 0}
N(0,1) is the generator's exact-arithmetic Irwin-Hall normal (mean 0, var 1,
support ±6); see synth.h.
"""
from __future__ import annotations

import math

import torch

import synth

D, HIDDEN, NG, NH, WIN, BANK, PEND = 256, 2560, 4, 16, 1024, 1024, 256
QKV = 12288
BASE_SEED = 20261202

# The workloads, by name: sizes, state recipe and the offset of their seed.
DECODE_B1 = "decode_b1_l1_t4096"
COMMIT = "commit_b512_l8"
DECODE_B64 = "decode_b64_l8_t32768"
DECODE_B512 = "decode_b512_l8_t32768"
PREFILL = "prefill_b1_l8_131072"
CONFIGS = {
    DECODE_B1: dict(name=DECODE_B1, B=1, n_layers=1, t0=4096, pend="zero", steps=256,
                    seed_offset=0),
    COMMIT: dict(name=COMMIT, B=512, n_layers=8, t0=32768, pend="full", steps=0, seed_offset=1),
    DECODE_B64: dict(name=DECODE_B64, B=64, n_layers=8, t0=32768, pend="uniform", steps=1024,
                     seed_offset=2),
    DECODE_B512: dict(name=DECODE_B512, B=512, n_layers=8, t0=32768, pend="uniform",
                      steps=2048, seed_offset=3),
    PREFILL: dict(name=PREFILL, B=1, n_layers=8, t0=0, pend="zero", tokens=131072, chunk=256,
                  seed_offset=4),
}


def seed_of(workload: str) -> int:
    """The base seed of a named workload (CONFIGS)."""
    return BASE_SEED + CONFIGS[workload]["seed_offset"]


# --------------------------------------------------------------- weights

def make_weights(seed: int, layer: int, device="cpu") -> dict:
    """One layer's synthetic weights; identical bits on every device."""
    sid = lambda base: synth.stream_id(base, layer)
    s_qkv = float(torch.tensor(1.0 / math.sqrt(HIDDEN), dtype=torch.float32))
    bf, f32 = torch.bfloat16, torch.float32
    w = {
        "w_qkv": synth.normal((QKV, HIDDEN), seed, sid(synth.W_QKV), bf, device, scale=s_qkv),
        "w_o": synth.normal((HIDDEN, NH * D), seed, sid(synth.W_O), bf, device, scale=1.0 / 64),
        "q_norm_swa": synth.normal((D,), seed, sid(synth.G_Q_SWA), bf, device, scale=0.1,
                                   offset=1.0),
        "k_norm_swa": synth.normal((D,), seed, sid(synth.G_K_SWA), bf, device, scale=0.1,
                                   offset=1.0),
        "q_norm_rma": synth.normal((D,), seed, sid(synth.G_Q_RMA), bf, device, scale=0.1,
                                   offset=1.0),
        "k_norm_rma": synth.normal((D,), seed, sid(synth.G_K_RMA), bf, device, scale=0.1,
                                   offset=1.0),
        "w1": synth.normal((256, HIDDEN), seed, sid(synth.W1), f32, device, scale=s_qkv),
        "w2": synth.normal((NG, 256), seed, sid(synth.W2), f32, device, scale=1.0 / 16),
    }
    return w


def make_x(seed: int, layer: int, step: int, seqs, device="cpu", big_every: int = 0,
           first_pos: int = 0) -> torch.Tensor:
    """Hidden states [len(seqs), 2560] for one (step, layer).  `seqs` are global
    sequence ids (rows of the full batch).  With big_every > 0 (prefill), the
    rows are the tokens first_pos.. of one stream and every big_every-th token
    (1-based) is scaled by 4."""
    stream = synth.stream_id(synth.X, layer, step)
    seqs = list(seqs)
    if seqs == list(range(len(seqs))):
        x = synth.normal((len(seqs), HIDDEN), seed, stream, torch.bfloat16, device)
    else:
        x = torch.empty(len(seqs), HIDDEN, dtype=torch.bfloat16, device=device)
        for i, s in enumerate(seqs):
            synth.fill_normal_(x[i], seed, stream, index0=s * HIDDEN)
    if big_every:
        pos = torch.arange(first_pos, first_pos + len(seqs))
        big = ((pos + 1) % big_every == 0).nonzero().flatten().tolist()
        for i in big:
            x[i] = x[i] * 4
    return x


# ---------------------------------------------------------------- state

def window_positions(t0: int, device="cpu") -> torch.Tensor:
    """Position held by each ring slot when the stream is at t0 (t0 >= 1024)."""
    s = torch.arange(WIN, dtype=torch.int64)
    return (t0 - WIN + torch.remainder(s - t0, WIN)).to(torch.int32).to(device)


def pend_fill(seed: int, mode, seqs, device="cpu") -> torch.Tensor:
    """Pending fill per sequence: "zero", "full", "uniform" (U{0..255}), or explicit values."""
    seqs = list(seqs)
    if not isinstance(mode, str):
        return torch.as_tensor(mode, dtype=torch.int32).reshape(len(seqs)).to(device)
    if mode == "zero":
        return torch.zeros(len(seqs), dtype=torch.int32, device=device)
    if mode == "full":
        return torch.full((len(seqs),), PEND, dtype=torch.int32, device=device)
    out = torch.empty(len(seqs), dtype=torch.int32, device=device)
    if seqs == list(range(len(seqs))):
        synth.fill_uniform_(out, seed, synth.PEND_FILL, PEND)
    else:
        for i, s in enumerate(seqs):
            synth.fill_uniform_(out[i:i + 1], seed, synth.PEND_FILL, PEND, index0=s)
    return out


def seed_state(arrays: dict, seqs, n_layers: int, t0: int, pend_mode: str, seed: int,
               weights: list, normrope, device="cpu", plain_keys: bool = False,
               dup_scores: bool = False) -> torch.Tensor:
    """Fill state `arrays` (dict of tensors shaped [n_local, L, 4, slots(, 256)] plus
    meta [n_local, 4]) for local rows 0..len(seqs)-1 holding global sequences `seqs`.

    normrope(x_rows[n,256], gain[256], pos[n] int32) -> rows, applied to seeded
    keys (skipped with plain_keys, the commit workload).  dup_scores plants
    ~5% exact score ties inside each (seq, layer, group) merge.
    Returns the pending fill per local row."""
    seqs = list(seqs)
    n = len(seqs)
    L = n_layers
    ident = seqs == list(range(n))
    bf = torch.bfloat16

    def fill(t: torch.Tensor, stream: int, per_seq: int, kind: str, **kw):
        """Fill t ([n, ...]) so element e of global sequence s uses index s*per_seq + e."""
        if ident:
            _fill_one(t, stream, 0, kind, **kw)
        else:
            for i, s in enumerate(seqs):
                _fill_one(t[i], stream, s * per_seq, kind, **kw)

    def _fill_one(t, stream, index0, kind, **kw):
        if kind == "normal":
            synth.fill_normal_(t, seed, stream, index0=index0)
        elif kind == "strata":
            synth.fill_strata_(t, seed, stream, kw["period"], kw["width"], index0=index0)
        elif kind == "dup":
            synth.fill_normal_dup_(t, seed, stream, kw["group"], kw["one_in"], index0=index0)

    rows_w = L * NG * WIN * D
    rows_b = L * NG * BANK * D
    rows_p = L * NG * PEND * D
    fill(arrays["win_k"], synth.WIN_K, rows_w, "normal")
    fill(arrays["win_v"], synth.WIN_V, rows_w, "normal")
    fill(arrays["bank_k"], synth.BANK_K, rows_b, "normal")
    fill(arrays["bank_v"], synth.BANK_V, rows_b, "normal")
    fill(arrays["pend_k"], synth.PEND_K, rows_p, "normal")
    fill(arrays["pend_v"], synth.PEND_V, rows_p, "normal")
    width = max(1, (t0 - WIN) // BANK)
    fill(arrays["bank_pos"], synth.BANK_POS, L * NG * BANK, "strata", period=BANK, width=width)

    fills = pend_fill(seed, pend_mode, seqs, device)
    if dup_scores:
        sc = torch.empty(n, L, NG, BANK + PEND, dtype=torch.float32, device=device)
        fill(sc, synth.BANK_SCORE, L * NG * (BANK + PEND), "dup", group=BANK + PEND, one_in=20)
        arrays["bank_score"].copy_(sc[..., :BANK])
        arrays["pend_score"].copy_(sc[..., BANK:])
    else:
        fill(arrays["bank_score"], synth.BANK_SCORE, L * NG * BANK, "normal")
        fill(arrays["pend_score"], synth.PEND_SCORE, L * NG * PEND, "normal")

    # pending positions: record j of a sequence with fill f sits at t0 - f + j
    j = torch.arange(PEND, dtype=torch.int32, device=device)
    pp = (t0 - fills.view(n, 1) + j.view(1, PEND)).to(torch.int32)
    arrays["pend_pos"].copy_(pp.view(n, 1, 1, PEND).expand(n, L, NG, PEND))

    if not plain_keys:
        wpos = window_positions(t0, device)
        for i in range(n):
            for l in range(L):
                wk = arrays["win_k"][i, l].reshape(NG * WIN, D)
                wk.copy_(normrope(wk, weights[l]["k_norm_swa"], wpos.repeat(NG)))
                bk = arrays["bank_k"][i, l].reshape(NG * BANK, D)
                bk.copy_(normrope(bk, weights[l]["k_norm_rma"],
                                  arrays["bank_pos"][i, l].reshape(-1).contiguous()))
                f = int(fills[i])
                if f:
                    pk = arrays["pend_k"][i, l, :, :f]
                    rows = pk.reshape(NG * f, D) if pk.is_contiguous() else pk.contiguous().view(
                        NG * f, D)
                    res = normrope(rows.contiguous(), weights[l]["k_norm_rma"],
                                   arrays["pend_pos"][i, l, :, :f].reshape(-1).contiguous())
                    arrays["pend_k"][i, l, :, :f].copy_(res.view(NG, f, D))
    meta = arrays["meta"]
    meta[:, 0] = t0
    meta[:, 1] = fills
    meta[:, 2] = BANK
    meta[:, 3] = 0
    return fills


# ------------------------------------------------------- commit workload

def seed_commit_workload(arrays: dict, seqs, n_layers: int, t0: int, seed: int, rep: int,
                         device="cpu") -> None:
    """The commit microbench workload, repetition `rep`: every (sequence, layer,
    group) holds a full bank (positions stratified below t0-1024) and a full pending
    block (positions t0..t0+255), scores N(0,1) with ~5% exact ties inside each
    merge, meta {t0+256, 256, 1024, 0}.  rep 0 also fills the K/V rows with N(0,1)
    (plain, un-normed); a later repetition draws fresh scores (stream keyed by
    seed and rep) and restores the positions and metadata, leaving the K/V rows as
    they are (their contents do not change which records a merge keeps or moves)."""
    seqs = list(seqs)
    n, L = len(seqs), n_layers
    if rep == 0:
        seed_state(arrays, seqs, L, t0, "full", seed, [None] * L, None, device=device,
                   plain_keys=True, dup_scores=True)
    else:
        seed_r = seed + 7919 * rep
        ident = seqs == list(range(n))
        per = L * NG * (BANK + PEND)
        sc = torch.empty(n, L, NG, BANK + PEND, dtype=torch.float32, device=device)
        width = max(1, (t0 - WIN) // BANK)
        if ident:
            synth.fill_normal_dup_(sc, seed_r, synth.BANK_SCORE, BANK + PEND, 20)
            synth.fill_strata_(arrays["bank_pos"], seed, synth.BANK_POS, BANK, width)
        else:
            for i, s in enumerate(seqs):
                synth.fill_normal_dup_(sc[i], seed_r, synth.BANK_SCORE, BANK + PEND, 20,
                                       index0=s * per)
                synth.fill_strata_(arrays["bank_pos"][i], seed, synth.BANK_POS, BANK, width,
                                   index0=s * L * NG * BANK)
        arrays["bank_score"].copy_(sc[..., :BANK])
        arrays["pend_score"].copy_(sc[..., BANK:])
    j = torch.arange(PEND, dtype=torch.int32, device=device)
    arrays["pend_pos"].copy_((t0 + j).view(1, 1, 1, PEND).expand_as(arrays["pend_pos"]))
    meta = arrays["meta"]
    meta[:, 0] = t0 + PEND
    meta[:, 1] = PEND
    meta[:, 2] = BANK
    meta[:, 3] = 0
