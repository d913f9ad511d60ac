"""The long prefill workload at full length on the device: one stream of 131,072
tokens through 8 layers in 512 chunks of 256, every 4096th token scaled by 4.

Three checks, all against things the device path does not compute:

- the first two chunks of every layer against the oracle run from the empty state;
- the last chunk against the oracle after a state handoff: the device state just
  before that chunk is copied into the oracle, both run the chunk, and the outputs,
  the metadata and the kept anchor sets are compared;
- the selection over the whole stream.  Chunks are aligned to the 256-record
  pending block, so every commit keeps the top 1024 of (bank ∪ block).  For a total
  order, top-k(top-k(A) ∪ B) = top-k(A ∪ B), so the final bank of each (layer,
  group) must be the top 1024 of all 131,072 records by (score desc, position
  asc).  That includes the scaled tokens: each one stays exactly when fewer than
  1024 records outrank it.  The exact scores come from a float64 matmul of the
  same inputs (W2·SiLU(W1·x)), pinned on the chunks above against the oracle's
  scorer.

The bars are the attention tolerance |Δ| <= 1e-2 + 1e-2·|oracle|, kept sets equal
except for records within 1e-5 relative of the boundary score, and stored scores
within 1e-4·(|s| + Σ_j |W2_gj|·|SiLU(h_j)|) of the exact ones.
"""
from concurrent.futures import ThreadPoolExecutor

import pytest
import torch

import oracle
from synth import workloads as wl
from tests import helpers as H

pytestmark = pytest.mark.gpu

CHUNK, N_CHUNKS, L, BIG, NG, BANK = 256, 512, 8, 4096, 4, 1024
FIRST = 2  # chunks checked from the empty state


@pytest.fixture(scope="module")
def sab():
    from sliding_window_anchor_b200 import build
    build.build()
    import sliding_window_anchor_b200 as m
    return m


def _layer_slice(row, l):
    """One layer of a downloaded state row, shaped like a one-layer oracle row."""
    return {n: (v if n == "meta" else v[l:l + 1]) for n, v in row.items()}


def test_prefill_stream_131072_tokens_8_layers(sab):
    seed = wl.seed_of(wl.PREFILL)
    cfg = wl.CONFIGS[wl.PREFILL]
    assert cfg["tokens"] == CHUNK * N_CHUNKS and cfg["n_layers"] == L and cfg["chunk"] == CHUNK
    gws, gdicts = zip(*[H.gpu_weights(seed, l) for l in range(L)])
    w1 = [d["w1"].double() for d in gdicts]
    w2 = [d["w2"].double() for d in gdicts]
    n_tok = CHUNK * N_CHUNKS

    st = sab.State(1, L)
    sab.state_init(st, [0])
    ws = torch.empty(sab.prefill_workspace_bytes(CHUNK), dtype=torch.uint8, device="cuda")
    ids = torch.zeros(1, dtype=torch.int32, device="cuda")
    s_exact = torch.empty(L, n_tok, NG, dtype=torch.float64, device="cuda")
    s_cond = torch.empty(L, n_tok, NG, dtype=torch.float64, device="cuda")
    xs, outs, snap = {}, {}, None
    pos = 0
    for c in range(N_CHUNKS):
        if c == N_CHUNKS - 1:
            torch.cuda.synchronize()
            snap = H.download_row(st, 0)
        for l in range(L):
            x = wl.make_x(seed, l, c, range(CHUNK), device="cuda", big_every=BIG, first_pos=pos)
            out = sab.swa_rma_prefill_chunk(st, gws[l], l, 0, x, ws=ws)
            a = torch.nn.functional.silu(x.double() @ w1[l].t())
            s_exact[l, pos:pos + CHUNK] = a @ w2[l].t()
            s_cond[l, pos:pos + CHUNK] = a.abs() @ w2[l].abs().t()
            if c < FIRST or c == N_CHUNKS - 1:
                xs[(c, l)], outs[(c, l)] = x.cpu(), out.cpu()
        sab.advance(st, ids, CHUNK)
        pos += CHUNK
    torch.cuda.synchronize()
    assert sab.last_device_error(st) == 0
    final = H.download_row(st, 0)
    assert final["meta"][:3].tolist() == [n_tok, 0, BANK]

    # ------------------------------------------------------------ the oracle
    ows, wd = zip(*[H.oracle_weights(seed, l) for l in range(L)])

    def from_empty(l):
        ost = oracle.OracleState(1, 1)
        refs = []
        for c in range(FIRST):
            refs.append(ost.prefill_chunk(ows[l], 0, 0, xs[(c, l)]))
            ost.advance(0, CHUNK)
        return refs

    def after_handoff(l):
        ost = oracle.OracleState(1, 1)
        for n in oracle.OracleState.ARRAYS:
            dst = getattr(ost, n)
            if n == "meta":
                dst[0].copy_(snap[n])
            else:
                dst[0, 0].copy_(snap[n][l])
        ref = ost.prefill_chunk(ows[l], 0, 0, xs[(N_CHUNKS - 1, l)])
        ost.advance(0, CHUNK)
        return ref, {n: getattr(ost, n)[0] for n in oracle.OracleState.ARRAYS}

    def scorer(l):
        x = torch.cat([xs[(c, l)] for c in (*range(FIRST), N_CHUNKS - 1)])
        return oracle.score(wd[l]["w1"], wd[l]["w2"], x)

    with ThreadPoolExecutor(8) as ex:
        f_first = [ex.submit(from_empty, l) for l in range(L)]
        f_last = [ex.submit(after_handoff, l) for l in range(L)]
        f_score = [ex.submit(scorer, l) for l in range(L)]
        first = [f.result() for f in f_first]
        last = [f.result() for f in f_last]
        oscore = [f.result() for f in f_score]

    sample = torch.cat([torch.arange(c * CHUNK, (c + 1) * CHUNK)
                        for c in (*range(FIRST), N_CHUNKS - 1)])
    for l in range(L):
        # the float64 matmul scores agree with the oracle's scorer (FP64, rounded to FP32)
        se = s_exact[l, sample].cpu()
        cond = s_cond[l, sample].cpu()
        assert bool(((oscore[l].double() - se).abs()
                     <= 2.0 ** -23 * se.abs() + 1e-12 * cond).all()), l
        for c in range(FIRST):
            assert H.tol_ok(outs[(c, l)], first[l][c]), (l, c, H.max_err(outs[(c, l)], first[l][c]))
        ref, orow = last[l]
        got = outs[(N_CHUNKS - 1, l)]
        assert H.tol_ok(got, ref), (l, H.max_err(got, ref))
        assert torch.equal(final["meta"], orow["meta"])
        H.kept_sets_agree(_layer_slice(final, l), orow, 1)

    # ------------------------------------------- the whole stream's selection
    for l in range(L):
        for g in range(NG):
            s = s_exact[l, :, g]
            order = torch.argsort(-s, stable=True)  # ties: lower position first
            s_k = float(s[order[BANK - 1]])
            want = set(order[:BANK].tolist())
            bank_pos = final["bank_pos"][l, g]
            got = set(bank_pos.tolist())
            assert len(got) == BANK and min(got) >= 0 and max(got) < n_tok, (l, g)
            for p in want ^ got:
                assert abs(float(s[p]) - s_k) <= 1e-5 * max(abs(s_k), 1.0), (l, g, p)
            # stored scores are the kept records' scores within the scorer's bound
            bp = bank_pos.to("cuda", torch.int64)
            stored = final["bank_score"][l, g].to("cuda", torch.float64)
            err = (stored - s[bp]).abs()
            bound = 1e-4 * (s[bp].abs() + s_cond[l, bp, g])
            assert bool((err <= bound).all()), (l, g, float((err / bound).max()))
