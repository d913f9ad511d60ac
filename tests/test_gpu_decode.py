"""GPU parity of whole decode steps (a1–a7) and prefill chunks (a8) against the oracle.

Workloads follow the synthetic recipe of synth/workloads.py.  The device
seeds its own state (its norm/RoPE kernel) and the oracle seeds its own, from
the same generator numbers.  Bars: the stated |Δ| <= 1e-2 + 1e-2·|oracle| on
every layer output, and kept anchor sets equal except where two records'
scores differ by less than 1e-5 relative at the keep/evict boundary.
"""
import time
from concurrent.futures import ThreadPoolExecutor

import pytest
import torch

import oracle
import synth
from synth import workloads as wl
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sab():
    from sliding_window_anchor_b200 import build
    build.build()
    import sliding_window_anchor_b200 as m
    return m


def _run_oracle_seq(ow_list, ost, row, steps, layers, seed, gseq, x_of):
    outs = {}
    for step in range(steps):
        for l in layers:
            outs[(step, l)] = ost.decode_layer(ow_list[l], l, row, x_of(step, l, gseq))
        ost.advance(row)
    return outs


def test_decode_single_layer_256_steps_with_commit(sab):
    """B=1, one layer, state at 4096, empty pending: 256 steps, one commit at the last."""
    cfg, seed = wl.CONFIGS[wl.DECODE_B1], wl.seed_of(wl.DECODE_B1)
    L = cfg["n_layers"]
    ow, wdict = H.oracle_weights(seed, 0)
    gw, gdict = H.gpu_weights(seed, 0)
    ost = oracle.OracleState(1, L)
    H.seed_oracle_state(ost, [0], L, cfg["t0"], cfg["pend"], seed, [wdict])
    st = sab.State(1, L)
    H.seed_gpu_state(st, L, cfg["t0"], cfg["pend"], seed, [gdict])
    ws = torch.empty(sab.decode_workspace_bytes(1), dtype=torch.uint8, device="cuda")
    gouts = []
    for step in range(cfg["steps"]):
        x = wl.make_x(seed, 0, step, [0], device="cuda")
        gouts.append(sab.swa_rma_decode(st, gw, 0, [0], x, ws=ws).cpu())
        sab.advance(st, [0])
    assert sab.last_device_error(st) == 0
    worst = 0.0
    for step in range(cfg["steps"]):
        ref = ost.decode_layer(ow, 0, 0, wl.make_x(seed, 0, step, [0])[0])
        ost.advance(0)
        assert H.tol_ok(gouts[step][0], ref), (step, H.max_err(gouts[step][0], ref))
        worst = max(worst, H.max_err(gouts[step][0], ref) / float(ref.double().abs().max()))
    print(f"{wl.DECODE_B1} worst |Δ|/max|ref| = {worst:.3e}")
    assert worst < 2e-2
    grow, orow = H.download_row(st, 0), {n: getattr(ost, n)[0] for n in oracle.OracleState.ARRAYS}
    assert torch.equal(grow["meta"], orow["meta"])
    assert int(orow["meta"][1]) == 0 and int(orow["meta"][0]) == cfg["t0"] + 256
    H.kept_sets_agree(grow, orow, L)


def _pick_sequences(fills, steps, n_commit, n_other):
    """Rows whose blocks fill at distinct steps inside `steps` (a staggered commit
    each, spread over the run), plus rows that commit later or never in it."""
    commit_step = {b: 255 - int(f) for b, f in enumerate(fills)}  # first commit's step
    by_step = {}
    for b, s in commit_step.items():
        if s < steps:
            by_step.setdefault(s, b)
    steps_sorted = sorted(by_step)
    assert len(steps_sorted) >= n_commit, "the fills give too few distinct commit steps"
    idx = [round(i * (len(steps_sorted) - 1) / max(n_commit - 1, 1)) for i in range(n_commit)]
    chosen = [by_step[steps_sorted[i]] for i in idx]
    late = sorted((b for b, s in commit_step.items() if s >= steps), key=lambda b: commit_step[b])
    chosen += [b for b in late if b not in chosen][:n_other]
    return chosen


# the B=512 decode batch: the oracle follows 8 sequences for 64 steps, 6 of them
# committing at different steps; the B=64 batch: 300 steps, so every followed sequence
# crosses its commit (staggered by its fill) and the fullest ones a second one
BATCHED = {wl.DECODE_B64: dict(steps=300, n_commit=6, n_other=0),
           wl.DECODE_B512: dict(steps=64, n_commit=6, n_other=2)}


@pytest.mark.parametrize("workload", [wl.DECODE_B64, wl.DECODE_B512])
def test_decode_batched_sampled_sequences(sab, workload):
    """Full batch on the device (B=64 or 512, 8 layers, t0=32768, random fills); the
    oracle follows sampled sequences through staggered, device-gated commits.  Every
    layer output of every step within the stated tolerance; metadata equal and kept
    anchor sets equal (up to boundary near-ties) at the end."""
    cfg, seed = wl.CONFIGS[workload], wl.seed_of(workload)
    plan = BATCHED[workload]
    B, L, steps = cfg["B"], cfg["n_layers"], plan["steps"]
    gws, gdicts = zip(*[H.gpu_weights(seed, l) for l in range(L)])
    st = sab.State(B, L)
    fills = H.seed_gpu_state(st, L, cfg["t0"], cfg["pend"], seed, list(gdicts)).cpu()
    sampled = _pick_sequences(fills.tolist(), steps, plan["n_commit"], plan["n_other"])
    rows = torch.tensor(sampled, dtype=torch.long, device="cuda")
    ws = torch.empty(sab.decode_workspace_bytes(B), dtype=torch.uint8, device="cuda")
    ids = torch.arange(B, dtype=torch.int32, device="cuda")
    out = torch.empty(B, 2560, dtype=torch.bfloat16, device="cuda")
    gouts = torch.empty(steps, L, len(sampled), 2560, dtype=torch.bfloat16, device="cuda")
    for step in range(steps):
        for l in range(L):
            x = wl.make_x(seed, l, step, range(B), device="cuda")
            sab.swa_rma_decode(st, gws[l], l, ids, x, out=out, ws=ws)
            gouts[step, l] = out[rows]
        sab.advance(st, ids)
    assert sab.last_device_error(st) == 0
    gouts = gouts.cpu()
    commits = [255 - int(fills[b]) for b in sampled]
    assert len({c for c in commits if c < steps}) >= plan["n_commit"], commits

    ows, wdicts = zip(*[H.oracle_weights(seed, l) for l in range(L)])

    def run(gseq):
        ost = oracle.OracleState(1, L)
        H.seed_oracle_state(ost, [gseq], L, cfg["t0"], cfg["pend"], seed, list(wdicts))
        x_of = lambda step, l, s: wl.make_x(seed, l, step, [s])[0]
        return ost, _run_oracle_seq(ows, ost, 0, steps, range(L), seed, gseq, x_of)

    with ThreadPoolExecutor(len(sampled)) as ex:
        results = list(ex.map(run, sampled))
    for i, (gseq, (ost, outs)) in enumerate(zip(sampled, results)):
        for (step, l), ref in outs.items():
            got = gouts[step, l, i]
            assert H.tol_ok(got, ref), (gseq, step, l, H.max_err(got, ref))
        grow = H.download_row(st, gseq)
        orow = {n: getattr(ost, n)[0] for n in oracle.OracleState.ARRAYS}
        assert torch.equal(grow["meta"], orow["meta"]), gseq
        H.kept_sets_agree(grow, orow, L)


def test_graph_replayed_steps_equal_eager_steps_and_oracle(sab):
    """A whole 8-layer step (the layer calls with their device-gated commits, then
    the advance) captured once into a CUDA graph and replayed across steps in which
    some sequences commit and others do not: the same bits as the same steps run
    call by call on a copy of the state, outputs and every state array; sampled
    sequences (one committing, one not) within tolerance of the oracle."""
    cfg, seed = wl.CONFIGS[wl.DECODE_B64], wl.seed_of(wl.DECODE_B64)
    B, L = cfg["B"], cfg["n_layers"]
    gws, gdicts = zip(*[H.gpu_weights(seed, l) for l in range(L)])
    st_g = sab.State(B, L)
    fills = H.seed_gpu_state(st_g, L, cfg["t0"], cfg["pend"], seed, list(gdicts)).cpu()
    st_e = sab.State(B, L)
    st_e.blob.copy_(st_g.blob)
    steps = max(4, 257 - int(fills.max()))
    assert steps <= 48, steps
    committing = [b for b in range(B) if 255 - int(fills[b]) < steps]
    assert committing and len(committing) < B
    ids = torch.arange(B, dtype=torch.int32, device="cuda")
    xbuf = [torch.empty(B, 2560, dtype=torch.bfloat16, device="cuda") for _ in range(L)]
    obuf = [torch.empty(B, 2560, dtype=torch.bfloat16, device="cuda") for _ in range(L)]
    ws_g = torch.empty(sab.decode_workspace_bytes(B), dtype=torch.uint8, device="cuda")
    ws_e = torch.empty_like(ws_g)

    def step_calls(st, ws, xs, outs):
        for l in range(L):
            sab.swa_rma_decode(st, gws[l], l, ids, xs[l], out=outs[l], ws=ws)
        sab.advance(st, ids)

    # the library's per-device resources exist before capture (a warm-up call on a
    # scratch state), then one step is captured
    st_w = sab.State(B, L)
    st_w.blob.copy_(st_g.blob)
    step_calls(st_w, ws_g, [wl.make_x(seed, l, 0, range(B), device="cuda") for l in range(L)],
               obuf)
    torch.cuda.synchronize()
    del st_w
    side = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        step_calls(st_g, ws_g, xbuf, obuf)
    sampled = [committing[0], next(b for b in range(B) if b not in committing)]
    g_out, e_out = [], []
    for step in range(steps):
        xs = [wl.make_x(seed, l, step, range(B), device="cuda") for l in range(L)]
        for l in range(L):
            xbuf[l].copy_(xs[l])
        graph.replay()
        g_out.append(torch.stack([o.clone() for o in obuf]))
        outs = [torch.empty(B, 2560, dtype=torch.bfloat16, device="cuda") for _ in range(L)]
        step_calls(st_e, ws_e, xs, outs)
        e_out.append(torch.stack(outs))
    torch.cuda.synchronize()
    del graph
    assert sab.last_device_error(st_g) == 0 and sab.last_device_error(st_e) == 0
    for step in range(steps):
        assert torch.equal(g_out[step], e_out[step]), step
    assert torch.equal(st_g.blob, st_e.blob)
    assert all(int(st_g.meta[b, 1]) == (int(fills[b]) + steps) % 256 for b in range(B))

    ows, wdicts = zip(*[H.oracle_weights(seed, l) for l in range(L)])
    for gseq in sampled:
        ost = oracle.OracleState(1, L)
        H.seed_oracle_state(ost, [gseq], L, cfg["t0"], cfg["pend"], seed, list(wdicts))
        x_of = lambda step, l, s: wl.make_x(seed, l, step, [s])[0]
        outs = _run_oracle_seq(ows, ost, 0, steps, range(L), seed, gseq, x_of)
        for (step, l), ref in outs.items():
            got = g_out[step][l, gseq].cpu()
            assert H.tol_ok(got, ref), (gseq, step, l, H.max_err(got, ref))
        orow = {n: getattr(ost, n)[0] for n in oracle.OracleState.ARRAYS}
        grow = H.download_row(st_g, gseq)
        assert torch.equal(grow["meta"], orow["meta"])
        H.kept_sets_agree(grow, orow, L)


PREFILL_CASES = {
    # seeded at 4096: the ring wraps for every query; a full chunk (commits) then a ragged one
    "wrap_t4096": dict(t0=4096, pend=0, bank=None, chunks=(256, 37)),
    # the last chunk of the 131072-token stream (its last token is one of the x4 ones)
    "last_chunk_t130816": dict(t0=130816, pend=0, bank=None, chunks=(256,)),
    # a partly filled bank, 100 records already pending, an unaligned stream position
    "partial_bank_t5000": dict(t0=5000, pend=100, bank=700, chunks=(156, 40)),
    # the stream start: empty state, the ring partly written, the bank growing
    "stream_start": dict(t0=None, pend=0, bank=None, chunks=(256, 256, 77, 50)),
    # weights without preparation: the projection and the scorer as separate launches
    # (prefill and, through the replay, decode)
    "partial_bank_t5000_unprepared": dict(t0=5000, pend=100, bank=700, chunks=(156, 40),
                                          prepare=False),
}


@pytest.mark.parametrize("case", list(PREFILL_CASES))
def test_prefill_chunks_match_oracle_and_decode(sab, case):
    """One layer: each chunk through er_swa_rma_prefill_chunk against the oracle's
    prefill and against the same tokens replayed one by one through the decode path
    (state row 1); states and kept anchor sets must agree afterwards."""
    cfg = PREFILL_CASES[case]
    seed = wl.seed_of(wl.PREFILL)
    L = 1
    ow, wdict = H.oracle_weights(seed, 0)
    gw, gdict = H.gpu_weights(seed, 0, prepare=cfg.get("prepare", True))
    ost = oracle.OracleState(1, L)
    st = sab.State(2, L)
    if cfg["t0"] is None:
        sab.state_init(st, [0, 1])
        pos = 0
    else:
        H.seed_oracle_state(ost, [0], L, cfg["t0"], [cfg["pend"]], seed, [wdict])
        H.seed_gpu_state(st, L, cfg["t0"], [cfg["pend"]] * 2, seed, [gdict])
        if cfg["bank"] is not None:
            ost.meta[0, 2] = cfg["bank"]
            st.meta[:, 2] = cfg["bank"]
        pos = cfg["t0"]
    for n in oracle.OracleState.ARRAYS:
        getattr(st, n)[1].copy_(getattr(st, n)[0])
    for ci, T in enumerate(cfg["chunks"]):
        x = wl.make_x(seed, 0, 1000 + ci, range(T), big_every=4096, first_pos=pos)
        got = sab.swa_rma_prefill_chunk(st, gw, 0, 0, x.cuda())
        sab.advance(st, [0], T)
        dec = []
        for i in range(T):
            dec.append(sab.swa_rma_decode(st, gw, 0, [1], x[i:i + 1].cuda()))
            sab.advance(st, [1])
        dec = torch.cat(dec).cpu()
        ref = ost.prefill_chunk(ow, 0, 0, x)
        ost.advance(0, T)
        assert H.tol_ok(got.cpu(), ref), (case, ci, H.max_err(got.cpu(), ref))
        assert H.tol_ok(got.cpu(), dec), (case, ci, H.max_err(got.cpu(), dec))
        pos += T
    assert sab.last_device_error(st) == 0
    g0, g1 = H.download_row(st, 0), H.download_row(st, 1)
    orow = {n: getattr(ost, n)[0] for n in oracle.OracleState.ARRAYS}
    assert torch.equal(g0["meta"], orow["meta"]) and torch.equal(g1["meta"], orow["meta"])
    H.kept_sets_agree(g0, orow, L)
    H.kept_sets_agree(g1, orow, L)


def test_snapshot_restore_is_bit_identical(sab):
    """The state is flat fixed-size memory: a copy taken mid-stream replays exactly."""
    seed = 77
    gw, gdict = H.gpu_weights(seed, 0)
    st = sab.State(3, 1)
    H.seed_gpu_state(st, 1, 4096, [250, 0, 17], seed, [gdict])
    snap = st.blob.clone()
    runs = []
    for rep in range(2):
        st.blob.copy_(snap)
        outs = []
        for step in range(8):
            x = wl.make_x(seed, 0, step, range(3), device="cuda")
            outs.append(sab.swa_rma_decode(st, gw, 0, [0, 1, 2], x))
            sab.advance(st, [0, 1, 2])
        runs.append((torch.stack(outs), st.blob.clone()))
    assert torch.equal(runs[0][0], runs[1][0])
    assert torch.equal(runs[0][1], runs[1][1])


def test_out_of_range_sequence_is_recorded_not_faulted(sab):
    gw, gdict = H.gpu_weights(5, 0)
    st = sab.State(2, 1)
    H.seed_gpu_state(st, 1, 4096, [3, 4], 5, [gdict])
    x = wl.make_x(5, 0, 0, range(2), device="cuda")
    sab.swa_rma_decode(st, gw, 0, torch.tensor([0, 7], dtype=torch.int32, device="cuda"), x)
    torch.cuda.synchronize()
    assert sab.last_device_error(st) == -1
    # a block that is already full cannot take the token's record
    st.meta[1, 1] = 256
    sab.swa_rma_decode(st, gw, 0, [0, 1], x)
    assert sab.last_device_error(st) == -2


def test_bounded_wait_runs_out_and_the_context_survives(sab):
    """The failure path of every pipeline barrier: a wait that nothing completes
    gives up after ~2 s, records ER_ETIMEOUT and returns; afterwards the context
    runs the library's kernels normally (no fault, no hang)."""
    import time
    st = sab.State(1, 1)
    sab.state_init(st, [0])
    assert sab.last_device_error(st) == 0
    sab.wait_selftest(st, arrive=True)  # a completed barrier: nothing recorded
    assert sab.last_device_error(st) == 0
    t0 = time.time()
    sab.wait_selftest(st, arrive=False)
    code = sab.last_device_error(st)
    waited = time.time() - t0
    assert code == -5, code  # ER_ETIMEOUT
    assert 1.5 < waited < 30.0, waited
    # the context is intact: norm/RoPE through the library still matches the oracle
    x = synth.normal((64, 256), 9, synth.MISC, torch.bfloat16)
    g = synth.normal((256,), 9, synth.MISC + 1, torch.bfloat16, scale=0.1, offset=1.0)
    pos = torch.arange(64, dtype=torch.int32) * 977
    got = sab.qk_norm_rope(x.cuda(), g.cuda(), pos.cuda()).cpu()
    ref = oracle.norm_rope(x, g, pos)
    assert (got == ref).double().mean() > 0.99
    assert sab.last_device_error(st) == 0


def test_stateless_calls_report_a_wait_that_gave_up(sab):
    """The calls that take no state (the standalone scorers) record into the
    library's own error word: a bounded wait run out through it is reported by
    er_last_call_error, which then reads clear; the scorer with an explicit word
    records nothing on a normal call and its scores are unchanged."""
    assert sab.last_call_error() in (0, -5)  # clear whatever an earlier test left
    sab.wait_selftest(None, arrive=True)
    assert sab.last_call_error() == 0
    t0 = time.time()
    sab.wait_selftest(None, arrive=False)
    assert sab.last_call_error() == -5  # ER_ETIMEOUT
    assert 1.5 < time.time() - t0 < 30.0
    assert sab.last_call_error() == 0
    seed = 321
    gw, wdev = H.gpu_weights(seed, 0)
    x = synth.normal((64, 2560), seed, synth.MISC, torch.bfloat16, "cuda")
    word = torch.zeros(4, dtype=torch.int32, device="cuda")
    s_ex = sab.rma_score(gw, x, dev_error=word)
    s_lib = sab.rma_score(gw, x)
    assert torch.equal(s_ex, s_lib)
    assert int(word[0]) == 0 and sab.last_call_error() == 0


RMA_ARRAYS = ("bank_k", "bank_v", "pend_k", "pend_v", "bank_score", "pend_score", "bank_pos",
              "pend_pos")


def test_rma_off_decode_matches_oracle_and_freezes_the_memory(sab):
    """The pages' ablation (ER_FLAG_RMA_OFF): o_rma = 0, no score, append or commit; the
    anchor memory and its counters stay bit-identical while the window moves on."""
    seed, L, B, t0 = 61, 1, 8, 32768
    gw, gdict = H.gpu_weights(seed, 0)
    ow, wdict = H.oracle_weights(seed, 0)
    fills = [250, 255, 0, 17, 128, 254, 3, 200]  # several would commit within 8 steps
    st = sab.State(B, L)
    H.seed_gpu_state(st, L, t0, fills, seed, [gdict])
    before = {n: getattr(st, n).clone() for n in RMA_ARRAYS}
    meta0 = st.meta.clone()
    ids = torch.arange(B, dtype=torch.int32, device="cuda")
    steps = 8
    gouts = []
    for step in range(steps):
        x = wl.make_x(seed, 0, step, range(B), device="cuda")
        gouts.append(sab.swa_rma_decode(st, gw, 0, ids, x, rma_off=True).cpu())
        sab.advance(st, ids, rma_off=True)
    assert sab.last_device_error(st) == 0
    for n in RMA_ARRAYS:
        assert torch.equal(getattr(st, n), before[n]), n
    meta = st.meta.cpu()
    assert torch.equal(meta[:, 0], meta0[:, 0].cpu() + steps)
    assert torch.equal(meta[:, 1:], meta0[:, 1:].cpu())
    for gseq in (1, 3):  # one whose block is full, one that would not commit
        ost = oracle.OracleState(1, L)
        H.seed_oracle_state(ost, [gseq], L, t0, [fills[gseq]], seed, [wdict])
        for step in range(steps):
            ref = ost.decode_layer(ow, 0, 0, wl.make_x(seed, 0, step, [gseq])[0], rma_off=True)
            ost.advance(0, rma_off=True)
            got = gouts[step][gseq]
            assert H.tol_ok(got, ref), (gseq, step, H.max_err(got, ref))


def test_rma_off_prefill_matches_oracle_and_decode(sab):
    seed, L, t0 = 62, 1, 4096
    gw, gdict = H.gpu_weights(seed, 0)
    ow, wdict = H.oracle_weights(seed, 0)
    st = sab.State(2, L)
    H.seed_gpu_state(st, L, t0, [60, 60], seed, [gdict])
    ost = oracle.OracleState(1, L)
    H.seed_oracle_state(ost, [0], L, t0, [60], seed, [wdict])
    for n in oracle.OracleState.ARRAYS:
        getattr(st, n)[1].copy_(getattr(st, n)[0])
    before = {n: getattr(st, n).clone() for n in RMA_ARRAYS}
    T = 100
    x = wl.make_x(seed, 0, 0, range(T), big_every=4096, first_pos=t0)
    got = sab.swa_rma_prefill_chunk(st, gw, 0, 0, x.cuda(), rma_off=True).cpu()
    sab.advance(st, [0], T, rma_off=True)
    dec = []
    for i in range(T):
        dec.append(sab.swa_rma_decode(st, gw, 0, [1], x[i:i + 1].cuda(), rma_off=True))
        sab.advance(st, [1], rma_off=True)
    dec = torch.cat(dec).cpu()
    ref = ost.prefill_chunk(ow, 0, 0, x, rma_off=True)
    assert sab.last_device_error(st) == 0
    assert H.tol_ok(got, ref), H.max_err(got, ref)
    assert H.tol_ok(got, dec), H.max_err(got, dec)
    for n in RMA_ARRAYS:
        assert torch.equal(getattr(st, n), before[n]), n
    assert st.meta[0].tolist() == [t0 + T, 60, 1024, 0]


def test_two_caller_streams_run_layer_calls_side_by_side(sab):
    """Two host threads, each with its own stream, state and workspace, run decode
    steps (with commits) at the same time: each gets the bits of the same steps run
    alone.  The library gives each caller stream its own side stream and events,
    so neither caller's calls wait on the other's."""
    import threading
    seed, B, steps, t0 = 88, 8, 6, 4096
    gw, gdict = H.gpu_weights(seed, 0)
    fills = [250, 251, 252, 253, 254, 255, 3, 100]  # commits inside the six steps
    states = []
    for k in range(2):
        st = sab.State(B, 1)
        H.seed_gpu_state(st, 1, t0, fills, seed + k, [gdict])
        states.append(st)
    snaps = [st.blob.clone() for st in states]
    xs = [[wl.make_x(seed + k, 0, s, range(B), device="cuda") for s in range(steps)]
          for k in range(2)]
    ids = torch.arange(B, dtype=torch.int32, device="cuda")

    def run(k, stream, outs, start=None):
        if start is not None:
            start.wait()
        ws = torch.empty(sab.decode_workspace_bytes(B), dtype=torch.uint8, device="cuda")
        with torch.cuda.stream(stream):
            for s in range(steps):
                outs.append(sab.swa_rma_decode(states[k], gw, 0, ids, xs[k][s], ws=ws,
                                               stream=stream))
                sab.advance(states[k], ids, stream=stream)
        stream.synchronize()

    alone = [[], []]
    for k in range(2):
        run(k, torch.cuda.current_stream(), alone[k])
    ref_blobs = [st.blob.clone() for st in states]
    for k in range(2):
        states[k].blob.copy_(snaps[k])
    torch.cuda.synchronize()
    together = [[], []]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    start = threading.Event()
    threads = [threading.Thread(target=run, args=(k, streams[k], together[k], start))
               for k in range(2)]
    for t in threads:
        t.start()
    start.set()
    for t in threads:
        t.join()
    torch.cuda.synchronize()
    for k in range(2):
        assert sab.last_device_error(states[k]) == 0
        for s in range(steps):
            assert torch.equal(together[k][s], alone[k][s]), (k, s)
        assert torch.equal(states[k].blob, ref_blobs[k]), k
