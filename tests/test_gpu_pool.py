"""The pooled anchor layout (ER_STATE_POOL): a commit that moves no K/V row.

Bank and pending block of a group share one pool of 1280 slots; a record is
written once (at its append) and never moved; a commit ranks the occupied
slots exactly as in the plain layout, frees the evicted records' slots and
lists the next block's slots.  The method is the same, so the oracle (plain
layout) is the reference:
  - the records kept after every commit are those the oracle keeps: the same
    positions and scores per (sequence, layer, group), bit for bit for an
    explicit commit fed the same keys, and up to near-ties at the boundary
    after decode steps (where scores come from the tensor-core scorer);
  - layer outputs within |Δ| <= 1e-2 + 1e-2·|oracle|;
  - a commit leaves every K/V row of the pool untouched (nothing moves) and a
    valid slot list: 256 distinct free slots, ascending.
"""
import pytest
import torch

import oracle
from synth import workloads as wl
from tests import helpers as H

pytestmark = pytest.mark.gpu

FREE = 0x7FFFFFFF


@pytest.fixture(scope="module")
def sab():
    from sliding_window_anchor_b200 import build
    build.build()
    import sliding_window_anchor_b200 as m
    return m


def pooled_copy(sab, plain):
    st = sab.State(plain.s_max, plain.n_layers, pool=True)
    st.pool_from_plain(plain)
    return st


def kept_records(st, row, layer, group):
    """(position, score bits) of the occupied pool slots, sorted by position."""
    pos = st.bank_pos[row, layer, group].cpu()
    sc = st.bank_score[row, layer, group].cpu()
    occ = pos != FREE
    p, s = pos[occ], sc[occ].view(torch.int32)
    order = torch.argsort(p)
    return p[order], s[order]


def oracle_records(ost, row, layer, group):
    c = int(ost.meta[row, 2])
    p = ost.bank_pos[row, layer, group, :c]
    s = ost.bank_score[row, layer, group, :c].view(torch.int32)
    order = torch.argsort(p)
    return p[order], s[order]


def check_slot_list(st, row, n_layers):
    for l in range(n_layers):
        for g in range(4):
            sl = st.pend_pos[row, l, g].cpu()
            pos = st.bank_pos[row, l, g].cpu()
            p = int(st.meta[row, 1])
            assert bool((sl[1:] > sl[:-1]).all()), "slot list ascending, distinct"
            # slots not yet used by the block are free
            assert bool((pos[sl[p:].long()] == FREE).all())


def test_pool_explicit_commit_matches_oracle_and_moves_nothing(sab):
    """The commit workload (bank and pending full, ~5% exact score ties) in the pooled
    layout: the kept records equal the oracle's bit for bit, no K/V row changes."""
    seed, n, L, t0 = wl.seed_of(wl.COMMIT), 16, 2, 32768
    plain = sab.State(n, L)
    wl.seed_commit_workload(plain.arrays(), range(n), L, t0, seed, 0, "cuda")
    st = pooled_copy(sab, plain)
    k_before, v_before = st.bank_k.clone(), st.bank_v.clone()
    kept = sab.rma_commit(st, -1, list(range(n)), want_kept=True)
    assert sab.last_device_error(st) == 0
    assert torch.equal(st.bank_k, k_before) and torch.equal(st.bank_v, v_before)
    for seq in (0, 5, 15):
        ost = oracle.OracleState(1, L)
        wl.seed_commit_workload({k: getattr(ost, k) for k in oracle.OracleState.ARRAYS}, [seq],
                                L, t0, seed, 0, "cpu")
        ost.commit(-1, 0)
        assert torch.equal(st.meta[seq].cpu(), ost.meta[0])
        for l in range(L):
            for g in range(4):
                gp, gs = kept_records(st, seq, l, g)
                op, os_ = oracle_records(ost, 0, l, g)
                assert torch.equal(gp, op) and torch.equal(gs, os_), (seq, l, g)
                # the ranked list names pool slots, best first
                slots = kept[seq, l, g].cpu()
                assert int((slots >= 0).sum()) == 1024
                ranked = st.bank_pos[seq, l, g].cpu()[slots.long()]
                assert bool((ranked != FREE).all())
        check_slot_list(st, seq, L)
    # a second commit in the same state: the next block goes to the listed slots
    del st, plain
    torch.cuda.empty_cache()


def test_pool_decode_steps_match_oracle(sab):
    """Decode steps through commits (B=8, one layer, staggered fills) in the pooled
    layout against the oracle; outputs within tolerance, kept records equal."""
    seed, B, t0, steps = 91, 8, 4096, 8
    gw, gdict = H.gpu_weights(seed, 0)
    ow, wdict = H.oracle_weights(seed, 0)
    fills = [250, 251, 252, 253, 254, 255, 3, 100]
    plain = sab.State(B, 1)
    H.seed_gpu_state(plain, 1, t0, fills, seed, [gdict])
    st = pooled_copy(sab, plain)
    ids = torch.arange(B, dtype=torch.int32, device="cuda")
    outs = []
    for step in range(steps):
        x = wl.make_x(seed, 0, step, range(B), device="cuda")
        outs.append(sab.swa_rma_decode(st, gw, 0, ids, x).cpu())
        sab.advance(st, ids)
    assert sab.last_device_error(st) == 0
    for b in range(B):
        ost = oracle.OracleState(1, 1)
        H.seed_oracle_state(ost, [b], 1, t0, [fills[b]], seed, [wdict])
        for step in range(steps):
            ref = ost.decode_layer(ow, 0, 0, wl.make_x(seed, 0, step, [b])[0])
            ost.advance(0)
            assert H.tol_ok(outs[step][b], ref), (b, step, H.max_err(outs[step][b], ref))
        assert torch.equal(st.meta[b].cpu(), ost.meta[0])
        H.kept_sets_agree(plain_view(st, b), {n: getattr(ost, n)[0]
                                              for n in oracle.OracleState.ARRAYS}, 1)
        check_slot_list(st, b, 1)


def plain_view(st, row):
    """A pooled row as the plain layout would hold it: the bank is the occupied
    slots whose records came before the current block (position below pos - pend),
    in position order."""
    meta = st.meta[row].cpu()
    t, p, c = int(meta[0]), int(meta[1]), int(meta[2])
    bp = torch.zeros(st.n_layers, 4, 1024, dtype=torch.int32)
    bs = torch.zeros(st.n_layers, 4, 1024, dtype=torch.float32)
    for l in range(st.n_layers):
        for g in range(4):
            pos = st.bank_pos[row, l, g].cpu()
            sc = st.bank_score[row, l, g].cpu()
            sel = (pos != FREE) & (pos < t - p)
            order = torch.argsort(pos[sel])
            assert int(sel.sum()) == c, (l, g, int(sel.sum()), c)
            bp[l, g, :c] = pos[sel][order]
            bs[l, g, :c] = sc[sel][order]
    return {"meta": meta, "bank_pos": bp, "bank_score": bs}


def test_pool_stream_start_prefill_and_decode_match_oracle(sab):
    """From an empty pooled state: two prefill chunks (256, then a ragged 77, so the
    first commit keeps every record), then decode steps, against the oracle."""
    seed = wl.seed_of(wl.PREFILL)
    gw, gdict = H.gpu_weights(seed, 0)
    ow, wdict = H.oracle_weights(seed, 0)
    st = sab.State(1, 1, pool=True)
    sab.state_init(st, [0])
    ost = oracle.OracleState(1, 1)
    pos = 0
    for ci, T in enumerate((256, 77)):
        x = wl.make_x(seed, 0, 2000 + ci, range(T), big_every=4096, first_pos=pos)
        got = sab.swa_rma_prefill_chunk(st, gw, 0, 0, x.cuda()).cpu()
        sab.advance(st, [0], T)
        ref = ost.prefill_chunk(ow, 0, 0, x)
        ost.advance(0, T)
        assert H.tol_ok(got, ref), (ci, H.max_err(got, ref))
        pos += T
    for step in range(4):
        x = wl.make_x(seed, 0, 3000 + step, [0])
        got = sab.swa_rma_decode(st, gw, 0, [0], x.cuda()).cpu()[0]
        sab.advance(st, [0])
        ref = ost.decode_layer(ow, 0, 0, x[0])
        ost.advance(0)
        assert H.tol_ok(got, ref), (step, H.max_err(got, ref))
    assert sab.last_device_error(st) == 0
    assert torch.equal(st.meta[0].cpu(), ost.meta[0])
    for g in range(4):
        gp, _ = kept_records(st, 0, 0, g)
        c, p = int(ost.meta[0, 2]), int(ost.meta[0, 1])
        op = torch.sort(torch.cat([ost.bank_pos[0, 0, g, :c], ost.pend_pos[0, 0, g, :p]])).values
        assert torch.equal(gp, op), g
    check_slot_list(st, 0, 1)
