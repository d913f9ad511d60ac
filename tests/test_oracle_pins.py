"""Pins of the CPU oracle to facts outside itself (CPU only).

Each test checks the oracle against something the pages or mathematics fix:
printed numbers (tests/golden/budget.json), closed forms, invariants, special
cases with a textbook answer, or brute force on tiny inputs.  They are chosen
so a plausible slip (a dropped term, a wrong sign or index, a transposed
operand, the wrong RoPE pairing, an off-by-one window) fails at least one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
D = 256


def bf16(x):
    """Inputs: any doubles, rounded through float32 to BF16."""
    return torch.as_tensor(x, dtype=torch.float64).to(torch.float32).to(torch.bfloat16)


def bf16_exact(x):
    """Expected values: one round-to-nearest-even from float64 to BF16 (numpy frexp/rint)."""
    a = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(a)
    y = np.ldexp(np.rint(m * 256.0), e - 8)  # 8 significant bits, ties to even
    return torch.from_numpy(y.astype(np.float32)).to(torch.bfloat16)


def ones_gain():
    return torch.ones(D, dtype=torch.bfloat16)


# ------------------------------------------------------------- byte budget

def test_byte_budget_matches_pages():
    g = json.load(open(os.path.join(GOLDEN, "budget.json")))
    assert math.prod(g["factors_committed"]) == g["committed_bytes"] == 32 * 2**20
    st = oracle.OracleState(1, 8)
    committed = st.bank_k.numel() * 2 + st.bank_v.numel() * 2
    pending = st.pend_k.numel() * 2 + st.pend_v.numel() * 2
    window = st.win_k.numel() * 2 + st.win_v.numel() * 2
    assert committed == g["committed_bytes"]
    assert pending == g["pending_bytes"]
    assert window == g["window_bytes"]
    assert committed + pending + window == g["total_bytes"] == oracle.kv_bytes_per_seq(8)
    # the 31.97 / 71.97 MiB figures: 1023 persistent window rows (current token excluded)
    per_pos = window // 1024
    assert round(1023 * per_pos / 2**20, 2) == g["window_persistent_mib_2dp"]
    assert round((1023 * per_pos + committed + pending) / 2**20, 2) == g["total_persistent_mib_2dp"]
    # source model: 8 attention layers x 4 KV heads x 256 dims x (K,V) x 2 B
    src = 8 * 4 * 256 * 2 * 2
    assert src == g["source_model_bytes_per_token"]
    assert src * 65536 == g["source_model_bytes_64k"]
    assert src * 262144 == g["source_model_bytes_256k"]
    assert round(100 * (1 - g["total_bytes"] / g["source_model_bytes_256k"]), 1) == \
        g["reduction_pct_1dp"]
    # independent of stream length: the state has no length-dependent array
    assert oracle.OracleState(3, 8).win_k.numel() == 3 * st.win_k.numel()


# ------------------------------------------------------------ BF16 rounding

def test_bf16_rounding_matches_torch_and_ties_to_even():
    rng = np.random.default_rng(1)
    vals = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.integers(-6, 6, 2000),
                           [1.0, -2.5, 3.0e38, 1e-30]])
    for v in vals:
        v32 = float(np.float32(v))
        want = torch.tensor([v32], dtype=torch.float32).to(torch.bfloat16).view(torch.int16)
        assert oracle.f64_to_bf16_bits(v32) == int(want) & 0xFFFF, v
    # exact ties round to even; just above a tie rounds up
    assert oracle.f64_to_bf16_bits(1.0 + 2.0**-8) == 0x3F80
    assert oracle.f64_to_bf16_bits(1.0 + 3 * 2.0**-8) == 0x3F82
    assert oracle.f64_to_bf16_bits(1.0 + 2.0**-8 + 2.0**-40) == 0x3F81
    assert oracle.f64_to_bf16_bits(-0.0) == 0x8000


# --------------------------------------------------------- RMS-norm + RoPE

def test_rmsnorm_constant_vector_closed_form():
    # constant c: y_i = sign(c) g_i / sqrt(1 + eps/c^2); position 0 rotates nothing
    gain = bf16(np.linspace(0.5, 1.5, D))
    for c in (0.25, -3.0, 1e-2):
        x = bf16(np.full(D, c))
        y = oracle.norm_rope(x, gain, 0).double()
        cc = float(x[0].double())
        want = math.copysign(1.0, cc) * gain.double() / math.sqrt(1 + 1e-6 / cc**2)
        assert torch.equal(y, bf16_exact(want.numpy()).double())


def test_rmsnorm_unit_rms_and_scale_invariance():
    x = synth.normal((8, D), 7, synth.MISC, torch.bfloat16)
    y = oracle.norm_rope(x, ones_gain(), 0).double()
    rms = y.pow(2).mean(dim=1).sqrt()
    assert torch.all((rms - 1).abs() < 4e-3)
    for a in (2.0, 0.5, 8.0):  # exact scalings in BF16
        y2 = oracle.norm_rope((x.double() * a).to(torch.bfloat16), ones_gain(), 0).double()
        assert (y2 - y).abs().max() <= 2.0**-7 * y.abs().max()


def _unit_row(i, scale=1.0):
    x = torch.zeros(D, dtype=torch.float64)
    x[i] = scale
    return bf16(x.numpy())


def test_rope_pairing_frequency_and_direction():
    # e_i with i < 32 turns into the (i, i+32) plane: (cos a, sin a); e_{i+32} into (-sin a, cos a)
    # with a = pos * 1e7^(-2i/64); after the norm e_i has value 16/sqrt(1+256e-6).
    mag = 16 / math.sqrt(1 + 256e-6)
    for i in (0, 1, 17, 31):
        f = 1e7 ** (-2.0 * i / 64)
        for pos in (1, 7, 1000, 262143):
            a = pos * f
            y = oracle.norm_rope(_unit_row(i), ones_gain(), pos).double()
            assert abs(y[i] - mag * math.cos(a)) <= 2.0**-8 * mag
            assert abs(y[i + 32] - mag * math.sin(a)) <= 2.0**-8 * mag
            others = torch.ones(D, dtype=torch.bool)
            others[[i, i + 32]] = False
            assert torch.all(y[others] == 0)
            y2 = oracle.norm_rope(_unit_row(i + 32), ones_gain(), pos).double()
            assert abs(y2[i] + mag * math.sin(a)) <= 2.0**-8 * mag
            assert abs(y2[i + 32] - mag * math.cos(a)) <= 2.0**-8 * mag


def test_rope_leaves_dims_64_up_and_pair_norms():
    x = synth.normal((4, D), 11, synth.MISC, torch.bfloat16)
    g = synth.normal((D,), 11, synth.MISC + 1, torch.bfloat16, scale=0.1, offset=1.0)
    y0 = oracle.norm_rope(x, g, 0).double()
    for pos in (3, 4097, 131071):
        y = oracle.norm_rope(x, g, pos).double()
        assert torch.equal(y[:, 64:], y0[:, 64:])
        n0 = y0[:, :32] ** 2 + y0[:, 32:64] ** 2
        n1 = y[:, :32] ** 2 + y[:, 32:64] ** 2
        assert torch.all((n1 - n0).abs() <= 2.0**-6 * (n0 + 1e-3))


def test_rope_relative_position_property():
    # <R_a q, R_b k> depends on a - b only (a wrong sign makes it a reflection and fails)
    q = synth.normal((1, D), 5, synth.MISC, torch.bfloat16)
    k = synth.normal((1, D), 5, synth.MISC + 1, torch.bfloat16)
    dots = []
    for a, b in ((5, 2), (1027, 1024), (100003, 100000), (262143, 262140)):
        qa = oracle.norm_rope(q, ones_gain(), a).double()
        kb = oracle.norm_rope(k, ones_gain(), b).double()
        dots.append(float((qa * kb).sum()))
    ref = dots[0]
    assert all(abs(d - ref) < 0.1 for d in dots), dots
    # and it does depend on the offset
    qa = oracle.norm_rope(q, ones_gain(), 9).double()
    kb = oracle.norm_rope(k, ones_gain(), 2).double()
    assert abs(float((qa * kb).sum()) - ref) > 0.1


# ------------------------------------------------------------------- linear

def test_linear_against_float64_matmul_and_identity():
    W = synth.normal((96, 80), 3, synth.MISC, torch.bfloat16)
    x = synth.normal((80,), 3, synth.MISC + 1, torch.bfloat16)
    y = oracle.linear_bf16(W, x)
    ref = (W.double() @ x.double())
    assert torch.equal(y, bf16_exact(ref.numpy()))
    I = torch.eye(80, dtype=torch.bfloat16)
    assert torch.equal(oracle.linear_bf16(I, x), x)


# -------------------------------------------------------------------- score

def silu(h):
    return h / (1 + math.exp(-h))


def test_score_closed_forms():
    x = synth.normal((3, 2560), 2, synth.MISC, torch.bfloat16)
    xd = x.double()
    # W1 selects x_j (j < 256), W2 row g sums them: s_g = sum_j silu(x_j)
    w1 = torch.zeros(256, 2560, dtype=torch.float32)
    w1[torch.arange(256), torch.arange(256)] = 1
    w2 = torch.ones(4, 256, dtype=torch.float32)
    s = oracle.score(w1, w2, x)
    for t in range(3):
        want = sum(silu(float(xd[t, j])) for j in range(256))
        assert torch.all(s[t] == np.float32(want))
    # a single path W1[3,7]=1, W2[2,3]=1: only group 2 sees silu(x_7) (catches transposes)
    w1 = torch.zeros(256, 2560, dtype=torch.float32)
    w1[3, 7] = 1
    w2 = torch.zeros(4, 256, dtype=torch.float32)
    w2[2, 3] = 1
    s = oracle.score(w1, w2, x)
    for t in range(3):
        assert s[t, 2] == np.float32(silu(float(xd[t, 7])))
        assert s[t, 0] == 0 and s[t, 1] == 0 and s[t, 3] == 0
    # SiLU limits: zero in -> zero out; large h -> h
    assert torch.all(oracle.score(torch.zeros(256, 2560), torch.ones(4, 256), x) == 0)
    w1 = torch.zeros(256, 2560, dtype=torch.float32)
    w1[0, 0] = 64.0
    xs = torch.zeros(1, 2560, dtype=torch.bfloat16)
    xs[0, 0] = 1.0
    w2 = torch.zeros(4, 256, dtype=torch.float32)
    w2[:, 0] = 1
    assert abs(float(oracle.score(w1, w2, xs)[0, 0]) - 64.0) < 1e-12 * 64 + 2e-6


def test_score_against_float64_library_path():
    w = wl.make_weights(99, 0)
    x = synth.normal((5, 2560), 99, synth.MISC, torch.bfloat16)
    s = oracle.score(w["w1"], w["w2"], x).double()
    h = x.double() @ w["w1"].double().T
    ref = torch.nn.functional.silu(h) @ w["w2"].double().T
    assert torch.allclose(s, ref, rtol=2e-7, atol=1e-9)


# ---------------------------------------------------------------- attention

def test_attend_special_cases():
    q = synth.normal((D,), 4, synth.MISC, torch.bfloat16)
    v = synth.normal((5, D), 4, synth.MISC + 1, torch.bfloat16)
    k = synth.normal((5, D), 4, synth.MISC + 2, torch.bfloat16)
    # one key: o = v
    assert torch.equal(oracle.attend_rows(q, k[:1], v[:1]), v[0].double())
    # identical keys: the mean of the values
    kk = k[:1].repeat(5, 1)
    assert torch.allclose(oracle.attend_rows(q, kk, v), v.double().mean(0), atol=1e-14)
    # empty list: zero
    assert torch.equal(oracle.attend_rows(q, k[:0], v[:0]), torch.zeros(D, dtype=torch.float64))
    # permutation invariance
    perm = [3, 0, 4, 1, 2]
    assert torch.allclose(oracle.attend_rows(q, k[perm], v[perm]), oracle.attend_rows(q, k, v),
                          atol=1e-14)


def test_attend_scale_is_one_over_sixteen():
    # q = 16 e0, k1 = e0 (logit 1), k2 = 0 (logit 0): weights e/(e+1), 1/(e+1)
    q = _unit_row(0, 16.0)
    k = torch.stack([_unit_row(0, 1.0), torch.zeros(D, dtype=torch.bfloat16)])
    v = torch.stack([_unit_row(1, 1.0), _unit_row(2, 1.0)])
    o = oracle.attend_rows(q, k, v)
    e = math.e
    assert abs(o[1] - e / (e + 1)) < 1e-15 and abs(o[2] - 1 / (e + 1)) < 1e-15
    # one-hot limit: a key aligned with a large q takes all the weight
    q = _unit_row(0, 256.0)
    k = torch.stack([_unit_row(0, 8.0), _unit_row(5, 8.0)])
    o = oracle.attend_rows(q, k, v)
    assert abs(o[1] - 1) < 1e-50 + math.exp(-120) and o[2] < 1e-50


# -------------------------------------------------------------------- commit

def _order_key(score, pos):
    # (score desc, pos asc); NaN ranks below every number; -0 == +0
    s = float(score)
    return (1 if math.isnan(s) else 0, 0.0 if math.isnan(s) else -s, int(pos))


def _brute_commit(bank_s, bank_p, c, pend_s, pend_p, p):
    recs = [(bank_s[i], bank_p[i], i) for i in range(c)] + \
           [(pend_s[j], pend_p[j], 1024 + j) for j in range(p)]
    keys = [_order_key(s, q) for s, q, _ in recs]
    n = len(recs)
    rank = [sum(1 for j in range(n) if keys[j] < keys[i]) for i in range(n)]  # O(n^2)
    K = min(1024, n)
    kept = sorted([i for i in range(n) if rank[i] < K], key=lambda i: rank[i])
    return [recs[i][2] for i in kept]


def _commit_case(seed, c, p, tweak=None):
    st = oracle.OracleState(1, 1)
    gen = np.random.default_rng(seed)
    for g in range(4):
        st.bank_score[0, 0, g] = torch.from_numpy(gen.standard_normal(1024).astype(np.float32))
        st.pend_score[0, 0, g] = torch.from_numpy(gen.standard_normal(256).astype(np.float32))
        st.bank_pos[0, 0, g] = torch.from_numpy(gen.permutation(30000)[:1024].astype(np.int32))
        st.pend_pos[0, 0, g] = torch.arange(40000, 40256, dtype=torch.int32)
    synth.fill_normal_(st.bank_k, seed, 1)
    synth.fill_normal_(st.bank_v, seed, 2)
    synth.fill_normal_(st.pend_k, seed, 3)
    synth.fill_normal_(st.pend_v, seed, 4)
    if tweak:
        tweak(st)
    st.meta[0] = torch.tensor([40256, p, c, 0])
    before = st.clone()
    kept = st.commit(-1, 0, want_kept=True)[0]
    return before, st, kept


def _check_commit(before, st, kept, c, p):
    for g in range(4):
        want = _brute_commit(before.bank_score[0, 0, g].tolist(), before.bank_pos[0, 0, g].tolist(),
                             c, before.pend_score[0, 0, g].tolist(),
                             before.pend_pos[0, 0, g].tolist(), p)
        K = len(want)
        assert kept[g, :K].tolist() == want
        assert torch.all(kept[g, K:] == -1)
        # slot placement: survivors stay; evicted slots ascending then c.. take winners ascending
        keep_bank = sorted(i for i in want if i < 1024)
        winners = sorted(j - 1024 for j in want if j >= 1024)
        targets = [i for i in range(c) if i not in set(keep_bank)] + list(range(c, 1024))
        for i in keep_bank:
            assert torch.equal(st.bank_k[0, 0, g, i], before.bank_k[0, 0, g, i])
            assert st.bank_pos[0, 0, g, i] == before.bank_pos[0, 0, g, i]
        for t, j in zip(targets, winners):
            assert torch.equal(st.bank_k[0, 0, g, t], before.pend_k[0, 0, g, j])
            assert torch.equal(st.bank_v[0, 0, g, t], before.pend_v[0, 0, g, j])
            assert st.bank_score[0, 0, g, t] == before.pend_score[0, 0, g, j]
            assert st.bank_pos[0, 0, g, t] == before.pend_pos[0, 0, g, j]
    assert int(st.meta[0, 1]) == 0 and int(st.meta[0, 2]) == min(1024, c + p)


@pytest.mark.parametrize("c,p", [(1024, 256), (1024, 37), (700, 256), (100, 256), (0, 256),
                                 (1024, 0)])
def test_commit_matches_brute_force_rank(c, p):
    before, st, kept = _commit_case(10 + c + p, c, p)
    _check_commit(before, st, kept, c, p)


def test_commit_ties_signed_zero_nan_and_groups():
    def tweak(st):
        bs, ps = st.bank_score[0, 0], st.pend_score[0, 0]
        bs[0, :] = torch.from_numpy(np.linspace(5, 1, 1024).astype(np.float32))
        ps[0, :] = bs[0, 500]  # ties with one anchor and among themselves: positions decide
        bs[1, 5] = -0.0
        ps[1, 9] = 0.0
        bs[1, 6] = float("nan")
        ps[1, 10] = float("-inf")
        bs[2, :] = -1.0
        ps[2, :] = -1.0  # all tied: positions alone decide
        # the same source position wins in every group
        for g in range(4):
            st.pend_pos[0, 0, g, 3] = 123
            ps[g, 3] = 100.0
    before, st, kept = _commit_case(77, 1024, 256, tweak)
    _check_commit(before, st, kept, 1024, 256)
    assert all(1024 + 3 in kept[g].tolist() for g in range(4))
    # NaN ranked last of group 1, below -inf
    k1 = kept[1].tolist()
    assert 6 not in k1


def test_commit_keeps_anchor_contents_when_pending_loses():
    # immutability: with every pending score below the bank minimum the bank is unchanged
    def tweak(st):
        st.pend_score[0, 0] = st.bank_score[0, 0].min() - 1 - torch.rand(4, 256)
    before, st, kept = _commit_case(5, 1024, 256, tweak)
    for n in ("bank_k", "bank_v", "bank_score", "bank_pos"):
        assert torch.equal(getattr(st, n), getattr(before, n))


def test_commits_compose_to_one_top_k_over_the_stream():
    """Commits after every block of 256 keep, in the end, exactly the top 1024 of
    all records ever appended (for a total order, top-k(top-k(A) | B) =
    top-k(A | B)), and every kept slot still holds its own record's rows."""
    gen = np.random.default_rng(3)
    st = oracle.OracleState(1, 1)
    st.meta[0] = torch.tensor([0, 0, 0, 0])
    allrec = [[] for _ in range(4)]
    pos0 = 5000
    for blk in range(12):
        for g in range(4):
            sc = gen.standard_normal(256).astype(np.float32)
            if blk > 0:  # exact ties with earlier records and inside the block
                prev = np.array([r[0] for r in allrec[g]], dtype=np.float32)
                idx = gen.integers(0, 256, 13)
                sc[idx] = prev[gen.integers(0, len(prev), 13)]
            sc[gen.integers(0, 256, 3)] = sc[0]
            sc[7] = -0.0 if blk % 2 else 0.0
            sc[11] = np.float32("nan") if blk % 3 == 0 else np.float32("-inf")
            pos = pos0 + blk * 256 + np.arange(256, dtype=np.int32)
            st.pend_score[0, 0, g] = torch.from_numpy(sc)
            st.pend_pos[0, 0, g] = torch.from_numpy(pos)
            # each record's K and V rows carry its position (exact in BF16 below 256)
            tag = torch.from_numpy(((pos % 199) + g).astype(np.float32)).to(torch.bfloat16)
            st.pend_k[0, 0, g] = tag[:, None].expand(256, 256)
            st.pend_v[0, 0, g] = -tag[:, None].expand(256, 256)
            allrec[g] += list(zip(sc.tolist(), pos.tolist()))
        st.meta[0, 1] = 256
        st.commit(-1, 0)
        assert int(st.meta[0, 1]) == 0 and int(st.meta[0, 2]) == min(1024, 256 * (blk + 1))
    for g in range(4):
        want = sorted(allrec[g], key=lambda r: _order_key(r[0], r[1]))[:1024]
        got = st.bank_pos[0, 0, g].tolist()
        assert sorted(got) == sorted(q for _, q in want), g
        tags = st.bank_k[0, 0, g, :, 0].float()
        assert torch.equal(tags, torch.tensor([(q % 199) + g for q in got], dtype=torch.float32))
        assert torch.equal(st.bank_v[0, 0, g, :, 5].float(), -tags)
        by_pos = {q: sc for sc, q in allrec[g]}
        for i, q in enumerate(got):
            a, b = float(st.bank_score[0, 0, g, i]), by_pos[q]
            assert a == b or (math.isnan(a) and math.isnan(b))


# -------------------------------------------------------------- decode path

def _weights(seed, layer=0):
    w = wl.make_weights(seed, layer)
    return oracle.OracleWeights(w["w_qkv"], w["w_o"], w["q_norm_swa"], w["k_norm_swa"],
                                w["q_norm_rma"], w["k_norm_rma"], w["w1"], w["w2"]), w


def test_first_token_closed_form():
    # empty state at t=0: each read sees only the token itself, so o_swa = v_swa, o_rma = v_rma
    ow, w = _weights(123)
    st = oracle.OracleState(1, 1)
    x = synth.normal((2560,), 123, synth.MISC, torch.bfloat16)
    out, o_swa, o_rma = st.decode_layer(ow, 0, 0, x, want_branches=True)
    proj = oracle.linear_bf16(w["w_qkv"], x).double()
    v_swa = proj[5120:6144].view(4, 256)
    v_rma = proj[11264:12288].view(4, 256)
    for h in range(16):
        assert torch.equal(o_swa[h], v_swa[h // 4])
        assert torch.equal(o_rma[h], v_rma[h // 4])
    o = bf16_exact((v_swa.repeat_interleave(4, 0) + v_rma.repeat_interleave(4, 0)).reshape(-1).numpy())
    assert torch.equal(out, oracle.linear_bf16(w["w_o"], o))
    # the step wrote window slot 0 and pending slot 0 with the token's k/v and score
    assert torch.equal(st.win_v[0, 0, :, 0].double(), v_swa)
    assert torch.equal(st.pend_v[0, 0, :, 0].double(), v_rma)
    assert torch.equal(st.pend_score[0, 0, :, 0], oracle.score(w["w1"], w["w2"], x)[0])
    assert torch.all(st.pend_pos[0, 0, :, 0] == 0)


def _seeded(seed, t0, fill_mode="zero", n_layers=1):
    ow, w = _weights(seed)
    st = oracle.OracleState(1, n_layers)
    arrays = {n: getattr(st, n) for n in oracle.OracleState.ARRAYS}
    wl.seed_state(arrays, [0], n_layers, t0, fill_mode, seed, [w], oracle.norm_rope)
    return ow, w, st


def test_decode_reads_exactly_the_window_and_anchor_rows():
    # the two branch outputs equal attention over rows gathered here by position
    ow, w, st = _seeded(31, 4096, "uniform")
    p = int(st.meta[0, 1])
    x = synth.normal((2560,), 31, synth.MISC, torch.bfloat16)
    t = 4096
    _, o_swa, o_rma = st.decode_layer(ow, 0, 0, x, want_branches=True)
    proj = oracle.linear_bf16(w["w_qkv"], x)
    q_swa = oracle.norm_rope(proj[:4096].view(16, 256), w["q_norm_swa"], t)
    q_rma = oracle.norm_rope(proj[6144:10240].view(16, 256), w["q_norm_rma"], t)
    for h in (0, 5, 15):
        g = h // 4
        slots = [pos % 1024 for pos in range(t - 1023, t + 1)]
        ref = oracle.attend_rows(q_swa[h], st.win_k[0, 0, g, slots], st.win_v[0, 0, g, slots])
        assert torch.equal(o_swa[h], ref)
        kr = torch.cat([st.bank_k[0, 0, g], st.pend_k[0, 0, g, :p + 1]])
        vr = torch.cat([st.bank_v[0, 0, g], st.pend_v[0, 0, g, :p + 1]])
        assert torch.equal(o_rma[h], oracle.attend_rows(q_rma[h], kr, vr))
    # early in a stream only positions 0..t are attended
    ow2, w2 = _weights(32)
    st2 = oracle.OracleState(1, 1)
    xs = [synth.normal((2560,), 32, synth.MISC + i, torch.bfloat16) for i in range(3)]
    for i in range(3):
        _, o_swa2, _ = st2.decode_layer(ow2, 0, 0, xs[i], want_branches=True)
        st2.advance(0)
    proj = oracle.linear_bf16(w2["w_qkv"], xs[2])
    q = oracle.norm_rope(proj[:4096].view(16, 256), w2["q_norm_swa"], 2)
    ref = oracle.attend_rows(q[0], st2.win_k[0, 0, 0, :3], st2.win_v[0, 0, 0, :3])
    assert torch.equal(o_swa2[0], ref)


def test_prefill_equals_token_by_token_decode():
    # the aligned-chunk reading: a chunk of T tokens = T decode steps, bit for bit
    ow, w, st_a = _seeded(41, 4096, "zero")
    st_b = st_a.clone()
    T = 256
    xs = wl.make_x(41, 0, 0, range(T))
    out_chunk = st_a.prefill_chunk(ow, 0, 0, xs)
    st_a.advance(0, T)
    outs = []
    for i in range(T):
        outs.append(st_b.decode_layer(ow, 0, 0, xs[i]))
        st_b.advance(0)
    assert torch.equal(out_chunk, torch.stack(outs))
    for n in oracle.OracleState.ARRAYS:
        assert torch.equal(getattr(st_a, n), getattr(st_b, n)), n
    # and a ragged chunk that does not fill the block
    T = 17
    xs = wl.make_x(41, 0, 1, range(T))
    out_chunk = st_a.prefill_chunk(ow, 0, 0, xs)
    st_a.advance(0, T)
    outs = []
    for i in range(T):
        outs.append(st_b.decode_layer(ow, 0, 0, xs[i]))
        st_b.advance(0)
    assert torch.equal(out_chunk, torch.stack(outs))
    for n in oracle.OracleState.ARRAYS:
        assert torch.equal(getattr(st_a, n), getattr(st_b, n)), n


# ------------------------------------------------- RMA off (the pages' ablation)

RMA_ARRAYS = ("bank_k", "bank_v", "pend_k", "pend_v", "bank_score", "pend_score", "bank_pos",
              "pend_pos")


def test_rma_off_equals_rma_on_when_every_anchor_value_is_zero():
    # a special case that needs no flag: with zero v_rma weights and zero bank / pending
    # V rows, every RMA read averages zeros, so o_rma = 0 exactly and both settings agree
    _, w, st_on = _seeded(51, 3000, [100])
    wz = dict(w)
    wz["w_qkv"] = w["w_qkv"].clone()
    wz["w_qkv"][11264:12288] = 0
    ow = oracle.OracleWeights(wz["w_qkv"], wz["w_o"], wz["q_norm_swa"], wz["k_norm_swa"],
                              wz["q_norm_rma"], wz["k_norm_rma"], wz["w1"], wz["w2"])
    st_on.bank_v.zero_()
    st_on.pend_v.zero_()
    st_off = st_on.clone()
    for step in range(3):
        x = wl.make_x(51, 0, step, [0])[0]
        out_on, _, o_rma = st_on.decode_layer(ow, 0, 0, x, want_branches=True)
        out_off = st_off.decode_layer(ow, 0, 0, x, rma_off=True)
        st_on.advance(0)
        st_off.advance(0, rma_off=True)
        assert bool((o_rma == 0).all())
        assert torch.equal(out_on, out_off), step


def test_rma_off_output_is_the_swa_branch_alone_and_memory_stays():
    ow, w, st = _seeded(52, 5000, [200])
    other = st.clone()
    # different anchor memory in the second copy: K, V and scores
    other.bank_k.copy_(torch.flip(other.bank_k, dims=[3]))
    other.pend_v.mul_(-1)
    other.bank_score.add_(1.5)
    before = {n: getattr(st, n).clone() for n in RMA_ARRAYS}
    ref = st.clone()
    for step in range(3):
        x = wl.make_x(52, 0, step, [0])[0]
        out, o_swa, o_rma = st.decode_layer(ow, 0, 0, x, want_branches=True, rma_off=True)
        out_other = other.decode_layer(ow, 0, 0, x, rma_off=True)
        _, o_swa_on, _ = ref.decode_layer(ow, 0, 0, x, want_branches=True)
        for s_ in (st, other):
            s_.advance(0, rma_off=True)
        ref.advance(0)
        assert bool((o_rma == 0).all())
        assert torch.equal(o_swa, o_swa_on)  # the SWA branch does not see the RMA switch
        o = bf16_exact(o_swa.reshape(-1).numpy())
        assert torch.equal(out, oracle.linear_bf16(w["w_o"], o))
        assert torch.equal(out, out_other)  # the anchor memory is not read
    for n in RMA_ARRAYS:
        assert torch.equal(getattr(st, n), before[n]), n  # ... nor written
    assert st.meta[0].tolist() == [5003, 200, 1024, 0]  # only the position moves
    assert torch.equal(st.win_k, other.win_k) and torch.equal(st.win_v, other.win_v)


def test_rma_off_prefill_equals_token_by_token_decode():
    ow, w, st_a = _seeded(53, 4096, [40])
    st_b = st_a.clone()
    T = 17
    xs = wl.make_x(53, 0, 0, range(T))
    out_chunk = st_a.prefill_chunk(ow, 0, 0, xs, rma_off=True)
    st_a.advance(0, T, rma_off=True)
    outs = []
    for i in range(T):
        outs.append(st_b.decode_layer(ow, 0, 0, xs[i], rma_off=True))
        st_b.advance(0, rma_off=True)
    assert torch.equal(out_chunk, torch.stack(outs))
    for n in oracle.OracleState.ARRAYS:
        assert torch.equal(getattr(st_a, n), getattr(st_b, n)), n


def test_full_bank_ignores_low_scoring_tail():
    # after the bank is full, extending the stream with tokens that score below every anchor
    # leaves the bank bit-identical whatever the stream length
    ow, w, st = _seeded(51, 4096, "zero")
    st.bank_score.add_(1000.0)  # every anchor outranks any new token
    before = st.clone()
    for i in range(256):
        st.decode_layer(ow, 0, 0, synth.normal((2560,), 51, synth.MISC + i, torch.bfloat16))
        st.advance(0)
    for n in ("bank_k", "bank_v", "bank_score", "bank_pos"):
        assert torch.equal(getattr(st, n), getattr(before, n)), n
    assert int(st.meta[0, 1]) == 0 and int(st.meta[0, 2]) == 1024 and int(st.meta[0, 0]) == 4352


def test_position_shift_invariance():
    # moving the stream by a multiple of 1024 (same ring slots) changes the SWA read only
    # through the rounding of the rotated keys
    outs = []
    for t0 in (4096, 4096 + 1024 * 37):
        ow, w, st = _seeded(61, t0, "uniform")
        x = synth.normal((2560,), 61, synth.MISC, torch.bfloat16)
        _, o_swa, _ = st.decode_layer(ow, 0, 0, x, want_branches=True)
        outs.append(o_swa)
    assert (outs[0] - outs[1]).abs().max() < 2e-2


# ---------------------------------------------------------- pending append

def test_append_pending_writes_only_the_next_slot_of_each_group():
    # neodrop.ai "内存还会跌吗？…" §三段记忆，只记值得记的: each token becomes one candidate
    # record per KV group, appended behind the ones already pending; the counters are
    # not touched by the append (the step's advance moves them)
    g = torch.Generator().manual_seed(77)
    st = oracle.OracleState(3, 2)
    for n in oracle.OracleState.ARRAYS:
        t = getattr(st, n)
        if t.dtype == torch.bfloat16 or t.dtype == torch.float32:
            t.copy_(torch.randn(t.shape, generator=g).to(t.dtype))
        else:
            t.copy_(torch.randint(-5, 10**6, t.shape, generator=g, dtype=torch.int32))
    st.meta.copy_(torch.tensor([[9000, 5, 1024, 0], [100, 0, 0, 0], [40000, 255, 1024, 0]],
                               dtype=torch.int32))
    before = {n: getattr(st, n).clone() for n in oracle.OracleState.ARRAYS}
    seqs = [2, 0]  # batch row b belongs to sequence seqs[b]; not in row order on purpose
    k = torch.randn(2, 4, 256, generator=g).to(torch.bfloat16)
    v = torch.randn(2, 4, 256, generator=g).to(torch.bfloat16)
    s = torch.randn(2, 4, generator=g, dtype=torch.float32)
    pos = torch.tensor([40000, 9000], dtype=torch.int32)
    st.append_pending(1, seqs, k, v, s, pos)
    expect = {n: t.clone() for n, t in before.items()}
    for b, seq in enumerate(seqs):
        p = int(before["meta"][seq, 1])
        for grp in range(4):
            expect["pend_k"][seq, 1, grp, p] = k[b, grp]
            expect["pend_v"][seq, 1, grp, p] = v[b, grp]
            expect["pend_score"][seq, 1, grp, p] = s[b, grp]
            expect["pend_pos"][seq, 1, grp, p] = pos[b]
    for n in oracle.OracleState.ARRAYS:
        assert torch.equal(getattr(st, n), expect[n]), n
    # slot 255 of sequence 2 really was written (the last slot of a block)
    assert torch.equal(st.pend_k[2, 1, 3, 255], k[0, 3])


def test_append_pending_equals_the_record_a_decode_step_appends():
    # the record a decode step appends is the token's k_rma (normed, rotated at its
    # position), v_rma, the group's FP32 score and the position: build it here from the
    # pinned pieces and append it to a copy of the same state
    ow, w, st = _seeded(55, 4096, "uniform")
    p = int(st.meta[0, 1])
    assert 0 < p < 255
    t = int(st.meta[0, 0])
    x = synth.normal((2560,), 55, synth.MISC, torch.bfloat16)
    st_b = st.clone()
    st.decode_layer(ow, 0, 0, x)
    proj = oracle.linear_bf16(w["w_qkv"], x)
    k = oracle.norm_rope(proj[10240:11264].view(4, 256), w["k_norm_rma"], t).view(1, 4, 256)
    v = proj[11264:12288].view(1, 4, 256)
    s = oracle.score(w["w1"], w["w2"], x)
    st_b.append_pending(0, [0], k, v, s, torch.tensor([t], dtype=torch.int32))
    for n in ("pend_k", "pend_v", "pend_score", "pend_pos", "bank_k", "bank_v", "bank_score",
              "bank_pos", "meta"):
        assert torch.equal(getattr(st, n), getattr(st_b, n)), n
    assert int(st.pend_pos[0, 0, 2, p]) == t
