"""The synthetic input generator (CPU side): determinism, sub-ranges, distributions."""
import torch

import synth
from synth import workloads as wl


def test_normal_is_deterministic_and_subrange_consistent():
    a = synth.normal((1000,), 1, synth.MISC)
    b = synth.normal((1000,), 1, synth.MISC)
    assert torch.equal(a, b)
    part = torch.empty(300)
    synth.fill_normal_(part, 1, synth.MISC, index0=500)
    assert torch.equal(part, a[500:800])
    assert not torch.equal(a, synth.normal((1000,), 2, synth.MISC))
    assert not torch.equal(a, synth.normal((1000,), 1, synth.MISC + 1))


def test_normal_moments_and_support():
    x = synth.normal((400000,), 3, synth.MISC).double()
    assert abs(x.mean()) < 0.01 and abs(x.var() - 1) < 0.01
    assert x.abs().max() <= 6.0
    xb = synth.normal((4096,), 3, synth.MISC, torch.bfloat16)
    assert torch.equal(xb, x[:4096].float().to(torch.bfloat16))


def test_affine_and_integer_fills():
    g = synth.normal((256,), 4, synth.MISC, torch.float32, scale=0.1, offset=1.0)
    base = synth.normal((256,), 4, synth.MISC)
    assert torch.equal(g, base * 0.1 + 1.0)
    u = torch.empty(100000, dtype=torch.int32)
    synth.fill_uniform_(u, 5, synth.MISC, 256)
    assert int(u.min()) == 0 and int(u.max()) == 255
    s = torch.empty(4 * 1024, dtype=torch.int32)
    synth.fill_strata_(s, 6, synth.MISC, 1024, 3)
    for g4 in s.view(4, 1024):
        assert len(set(g4.tolist())) == 1024 and int(g4.max()) < 3072
    d = torch.empty(20 * 1280)
    synth.fill_normal_dup_(d, 7, synth.MISC, 1280, 20)
    ties = sum(1280 - len(set(r.tolist())) for r in d.view(20, 1280))
    assert 0.03 * 20 * 1280 < ties < 0.07 * 20 * 1280


def test_workload_weights_shapes():
    w = wl.make_weights(wl.seed_of(wl.DECODE_B1), 0)
    assert w["w_qkv"].shape == (12288, 2560) and w["w_qkv"].dtype == torch.bfloat16
    assert w["w_o"].shape == (2560, 4096)
    assert w["w1"].shape == (256, 2560) and w["w1"].dtype == torch.float32
    assert abs(float(w["w_qkv"].double().std()) * 2560 ** 0.5 - 1) < 0.01
    assert abs(float(w["q_norm_swa"].double().mean()) - 1) < 0.03
    pos = wl.window_positions(4096)
    assert sorted(pos.tolist()) == list(range(3072, 4096))
    assert all(int(p) % 1024 == s for s, p in enumerate(pos))


def test_commit_workload_rows_do_not_depend_on_which_rows_are_seeded():
    # a sampled sequence seeded alone gets the same keys as in the full batch, for the
    # first repetition and a later one (the oracle side seeds sampled rows alone)
    import oracle
    from synth import workloads as wl
    full = oracle.OracleState(6, 2, kv=False)
    part = oracle.OracleState(2, 2, kv=False)
    arrs = lambda o: {n: getattr(o, n) for n in oracle.OracleState.ARRAYS}
    for rep in (1, 2):
        wl.seed_commit_workload(arrs(full), range(6), 2, 32768, 99, rep)
        wl.seed_commit_workload(arrs(part), [1, 4], 2, 32768, 99, rep)
        for n in ("bank_score", "pend_score", "bank_pos", "pend_pos", "meta"):
            assert torch.equal(getattr(full, n)[[1, 4]], getattr(part, n)), (rep, n)
    # fresh scores per repetition, ~5% exact ties inside a merge
    a = oracle.OracleState(1, 1, kv=False)
    wl.seed_commit_workload(arrs(a), [0], 1, 32768, 99, 1)
    s1 = torch.cat([a.bank_score[0, 0, 0], a.pend_score[0, 0, 0]])
    wl.seed_commit_workload(arrs(a), [0], 1, 32768, 99, 2)
    s2 = torch.cat([a.bank_score[0, 0, 0], a.pend_score[0, 0, 0]])
    assert not torch.equal(s1, s2)
    dup = 1280 - torch.unique(s1).numel()
    assert 20 <= dup <= 120, dup
