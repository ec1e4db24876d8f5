"""Pins of the CPU oracle against the pages and the mathematics (no GPU).

Each test ties an oracle function to something other than its own formula:
hand-worked fixtures, closed forms, invariants, brute force on tiny inputs.
"""
import itertools
import math
import os

import numpy as np
import pytest

import oracle as O


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------


def _attend_scalar(q, K, V):
    """Scalar-loop softmax attention (math.exp, python floats)."""
    D = len(q)
    s = [sum(q[d] * K[i][d] for d in range(D)) / math.sqrt(D) for i in range(len(K))]
    m = max(s)
    e = [math.exp(x - m) for x in s]
    tot = sum(e)
    p = [x / tot for x in e]
    o = [sum(p[i] * V[i][d] for i in range(len(K))) for d in range(D)]
    return o, p


@pytest.mark.parametrize("n,D", [(1, 4), (5, 8), (64, 16), (37, 32)])
def test_attend_brute_force(n, D):
    r = _rng(n * 100 + D)
    q, K, V = r.standard_normal(D) * 2, r.standard_normal((n, D)), r.standard_normal((n, D))
    o, p = O.attend(q, K, V)
    o2, p2 = _attend_scalar(q.tolist(), K.tolist(), V.tolist())
    np.testing.assert_allclose(o, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(p, p2, rtol=1e-12, atol=1e-15)


def test_attend_closed_forms():
    r = _rng(1)
    V = r.standard_normal((9, 8))
    K = np.tile(r.standard_normal(8), (9, 1))  # identical keys -> uniform weights
    o, p = O.attend(r.standard_normal(8), K, V)
    np.testing.assert_allclose(p, np.full(9, 1 / 9), rtol=1e-14)
    np.testing.assert_allclose(o, V.mean(0), rtol=1e-12, atol=1e-14)
    o1, p1 = O.attend(r.standard_normal(8), K[:1], V[:1])  # one token -> its value
    np.testing.assert_allclose(o1, V[0], rtol=1e-15)
    # one dominant key: q aligned with a key of very large norm -> o ~ that value
    K2 = r.standard_normal((9, 8))
    K2[4] = 1e3 * np.ones(8)
    o2, p2 = O.attend(np.ones(8), K2, V)
    np.testing.assert_allclose(o2, V[4], rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# INT2 quantiser
# ---------------------------------------------------------------------------


def _read_int2_golden(golden_dir):
    rows = []
    with open(os.path.join(golden_dir, "int2_groups.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, vals, s, z, codes = [t.strip() for t in line.split("|")]
            rows.append((name, np.array([float(v) for v in vals.split()], np.float32),
                         float(s), float(z), np.array([int(c) for c in codes.split()])))
    return rows


def test_int2_golden_groups(golden_dir):
    rows = _read_int2_golden(golden_dir)
    assert len(rows) == 3
    for name, x, s, z, codes in rows:
        c, s16, z16 = O.int2_quantize(x[None, :])
        assert float(s16[0, 0]) == s, name
        assert float(z16[0, 0]) == z, name
        np.testing.assert_array_equal(c[0], codes, err_msg=name)


def test_int2_grid_roundtrip():
    """Values on {z, z+s, z+2s, z+3s} with both ends present come back exactly."""
    r = _rng(2)
    T, D = 7, 64
    z = r.choice([-2.0, -1.0, -0.5, 0.25, 1.5], size=(T, D // 16))
    s = r.choice([0.125, 0.25, 0.5, 1.0], size=(T, D // 16))
    codes = r.integers(0, 4, size=(T, D // 16, 16))
    codes[..., 0], codes[..., 1] = 0, 3
    x = (codes * s[..., None] + z[..., None]).reshape(T, D)
    c, s16, z16 = O.int2_quantize(x)
    np.testing.assert_array_equal(c.reshape(T, D // 16, 16), codes)
    np.testing.assert_array_equal(s16.astype(np.float64), s)
    np.testing.assert_array_equal(O.int2_dequantize(c, s16, z16), x)


def test_int2_constant_group_and_range():
    x = np.full((2, 32), 0.3, np.float32)
    x[1] = -7.0
    c, s16, z16 = O.int2_quantize(x)
    assert (c == 0).all() and (s16 == 0).all()
    np.testing.assert_array_equal(O.int2_dequantize(c, s16, z16)[1], -7.0)
    r = _rng(3)
    y = r.standard_normal((50, 128)).astype(np.float32)
    c, s16, z16 = O.int2_quantize(y)
    assert c.max() <= 3
    # dequantised values stay within half a step (plus fp16 rounding of s and z)
    err = np.abs(O.int2_dequantize(c, s16, z16) - y).reshape(50, 8, 16).max(-1)
    assert (err <= 0.5 * s16.astype(np.float64) * 1.01 + 2e-3 * np.abs(y).reshape(50, 8, 16).max(-1)).all()


def test_int2_decisions_match_exact_arithmetic_off_boundaries():
    """The float32 decision agrees with exact arithmetic except at rounding ties."""
    r = _rng(4)
    y = (r.standard_normal((200, 128)) * 3).astype(np.float32)
    c, s16, z16 = O.int2_quantize(y)
    g = y.astype(np.float64).reshape(200, 8, 16)
    s = s16.astype(np.float64)[..., None]
    z = z16.astype(np.float64)[..., None]
    t = (g - z) / s
    exact = np.clip(np.floor(t + 0.5), 0, 3)
    near = np.abs(t - np.floor(t) - 0.5) < 1e-4
    diff = (exact != c.reshape(200, 8, 16)) & ~near
    assert not diff.any()


# ---------------------------------------------------------------------------
# projected-value norms
# ---------------------------------------------------------------------------


def test_vwo_identity_reduces_to_value_l1():
    r = _rng(5)
    Hq, D = 4, 8
    V = r.standard_normal((11, D))
    W = np.eye(Hq * D)
    N = O.vwo_l1norm(V, W, [1, 3], D)
    np.testing.assert_allclose(N, np.repeat(np.abs(V).sum(1)[:, None], 2, 1), rtol=1e-15)


def test_vwo_hand_worked_and_invariances():
    # D = 2, one head, hidden = 3: W = [[1, -2, 0], [3, 1, -1]], v = [1, 2]
    # v W = [1 + 6, -2 + 2, 0 - 2] = [7, 0, -2] -> ||.||_1 = 9
    W = np.array([[1.0, -2, 0], [3, 1, -1]])
    assert O.vwo_l1norm(np.array([[1.0, 2.0]]), W, [0], 2)[0, 0] == 9.0
    r = _rng(6)
    V, W2 = r.standard_normal((5, 4)), r.standard_normal((8, 6))
    base = O.vwo_l1norm(V, W2, [0, 1], 4)
    perm = r.permutation(6)
    np.testing.assert_allclose(O.vwo_l1norm(V, W2[:, perm] * -1, [0, 1], 4), base, rtol=1e-14)
    np.testing.assert_allclose(O.vwo_l1norm(-V, W2, [0, 1], 4), base, rtol=1e-14)


# ---------------------------------------------------------------------------
# two-stage selection
# ---------------------------------------------------------------------------


def test_two_stage_golden(golden_dir):
    vals = {}
    with open(os.path.join(golden_dir, "two_stage.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            k, v = [t.strip() for t in line.split("|")]
            vals[k] = [float(x) for x in v.split()]
    mass, pert = np.array(vals["mass"]), np.array(vals["pert"])
    F, Q, alpha = int(vals["F"][0]), int(vals["Q"][0]), vals["alpha"][0]
    L = np.arange(6)
    f1, f2 = O.two_stage(L, mass, pert, F, alpha)
    full = np.sort(np.concatenate([f1, f2]))
    np.testing.assert_array_equal(full, np.array(vals["full"], int))
    rest = np.setdiff1d(L, full)
    q1, q2 = O.two_stage(rest, mass, pert, Q, alpha)
    np.testing.assert_array_equal(np.sort(np.concatenate([q1, q2])), np.array(vals["int2"], int))
    ev = np.setdiff1d(rest, np.concatenate([q1, q2]))
    np.testing.assert_array_equal(ev, np.array(vals["evicted"], int))


@pytest.mark.parametrize("seed", range(6))
def test_two_stage_exhaustive(seed):
    """Stage 1 is the best b' by attention; stage 2 the best b-b' subset of the rest
    by total perturbation score, checked over every subset (n <= 12)."""
    r = _rng(100 + seed)
    n = int(r.integers(5, 13))
    b = int(r.integers(2, n))
    attn, pert = r.random(n), r.random(n)
    ids = np.arange(n)
    s1, s2 = O.two_stage(ids, attn, pert, b, 0.5)
    b1 = b // 2
    assert len(s1) == b1 and len(s2) == b - b1 and not set(s1) & set(s2)
    best1 = max(itertools.combinations(range(n), b1), key=lambda c: sum(attn[list(c)]))
    assert sorted(best1) == sorted(s1.tolist())
    rest = [i for i in range(n) if i not in set(s1.tolist())]
    best2 = max(itertools.combinations(rest, b - b1), key=lambda c: sum(pert[list(c)]))
    assert sorted(best2) == sorted(s2.tolist())


def test_two_stage_true_perturbation_rank_informative():
    """Informative ("Resumo Técnico: CriticalKV", Framework Teórico): over every size-b subset
    of a small attention problem, the rank of the TwoStage pick by the true perturbation
    L = ||(o - o_hat) W_O||_1. Nothing is asserted about the rank: the pages bound L from above
    and give no value for it; the test only prints where the pick falls."""
    r = _rng(55)
    n, D, b = 10, 8, 4
    q = r.standard_normal(D) * 2
    K = r.standard_normal((n, D))
    V = r.standard_normal((n, D))
    Wo = r.standard_normal((D, 16)) / 4
    _, p = O.attend(q, K, V)
    norms = O.vwo_l1norm(V, Wo, [0], D)[:, 0]
    s1, s2 = O.two_stage(np.arange(n), p, p * norms, b, 0.5)
    pick = sorted(np.concatenate([s1, s2]).tolist())
    Ls = sorted((O.output_perturbation(q, K, V, list(c), Wo), list(c))
                for c in itertools.combinations(range(n), b))
    rank = [c for _, c in Ls].index(pick) + 1
    L_pick = O.output_perturbation(q, K, V, pick, Wo)
    assert L_pick >= Ls[0][0] - 1e-12
    print(f"TwoStage pick ranks {rank} of {len(Ls)} subsets by true L "
          f"(L = {L_pick:.4f}, best {Ls[0][0]:.4f}, worst {Ls[-1][0]:.4f})")


def test_two_stage_small_set_and_ties():
    ids = np.array([3, 1, 2])
    s1, s2 = O.two_stage(ids, np.zeros(4), np.zeros(4), 5, 0.5)
    assert sorted(s1.tolist()) == [1, 2, 3] and s2.size == 0
    # all-equal scores -> the lowest ids win in both stages
    s1, s2 = O.two_stage(np.arange(10), np.ones(10), np.ones(10), 4, 0.5)
    assert s1.tolist() == [0, 1] and s2.tolist() == [2, 3]


def test_stage1_mass_premise_on_peaked_distribution():
    """Stage 1 with alpha = 0.5 holds more than half the attention when it is peaked."""
    r = _rng(7)
    w = (np.arange(1, 201) ** -1.1)
    p = w[r.permutation(200)]
    p /= p.sum()
    s1, _ = O.two_stage(np.arange(200), p, r.random(200), 40, 0.5)
    assert p[s1].sum() > 0.5


# ---------------------------------------------------------------------------
# QEvict unit
# ---------------------------------------------------------------------------


def _unit(seed, n0=96, D=32, G=2, w=16, F=2, Q=2, dtype="bf16"):
    r = _rng(seed)
    K0 = r.standard_normal((n0, D)).astype(np.float32)
    V0 = r.standard_normal((n0, D)).astype(np.float32)
    K0 = O.round_to_cache_dtype(K0, dtype)
    V0 = O.round_to_cache_dtype(V0, dtype)
    W = r.standard_normal((2 * G * D, 24)) / 8
    u = O.QEvictUnit(K0, V0, W, 1, G, w, F, Q, 0.5, dtype, n0 + 64)
    return u, r


def test_unit_mass_invariant_and_tiers():
    u, r = _unit(8)
    D, G = u.D, u.G
    for s in range(40):
        k = O.round_to_cache_dtype(r.standard_normal(D).astype(np.float32), "bf16")
        v = O.round_to_cache_dtype(r.standard_normal(D).astype(np.float32), "bf16")
        u.append(k, v)
        _, step_mass = u.attend_and_score(r.standard_normal((G, D)))
        # sum over live windows (tail included) of this step's mass = G exactly
        assert abs(step_mass.sum() - G) < 1e-12
        assert (step_mass[u.tier == 0] == 0).all()
        if s % 4 == 0:
            u.route()
            assert (u.tier == 2).sum() <= u.F + 0 and (u.tier == 1).sum() <= u.Q
    assert (u.tier == 3).sum() <= 1


def test_unit_full_budget_is_plain_attention():
    """With budgets covering every window nothing is demoted or evicted: the step
    output equals plain attention over every token with its original values."""
    u, r = _unit(9, F=100, Q=0)
    allK, allV = list(u.Kst[:u.n]), list(u.Vst[:u.n])
    for s in range(20):
        k = O.round_to_cache_dtype(r.standard_normal(u.D).astype(np.float32), "bf16")
        v = O.round_to_cache_dtype(r.standard_normal(u.D).astype(np.float32), "bf16")
        qG = r.standard_normal((u.G, u.D))
        o, _ = u.step(s, qG, k, v, 4)
        allK.append(k)
        allV.append(v)
        for j in range(u.G):
            o_ref, _ = _attend_scalar(qG[j].tolist(), allK, allV)
            np.testing.assert_allclose(o[j], o_ref, rtol=1e-10, atol=1e-12)
    assert len(u.ledger) == 0


def test_write_once_ledger():
    """demote -> promote -> demote returns byte-identical codes from the ledger."""
    u, r = _unit(10, n0=64, D=32, w=16)
    sl = u.tokens(1)
    before = u.Kst[sl].copy()
    u.apply({1: O.INT2})
    (ck, sk, zk), _ = u.ledger[1]
    ck, sk, zk = ck.copy(), sk.copy(), zk.copy()
    np.testing.assert_array_equal(u.Keff[sl], O.int2_dequantize(ck, sk, zk))
    u.apply({1: O.FULL})
    np.testing.assert_array_equal(u.Kst[sl], O.int2_promote_values(ck, sk, zk, "bf16"))
    assert not np.array_equal(u.Kst[sl], before)
    u.apply({1: O.INT2})
    (ck2, sk2, zk2), _ = u.ledger[1]
    np.testing.assert_array_equal(ck2, ck)
    np.testing.assert_array_equal(sk2, sk)
    np.testing.assert_array_equal(zk2, zk)
    u.apply({1: O.EVICTED})
    assert 1 not in u.ledger


def test_write_once_constructed_requantisation_drift(golden_dir):
    """Hand-worked fp16 group whose top code never occurs: re-quantising the
    promoted values shrinks the scale and moves codes; the ledger keeps them."""
    vals = {}
    with open(os.path.join(golden_dir, "write_once_fp16.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            k, v = [t.strip() for t in line.split("|")]
            vals[k] = [int(x) for x in v.split()]
    unit = 2.0 ** -24
    x = (np.array(vals["k"], np.float64) * unit).astype(np.float32)[None, :]
    c, s, z = O.int2_quantize(x)
    assert c[0].tolist() == vals["codes"]
    assert float(s[0, 0]) == vals["s_units"][0] * unit and float(z[0, 0]) == vals["z_units"][0] * unit
    promoted = O.int2_promote_values(c, s, z, "fp16")
    c2, s2, z2 = O.int2_quantize(promoted.astype(np.float32))
    assert c2[0].tolist() == vals["requant_codes"]
    assert float(s2[0, 0]) == vals["requant_s_units"][0] * unit
    # through the unit: the window's first K group carries the constructed values
    r = _rng(14)
    K0 = O.round_to_cache_dtype(r.standard_normal((32, 16)).astype(np.float32), "fp16")
    V0 = O.round_to_cache_dtype(r.standard_normal((32, 16)).astype(np.float32), "fp16")
    K0[16] = x[0]
    u = O.QEvictUnit(K0, V0, r.standard_normal((32, 4)), 0, 1, 16, 1, 1, 0.5, "fp16", 64)
    for t in (O.INT2, O.FULL, O.INT2, O.FULL, O.INT2):
        u.apply({1: t})
    (ck, sk, zk), _ = u.ledger[1]
    assert ck[0, :16].tolist() == vals["codes"]
    assert float(sk[0, 0]) == vals["s_units"][0] * unit


# ---------------------------------------------------------------------------
# observation-window mass (CriticalKV with a SnapKV-style window)
# ---------------------------------------------------------------------------


def test_observation_mass_brute_force_and_sum():
    r = _rng(11)
    G, n_obs, n, D = 2, 3, 10, 8
    q = r.standard_normal((G, n_obs, D))
    K = r.standard_normal((n, D))
    A = O.observation_mass(q, K)
    np.testing.assert_allclose(A.sum(1), np.full(G, n_obs), rtol=1e-13)
    for h in range(G):
        ref = np.zeros(n)
        for j in range(n_obs):
            last = n - n_obs + j + 1
            _, p = _attend_scalar(q[h, j].tolist(), K[:last].tolist(), np.zeros((last, D)).tolist())
            ref[:last] += p
        np.testing.assert_allclose(A[h], ref, rtol=1e-12, atol=1e-15)
    # causality: the last key is only seen by the last query
    assert A[:, -1].min() > 0


def test_criticalkv_select_hand():
    # G = 1, 4 tokens, b = 2, alpha 0.5: stage 1 takes the best A, stage 2 the best A*N
    A = np.array([[0.4, 0.3, 0.2, 0.1]])
    N = np.array([[1.0], [1.0], [10.0], [0.5]])
    s1, s2, a, p = O.criticalkv_select(A, N, 2, 0.5)
    assert s1.tolist() == [0] and s2.tolist() == [2]


# ---------------------------------------------------------------------------
# DBTrimKV global top-M
# ---------------------------------------------------------------------------


def test_trim_constant_beta_keeps_most_recent():
    pos = [np.array([1, 5, 9, 20]), np.array([2, 3, 30])]
    betas = [np.full(4, 0.9, np.float32), np.full(3, 0.9, np.float32)]
    masks, lens, _ = O.trim_global_topm(betas, pos, 32, 3)
    # ages: head0 31,27,23,12 ; head1 30,29,2 -> the three youngest: 2 (h1), 12 (h0), 23 (h0)
    assert masks[0].tolist() == [False, False, True, True]
    assert masks[1].tolist() == [False, False, True]
    assert lens.tolist() == [2, 1]


def test_trim_equal_age_prefers_larger_beta_and_ties_by_index():
    pos = [np.array([10, 10]), np.array([10])]
    betas = [np.array([0.5, 0.9], np.float32), np.array([0.9], np.float32)]
    masks, lens, _ = O.trim_global_topm(betas, pos, 20, 1)
    assert masks[0].tolist() == [False, True] and masks[1].tolist() == [False]
    masks, lens, _ = O.trim_global_topm([np.ones(3, np.float32)], [np.array([0, 1, 2])], 5, 2)
    assert masks[0].tolist() == [True, True, False]  # beta = 1: all keys 0, lowest indices


def test_trim_matches_argsort_random():
    r = _rng(12)
    betas = [r.beta(8, 1, size=int(r.integers(3, 30))).astype(np.float32) for _ in range(6)]
    poss = [np.sort(r.choice(100, size=b.size, replace=False)) for b in betas]
    M = 40
    masks, lens, keys = O.trim_global_topm(betas, poss, 100, M)
    # reference: the M largest beta^(t-i) by direct power (no logs)
    r_val = np.concatenate([b.astype(np.float64) ** (100 - p) for b, p in zip(betas, poss)])
    idx = np.argsort(-r_val, kind="stable")[:M]
    ref = np.zeros(r_val.size, bool)
    ref[idx] = True
    got = np.concatenate(masks)
    # ties between distinct entries are measure-zero here; the sets must agree
    assert (got == ref).all()
    assert lens.sum() == M


def test_output_perturbation_full_subset_is_zero():
    r = _rng(13)
    q, K, V = r.standard_normal(8), r.standard_normal((6, 8)), r.standard_normal((6, 8))
    assert O.output_perturbation(q, K, V, np.arange(6)) < 1e-14
    assert O.output_perturbation(q, K, V, np.arange(3)) > 0


# ---------------------------------------------------------------------------
# QEvict diagnostics ("Resumo Técnico: QEvict", Principais Contribuições 1)
# ---------------------------------------------------------------------------

_LETTER = {"E": O.EVICTED, "Q": O.INT2, "F": O.FULL, "T": O.TAIL}


def _golden_diag(golden_dir):
    units, counts, vals = {}, {}, {}
    for line in open(os.path.join(golden_dir, "diag_tiers.txt")):
        if line.startswith("#") or "|" not in line:
            continue
        key, val = (x.strip() for x in line.split("|"))
        if key.startswith("unit"):
            units[int(key.split()[1])] = [[_LETTER[c] for c in ev] for ev in val.split()]
        elif key.startswith("counts"):
            counts[int(key.split()[1])] = [int(x) for x in val.split()]
        else:
            vals[key] = float(val)
    return units, counts, vals


def test_tier_diagnostics_golden(golden_dir):
    units, counts, vals = _golden_diag(golden_dir)
    per = []
    for u in sorted(units):
        r = O.tier_diagnostics([np.array(ev) for ev in units[u]])
        assert r["per_unit"][0].tolist() == counts[u]
        per.append(r["per_unit"][0])
    # pooled over the two units
    tot = np.sum(per, axis=0)
    assert tot[1] / tot[0] == vals["churn"]
    assert abs(tot[5] / tot[4] - vals["lir"]) < 1e-15


def test_tier_diagnostics_invariants():
    F, Q, E, T = O.FULL, O.INT2, O.EVICTED, O.TAIL
    # a constant sequence: live windows counted every event, nothing changes or exits
    m = np.array([[F, Q, E, T]])
    r = O.tier_diagnostics([m, m, m])
    assert r["per_unit"][0].tolist() == [4, 0, 0, 0, 0, 0] and r["churn"] == 0.0
    assert np.isnan(r["lir"])
    # one window alternating F/Q over 5 events: 4 changes, 2 exits, 2 re-entries, 1 window each
    seq = [np.array([x]) for x in (F, Q, F, Q, F)]
    r = O.tier_diagnostics(seq)
    assert r["per_unit"][0].tolist() == [4, 4, 2, 2, 1, 1] and r["lir"] == 1.0
    # eviction is final: F -> E -> E counts one exit and nothing after it
    r = O.tier_diagnostics([np.array([F]), np.array([E]), np.array([E])])
    assert r["per_unit"][0].tolist() == [1, 1, 1, 0, 1, 0] and r["lir"] == 0.0
    # tail and not-yet-existing windows are not live; their first F is not a re-entry
    r = O.tier_diagnostics([np.array([E, T]), np.array([T, F]), np.array([F, F])])
    assert r["per_unit"][0].tolist() == [1, 0, 0, 0, 0, 0]
    # units are independent: stacking two units adds their counts
    a = [np.array([F, Q]), np.array([Q, F]), np.array([F, F])]
    b = [np.array([Q, F]), np.array([F, E]), np.array([E, E])]
    ra, rb = O.tier_diagnostics(a)["per_unit"][0], O.tier_diagnostics(b)["per_unit"][0]
    rab = O.tier_diagnostics([np.stack([x, y]) for x, y in zip(a, b)])["per_unit"]
    assert rab[0].tolist() == ra.tolist() and rab[1].tolist() == rb.tolist()


def _fmm_brute(qG, K, tiers, window):
    n, D = len(K), len(K[0])
    acc = 0.0
    for q in qG:
        s = [sum(float(q[d]) * float(K[i][d]) for d in range(D)) / math.sqrt(D) for i in range(n)]
        mx = max(s)
        e = [math.exp(x - mx) for x in s]
        tot = sum(e)
        acc += sum(e[i] for i in range(n) if tiers[i // window] == O.EVICTED) / tot
    return acc / len(qG)


def test_future_missed_mass_brute_force():
    rng = np.random.default_rng(91)
    for n, G, D, w in [(37, 3, 8, 8), (16, 1, 4, 16), (50, 5, 16, 4)]:
        qG = rng.normal(size=(G, D)) * 2
        K = rng.normal(size=(n, D))
        tiers = rng.choice([O.EVICTED, O.INT2, O.FULL], size=(n + w - 1) // w)
        tiers[-1] = O.TAIL
        assert abs(O.future_missed_mass(qG, K, tiers, w) - _fmm_brute(qG, K, tiers, w)) < 1e-12


def test_future_missed_mass_closed_forms():
    rng = np.random.default_rng(92)
    n, D, w = 40, 8, 8
    K = rng.normal(size=(n, D))
    tiers = np.array([O.EVICTED, O.FULL, O.EVICTED, O.INT2, O.TAIL])
    # q = 0: uniform attention, so the missed mass is the evicted share of the tokens
    assert abs(O.future_missed_mass(np.zeros((3, D)), K, tiers, w) - 16 / 40) < 1e-15
    # nothing evicted -> 0; everything evicted -> 1; no tokens -> 0
    q = rng.normal(size=(2, D))
    assert O.future_missed_mass(q, K, np.full(5, O.FULL), w) == 0.0
    assert abs(O.future_missed_mass(q, K, np.full(5, O.EVICTED), w) - 1.0) < 1e-15
    assert O.future_missed_mass(q, K[:0], tiers, w) == 0.0
    # hand-worked: D = 4 (sqrt D = 2), q = (2, 0, 0, 0), K_i = (ln a_i, 0, 0, 0) gives
    # scores ln a_i and p proportional to a = 1:2:3:4; window 2 with window 0 evicted -> 3/10
    a = np.array([1.0, 2.0, 3.0, 4.0])
    Kh = np.zeros((4, 4))
    Kh[:, 0] = np.log(a)
    fmm = O.future_missed_mass(np.array([[2.0, 0, 0, 0]]), Kh, np.array([O.EVICTED, O.FULL]), 2)
    assert abs(fmm - 0.3) < 1e-15


# ---------------------------------------------------------------------------
# global routing across layers ("Make Each Token Count", Metodologia 3, on QEvict's tiers)
# ---------------------------------------------------------------------------


def _scored_units(n_units, seed, n0=48, w=16):
    units = []
    for k in range(n_units):
        u, _ = _unit(seed + k, n0=n0, w=w)
        units.append(u)
    return units


def test_route_global_golden(golden_dir):
    vals = {}
    for line in open(os.path.join(golden_dir, "route_global.txt")):
        if line.startswith("#") or "|" not in line:
            continue
        key, val = (x.strip() for x in line.split("|"))
        vals[key] = val.split()
    units = _scored_units(2, 300)  # 3 complete windows each (48 tokens of 16)
    for k, u in enumerate(units):
        u.mass[:3] = [float(x) for x in vals[f"mass {k}"]]
        u.pert[:3] = [float(x) for x in vals[f"pert {k}"]]
    O.route_global(units, int(vals["F"][0]), int(vals["Q"][0]), float(vals["alpha"][0]))
    letter = {O.FULL: "F", O.INT2: "Q", O.EVICTED: "E"}
    for k, u in enumerate(units):
        assert [letter[int(t)] for t in u.tier[:3]] == vals[f"tiers {k}"]


def test_route_global_one_unit_is_the_unit_routing():
    r = _rng(301)
    a, b = _scored_units(1, 302, n0=160)[0], _scored_units(1, 302, n0=160)[0]
    for u in (a, b):
        u.mass[:10] = r.random(10) if u is a else a.mass[:10]
        u.pert[:10] = r.random(10) if u is a else a.pert[:10]
    a.pert[:10] = b.pert[:10] = r.random(10)
    b.mass[:10] = a.mass[:10]
    a.F = b.F = 3
    a.Q = b.Q = 4
    a.route()
    O.route_global([b], 3, 4, 0.5)
    np.testing.assert_array_equal(a.tier, b.tier)


def test_route_global_budget_covers_everything_and_ties():
    units = _scored_units(3, 310)
    for u in units:
        u.mass[:3] = 1.0
        u.pert[:3] = 1.0
    # budgets for all 9 live windows: nothing evicted, all full
    O.route_global(units, 9, 0, 0.5)
    assert all((u.tier[:3] == O.FULL).all() for u in units)
    # equal scores everywhere: the lower flat ids (earlier units) win both stages
    units = _scored_units(3, 320)
    for u in units:
        u.mass[:3] = 0.5
        u.pert[:3] = 0.5
    O.route_global(units, 4, 3, 0.5)
    assert units[0].tier[:3].tolist() == [O.FULL] * 3 and units[1].tier[0] == O.FULL
    assert units[1].tier[1:3].tolist() == [O.INT2] * 2 and units[2].tier[0] == O.INT2
    assert units[2].tier[1:3].tolist() == [O.EVICTED] * 2


# ---------------------------------------------------------------------------
# SEKV mixed-resolution attention ("Resumo Técnico: SEKV", Metodologia 1-3)
# ---------------------------------------------------------------------------


def test_sekv_segmentation_hand_worked():
    # surprisal 5 0 0 7 1 2 9 0 with tau = 5: anchors at 0, 3, 6; spans [1, 3), [4, 6), [7, 8)
    anchors, spans = O.sekv_segment(np.array([5, 0, 0, 7, 1, 2, 9, 0], np.float32), 5.0)
    assert anchors.tolist() == [0, 3, 6] and spans == [(1, 3), (4, 6), (7, 8)]
    # no anchor: one span over everything; every token an anchor: no span
    assert O.sekv_segment(np.zeros(5, np.float32), 1.0)[1] == [(0, 5)]
    assert O.sekv_segment(np.ones(4, np.float32), 0.5)[1] == []


def test_sekv_summary_weighted_mean_and_zero_fallback():
    K = np.array([[1.0, 0.0], [3.0, 4.0], [0.0, 8.0]])
    V = np.array([[2.0, 2.0], [6.0, -2.0], [1.0, 1.0]])
    # weights 1 and 3 over tokens 0..1: (k0 + 3 k1) / 4 = (2.5, 3.0); (v0 + 3 v1) / 4 = (5.0, -1.0)
    kb, vb, sz = O.sekv_summaries(K, V, np.array([1.0, 3.0, 0.0]), [(0, 2), (2, 3)])
    assert np.allclose(kb[0], [2.5, 3.0]) and np.allclose(vb[0], [5.0, -1.0]) and sz.tolist() == [2, 1]
    # zero surprisal over a span: the plain mean
    kb, vb, _ = O.sekv_summaries(K, V, np.zeros(3), [(0, 3)])
    assert np.allclose(kb[0], K.mean(axis=0)) and np.allclose(vb[0], V.mean(axis=0))


def test_sekv_identical_span_summary_is_exact():
    """A span of w identical tokens summarised with ln w added to its score carries exactly
    the attention of its w tokens: w e^s = e^(s + ln w)."""
    r = _rng(401)
    D, G = 16, 3
    K = r.standard_normal((12, D))
    V = r.standard_normal((12, D))
    K[4:9] = K[4]
    V[4:9] = V[4]
    H = np.full(12, 9.0, np.float32)
    H[4:9] = r.random(5).astype(np.float32)  # tokens 4..8 below tau: one span
    q = r.standard_normal((G, D))
    o, exp_ = O.sekv_attend(q, K, V, H, 5.0, np.inf)
    assert exp_.tolist() == [False]
    for h in range(G):
        o_full, _ = O.attend(q[h], K, V)
        assert np.allclose(o[h], o_full, rtol=1e-12, atol=1e-12)


def test_sekv_everything_expanded_or_anchored_is_plain_attention():
    r = _rng(402)
    D, G, n = 16, 2, 40
    K = r.standard_normal((n, D))
    V = r.standard_normal((n, D))
    H = r.exponential(size=n).astype(np.float32)
    q = r.standard_normal((G, D))
    for tau, theta in ((1.0, -np.inf), (-1.0, 0.0)):
        o, _ = O.sekv_attend(q, K, V, H, tau, theta)
        for h in range(G):
            o_full, _ = O.attend(q[h], K, V)
            assert np.allclose(o[h], o_full, rtol=1e-12, atol=1e-12)
    # the gate of a span is the largest scaled score over the heads
    _, spans = O.sekv_segment(H, 1.0)
    kb, _, _ = O.sekv_summaries(K, V, H, spans)
    g = O.sekv_gates(q, kb)
    assert np.allclose(g, np.max(q @ kb.T, axis=0) / math.sqrt(D))


# ---------------------------------------------------------------------------
# hand-worked pins of the unit's perturbation accumulation, the SEKV gate and the
# output perturbation (fixtures carry the citation and the arithmetic)
# ---------------------------------------------------------------------------


def _read_kv_golden(golden_dir, name):
    vals = {}
    with open(os.path.join(golden_dir, name)) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            k, v = [t.strip() for t in line.split("|")]
            vals[k] = np.array([float(x) for x in v.split()])
    return vals


def test_unit_perturbation_golden(golden_dir):
    g = _read_kv_golden(golden_dir, "qevict_pert.txt")
    K0 = np.stack([np.log(g["a"]), np.log(g["b"])], axis=1)
    V0 = g["V"].reshape(4, 2)
    W_O = g["W_O"].reshape(4, 2)
    u = O.QEvictUnit(K0, V0, W_O, 0, 2, 2, 8, 8, 0.5, "fp16", 8)
    # the two windows of the prefill are full precision and every token is live
    assert list(u.tier[:2]) == [O.FULL, O.FULL]
    qG = np.array([[math.sqrt(2), 0.0], [0.0, math.sqrt(2)]])
    _, step_mass = u.attend_and_score(qG)
    np.testing.assert_allclose(step_mass[:2], g["mass_step"], rtol=1e-12)
    np.testing.assert_allclose(u.pert[:2], g["pert_step"], rtol=1e-12)
    # undecayed sums: a second identical step doubles both scores
    u.attend_and_score(qG)
    np.testing.assert_allclose(u.mass[:2], 2 * g["mass_step"], rtol=1e-12)
    np.testing.assert_allclose(u.pert[:2], 2 * g["pert_step"], rtol=1e-12)


def test_sekv_gates_golden(golden_dir):
    g = _read_kv_golden(golden_dir, "sekv_gates.txt")
    q = g["q"].reshape(2, 4)
    kbar = g["kbar"].reshape(2, 4)
    np.testing.assert_allclose(O.sekv_gates(q, kbar), g["gates"], rtol=1e-15)
    # the gate decides expansion inside sekv_attend: with surprisal (0, 5, 0) and tau = 1 the
    # middle token is an anchor and the other two are one-token spans whose summaries are
    # exactly kbar_0 and kbar_1
    H = np.array([0.0, 5.0, 0.0])
    anchors, spans = O.sekv_segment(H, 1.0)
    assert list(anchors) == [1] and [tuple(s) for s in spans] == [(0, 1), (2, 3)]
    K3 = np.stack([kbar[0], np.zeros(4), kbar[1]])
    V3 = np.eye(3, 4)
    _, expanded = O.sekv_attend(q, K3, V3, H, 1.0, g["theta"][0])
    np.testing.assert_array_equal(expanded.astype(int), g["expanded"].astype(int))


def test_output_perturbation_golden(golden_dir):
    g = _read_kv_golden(golden_dir, "output_perturbation.txt")
    K = np.stack([np.log(g["a"]), np.zeros(3)], axis=1)
    V = g["V"].reshape(3, 2)
    q = np.array([math.sqrt(2), 0.0])
    subset = g["subset"].astype(int)
    assert O.output_perturbation(q, K, V, subset) == pytest.approx(g["L"][0], rel=1e-12)
    W = g["W_O_h"].reshape(2, 2)
    assert O.output_perturbation(q, K, V, subset, W) == pytest.approx(g["L_projected"][0], rel=1e-12)
    # the full set perturbs nothing
    assert O.output_perturbation(q, K, V, np.arange(3), W) == pytest.approx(0.0, abs=1e-15)
