"""CriticalKV observation-window scoring and two-stage selection on the GPU against the oracle
("Resumo Técnico: CriticalKV", Algoritmo, Etapas 1 e 2).

Element-wise: A (observation attention mass per query head) and N (||V_i W_O^h||_1) within
1e-4 relative per element. Selection: the stage-1 and stage-2 index sets equal the oracle's
except entries whose oracle score lies within 1e-4 relative of that stage's cut (near-ties,
counted); each stage's list is in descending oracle score up to the same tolerance.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from kv_cache_eviction_gqa_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = 1e-4


def _tdt(cfg):
    return torch.bfloat16 if cfg.dtype == "bf16" else torch.float16


def draw(cfg):
    Ks, Vs, Qs = [], [], []
    for b in range(cfg.B):
        for kvh in range(cfg.Hkv):
            K, V, q = W.draw_critical_unit(cfg, b, kvh)
            Ks.append(K), Vs.append(V), Qs.append(q)
    D = cfg.D
    K = np.stack(Ks).reshape(cfg.B, cfg.Hkv, cfg.n, D)
    V = np.stack(Vs).reshape(cfg.B, cfg.Hkv, cfg.n, D)
    q = np.stack(Qs).reshape(cfg.B, cfg.Hkv * cfg.G, cfg.n_obs, D)  # heads kvh*G + g
    return K, V, q, W.draw_critical_w_o(cfg)


def run_gpu(cfg, K, V, q, Wo):
    from kv_cache_eviction_gqa_b200 import binding as B
    t = _tdt(cfg)
    dev = torch.device("cuda")
    cv = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(dev, t)
    A, N, idx, scratch = B.criticalkv_select(cv(q), cv(K), cv(V), cv(Wo), cfg.budget, cfg.alpha)
    torch.cuda.synchronize()
    assert B.trim_status(scratch) == (0, 0)
    return A.cpu().numpy(), N.cpu().numpy(), idx.cpu().numpy()


def rel_err(got, ref):
    return np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)


def check_stage(got_ids, ref_ids, score, allowed_extra=()):
    """Sets equal up to near-ties at the cut; list in descending score. Returns #near-ties."""
    got_ids = np.asarray(got_ids)
    assert len(set(got_ids.tolist())) == len(got_ids), "duplicate picks"
    if len(ref_ids) == 0:
        assert len(got_ids) == 0
        return 0
    cut = score[ref_ids].min()
    diff = set(got_ids.tolist()) ^ set(np.asarray(ref_ids).tolist())
    diff -= set(allowed_extra)
    bad = [i for i in diff if abs(score[i] - cut) > TOL * cut]
    assert not bad, f"{len(bad)} picks differ away from the cut (e.g. {bad[:5]})"
    s = score[got_ids]
    assert np.all(s[1:] <= s[:-1] * (1 + TOL) + 1e-300), "stage list not in descending score"
    return len(diff)


def check_unit(cfg, K, V, q, Wo, A_gpu, N_gpu, idx_gpu, b, kvh, full_n=True):
    G = cfg.G
    heads = list(range(kvh * G, kvh * G + G))
    A_ref = O.observation_mass(q[b, kvh * G:(kvh + 1) * G], K[b, kvh])
    assert rel_err(A_gpu[b, kvh], A_ref).max() <= TOL
    N_ref = O.vwo_l1norm(V[b, kvh], Wo, heads, cfg.D)
    assert rel_err(N_gpu[b, kvh], N_ref).max() <= TOL
    s1, s2, a, p = O.criticalkv_select(A_ref, N_ref, cfg.budget, cfg.alpha)
    got = idx_gpu[b, kvh]
    if cfg.n <= cfg.budget:
        np.testing.assert_array_equal(got[:cfg.n], np.arange(cfg.n))
        assert np.all(got[cfg.n:] == -1)
        return 0
    b1 = int(np.floor(cfg.alpha * cfg.budget))
    g1, g2 = got[:b1], got[b1:]
    nt = check_stage(g1, s1, a)
    moved = set(g1.tolist()) ^ set(s1.tolist())
    nt += check_stage(g2, s2, p, allowed_extra=moved)
    return nt


def small(**kw):
    base = dict(B=1, Hq=8, Hkv=2, n=3000, n_obs=32, budget=256, hidden=512, seed=55)
    base.update(kw)
    return W.C3.scaled(**base)


@pytest.mark.parametrize("cfg", [
    small(),                                   # G=4, R=128, ragged last tile
    small(B=2, Hq=4, Hkv=2, n=1000, n_obs=64, seed=56),     # G=2, n_obs 64
    small(Hq=2, Hkv=2, n=777, n_obs=32, budget=100, alpha=0.3, seed=57),  # G=1, R=32
    small(n=4096, hidden=384, seed=58),        # hidden not a multiple of 128: SIMT norms
    small(D=64, n=2050, seed=59, dtype="fp16"),
], ids=["g4", "g2_obs64", "g1_alpha03", "hidden384", "d64_fp16"])
def test_criticalkv_small_full_parity(cfg):
    K, V, q, Wo = draw(cfg)
    A, N, idx = run_gpu(cfg, K, V, q, Wo)
    near = 0
    for b in range(cfg.B):
        for kvh in range(cfg.Hkv):
            near += check_unit(cfg, K, V, q, Wo, A, N, idx, b, kvh)
    print(cfg.name, "near-ties", near)


@pytest.mark.parametrize("case", ["n_le_budget", "alpha0", "alpha1", "n_equals_obs"])
def test_criticalkv_edges(case):
    cfg = {"n_le_budget": small(n=200, budget=256, seed=60),
           "alpha0": small(n=600, alpha=0.0, seed=61),
           "alpha1": small(n=600, alpha=1.0, seed=62),
           "n_equals_obs": small(n=32, budget=16, seed=63)}[case]
    K, V, q, Wo = draw(cfg)
    A, N, idx = run_gpu(cfg, K, V, q, Wo)
    for kvh in range(cfg.Hkv):
        check_unit(cfg, K, V, q, Wo, A, N, idx, 0, kvh)


@pytest.mark.slow
def test_criticalkv_full_c3_sampled_units():
    cfg = W.C3
    K, V, q, Wo = draw(cfg)
    A, N, idx = run_gpu(cfg, K, V, q, Wo)
    # every unit: stage-1 premise reported, picks distinct and in range
    for b in range(cfg.B):
        for kvh in range(cfg.Hkv):
            g = idx[b, kvh]
            assert g.min() >= 0 and g.max() < cfg.n and len(np.unique(g)) == cfg.budget
    near = 0
    for (b, kvh) in [(0, 0), (3, 7)]:
        near += check_unit(cfg, K, V, q, Wo, A, N, idx, b, kvh)
    a = A.sum(axis=2)
    b1 = cfg.budget // 2
    mass = np.take_along_axis(a, idx[..., :b1].astype(np.int64), axis=-1).sum(-1) / a.sum(-1)
    print("c3 near-ties", near, "stage-1 mass share min/mean", mass.min(), mass.mean())
