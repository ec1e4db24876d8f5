"""QEvict diagnostics on the GPU against the oracle ("Resumo Técnico: QEvict", Principais
Contribuições 1: Churn de Seleção, LIR Global, Massa Perdida Futura).

Tier diagnostics are integer counts: every per-unit counter must equal the oracle's exactly,
over seeded routing-like histories of tier maps (not produced by the CUDA path).

Future missed mass is a ratio of sums of softmax weights. The kernel takes the scores from
fp32 tensor-core accumulation of 16-bit inputs (exact products), the weights from ex2.approx
(relative error about 2^-22) and sums up to 32K weights per lane group in fp32, so its
relative error is a few 1e-6; the bar is |gpu - oracle| <= 1e-6 + 1e-4 * oracle per unit.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from kv_cache_eviction_gqa_b200 import workloads as W

pytestmark = pytest.mark.gpu

RTOL, ATOL = 1e-4, 1e-6


def _tdt(dtype: str):
    return torch.bfloat16 if dtype == "bf16" else torch.float16


TIER_CASES = [
    W.DIAG_C2.scaled(name="tiers_c1", base=W.C1, n=2048 + 5, events=12),
    W.DIAG_C2.scaled(name="tiers_c5_small", base=W.C5.scaled(B=1, Hkv=3, full_windows=9, int2_windows=20),
                     n=64 * 70, events=20, extra_windows=0),
    W.DIAG_C2,
]


@pytest.mark.parametrize("cfg", TIER_CASES, ids=[c.name for c in TIER_CASES])
def test_tier_diagnostics_match_oracle(cfg):
    from kv_cache_eviction_gqa_b200.binding import TierDiagnostics
    hist = W.draw_tier_history(cfg)
    ref = O.tier_diagnostics(list(hist))
    d = TierDiagnostics(cfg.base.units, cfg.W, "cuda")
    for e in range(cfg.events):
        d.update(torch.from_numpy(hist[e]).cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(d.counters.cpu().numpy(), ref["per_unit"])
    s = d.summary()
    assert s["churn"] == ref["churn"] and (s["lir"] == ref["lir"] or np.isnan(ref["lir"]))
    print(cfg.name, "churn", s["churn"], "lir", s["lir"])


def test_tier_diagnostics_golden_sequence(golden_dir):
    """The hand-worked sequence of the oracle pin, run through the kernel."""
    import os
    from kv_cache_eviction_gqa_b200.binding import TierDiagnostics
    letter = {"E": W.TIER_EVICTED, "Q": W.TIER_INT2, "F": W.TIER_FULL, "T": W.TIER_TAIL}
    units, counts = {}, {}
    for line in open(os.path.join(golden_dir, "diag_tiers.txt")):
        if line.startswith("#") or "|" not in line:
            continue
        key, val = (x.strip() for x in line.split("|"))
        if key.startswith("unit"):
            units[int(key.split()[1])] = [[letter[c] for c in ev] for ev in val.split()]
        elif key.startswith("counts"):
            counts[int(key.split()[1])] = [int(x) for x in val.split()]
    Wn = max(len(units[u][0]) for u in units)
    maps = np.zeros((len(units[0]), len(units), Wn), dtype=np.uint8)  # missing windows: EVICTED
    for u in units:
        for e, ev in enumerate(units[u]):
            maps[e, u, :len(ev)] = ev
    d = TierDiagnostics(len(units), Wn, "cuda")
    for e in range(maps.shape[0]):
        d.update(torch.from_numpy(maps[e]).cuda())
    got = d.counters.cpu().numpy()
    for u in units:
        assert got[u].tolist() == counts[u]


def _fmm_case(cfg: W.DiagConfig, tiers=None):
    from kv_cache_eviction_gqa_b200.binding import diag_fmm, trim_status
    b = cfg.base
    t = _tdt(b.dtype)
    q = W.draw_diag_queries(cfg)
    if tiers is None:
        tiers = W.draw_tier_history(cfg)[-1]
    K = torch.zeros((b.B, b.Hkv, cfg.n_stride, b.D), dtype=t)
    Ks = {}
    for bb in range(b.B):
        for h in range(b.Hkv):
            Ks[bb, h] = W.draw_ghost_keys(cfg, bb, h) if cfg.n else np.zeros((0, b.D), np.float32)
            K[bb, h, :cfg.n] = torch.from_numpy(Ks[bb, h])
    fmm, scratch = diag_fmm(torch.from_numpy(q).to("cuda", t), K.cuda(), cfg.n,
                            torch.from_numpy(np.ascontiguousarray(tiers)).cuda(), b.window)
    torch.cuda.synchronize()
    assert trim_status(scratch) == (0, 0)
    return q, Ks, tiers, fmm.cpu().numpy()


def _check_unit(cfg, q, Ks, tiers, got, bb, h):
    G = cfg.base.G
    ref = O.future_missed_mass(q[bb, h * G:(h + 1) * G], Ks[bb, h], tiers[bb * cfg.base.Hkv + h],
                               cfg.base.window)
    u = bb * cfg.base.Hkv + h
    assert abs(got[u] - ref) <= ATOL + RTOL * ref, f"unit {u}: {got[u]} vs {ref}"
    return ref


FMM_CASES = [
    W.DIAG_C2.scaled(name="fmm_c1_fp16_d64", base=W.C1, n=2048 + 5, events=12),
    W.DIAG_C2.scaled(name="fmm_g5_w64", base=W.C5.scaled(B=1, Hkv=2, Hq=10, full_windows=3, int2_windows=4),
                     n=700, events=6, n_pad=37),
    W.DIAG_C2.scaled(name="fmm_g1", base=W.C2.scaled(B=2, Hq=2, Hkv=2, full_windows=5, int2_windows=6),
                     n=1000, events=9),
    W.DIAG_C2.scaled(name="fmm_g2_fp16", base=W.C2.scaled(B=1, Hq=4, Hkv=2, dtype="fp16", full_windows=4,
                                                         int2_windows=4), n=517, events=5),
    W.DIAG_C2.scaled(name="fmm_g8_d64", base=W.C1.scaled(Hq=16, Hkv=2, full_windows=8, int2_windows=8),
                     n=999, events=7),
    W.DIAG_C2.scaled(name="fmm_tiny_n7", base=W.C1.scaled(full_windows=1, int2_windows=1), n=7, events=1),
    W.DIAG_C2.scaled(name="fmm_one_tile", base=W.C1.scaled(full_windows=1, int2_windows=0), n=48, events=3),
    # windows that are not a multiple of the 16-key tile: tiles that straddle two windows
    W.DIAG_C2.scaled(name="fmm_window24", base=W.C1.scaled(window=24, full_windows=6, int2_windows=10),
                     n=1001, events=5),
    # windows shorter than a tile: one tier lookup per key
    W.DIAG_C2.scaled(name="fmm_window7", base=W.C1.scaled(window=7, full_windows=20, int2_windows=30),
                     n=500, events=4),
]


@pytest.mark.parametrize("cfg", FMM_CASES, ids=[c.name for c in FMM_CASES])
def test_fmm_matches_oracle(cfg):
    q, Ks, tiers, got = _fmm_case(cfg)
    vals = [_check_unit(cfg, q, Ks, tiers, got, bb, h) for bb in range(cfg.base.B) for h in range(cfg.base.Hkv)]
    print(cfg.name, "fmm", np.round(vals, 5).tolist())


@pytest.mark.parametrize("case", ["none_evicted", "all_evicted", "empty"])
def test_fmm_edges(case):
    base = W.C2.scaled(B=1, Hq=8, Hkv=2, full_windows=4, int2_windows=4)
    cfg = W.DIAG_C2.scaled(name=case, base=base, n=0 if case == "empty" else 333, events=3, n_pad=16)
    U, Wn = base.units, cfg.W
    if case == "none_evicted":
        tiers = np.full((U, Wn), W.TIER_FULL, np.uint8)
    elif case == "all_evicted":
        tiers = np.full((U, Wn), W.TIER_EVICTED, np.uint8)
    else:
        tiers = np.zeros((U, Wn), np.uint8)
    q, Ks, tiers, got = _fmm_case(cfg, tiers)
    want = {"none_evicted": 0.0, "all_evicted": 1.0, "empty": 0.0}[case]
    assert np.all(np.abs(got - want) <= 1e-6), got
    if cfg.n:
        for h in range(base.Hkv):
            _check_unit(cfg, q, Ks, tiers, got, 0, h)


def test_fmm_host_errors():
    from kv_cache_eviction_gqa_b200 import binding as B
    q = torch.zeros((1, 8, 128), dtype=torch.bfloat16, device="cuda")
    K = torch.zeros((1, 2, 64, 128), dtype=torch.bfloat16, device="cuda")
    tiers = torch.zeros((2, 2), dtype=torch.uint8, device="cuda")
    with pytest.raises(RuntimeError, match="invalid"):
        B.diag_fmm(q, K, 64, tiers, 16)          # 4 windows do not fit a 2-window map
    with pytest.raises(RuntimeError, match="invalid"):
        B.diag_fmm(q, K, 65, tiers, 64)          # n above the ghost cache's rows
    small = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(RuntimeError, match="workspace"):
        B.diag_fmm(q, K, 64, tiers, 32, scratch=small)


@pytest.mark.slow
def test_fmm_full_c2_sampled_units():
    cfg = W.DIAG_C2
    q, Ks, tiers, got = _fmm_case(cfg)
    assert np.all((got >= 0) & (got <= 1))
    vals = [_check_unit(cfg, q, Ks, tiers, got, bb, h) for (bb, h) in [(0, 0), (3, 5), (7, 7)]]
    print("c2 fmm sampled", vals, "mean over units", float(got.mean()))


ROUTED = [
    W.C1,
    W.C5.scaled(name="c5_small", B=1, Hkv=2, Hq=10, ctx=3000, full_windows=5, int2_windows=20,
                route_every=8, steps=70, hidden=1280),
]


@pytest.mark.parametrize("cfg", ROUTED, ids=[c.name for c in ROUTED])
def test_diagnostics_over_a_routed_decode_run(cfg):
    """The diagnostics fed by a context's own routing history (oracle: by its own history)."""
    from tests.parity_helpers import run_decode_parity
    rep = run_decode_parity(cfg, diag=True)
    assert rep.route_events > 0 and rep.max_fmm > 0
    print(cfg.name, rep.diag, "max fmm", rep.max_fmm, "near-ties", rep.near_ties)
