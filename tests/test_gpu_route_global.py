"""Routing under budgets shared by every layer and kv head of a sequence, on the GPU against the
oracle ("Make Each Token Count", Metodologia 3: Orçamento Global, applied to the window tiers of
"Resumo Técnico: QEvict", Metodologia).

Several layers (one context each, different seeded caches) decode through qe_decode_step with
route_every = 0, and every R steps qe_route_windows_global routes all of them at once. Every
step: outputs and cumulative scores of every unit match the oracle (the decode tolerances).
Every event: each unit's tiers match oracle.route_global over the oracle's own units, except
windows whose score lies within 1e-4 relative of one of the four selection cuts (near-ties:
counted; the oracle then adopts the GPU's tiers so the histories stay aligned); INT2 codes of
windows quantised at the event are bit-exact.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle as O
from kv_cache_eviction_gqa_b200 import workloads as W

pytestmark = pytest.mark.gpu

OUT_TOL, SCORE_TOL, TIE_TOL = 2e-3, 1e-4, 1e-4


def _near_cut(info, j) -> bool:
    """Is flat candidate j within TIE_TOL of a cut of the last global selection (the lowest
    score each of the four stages took)?"""
    mass, pert = info["mass"], info["pert"]
    f1, f2 = info["full"]
    q1, q2 = info["int2"]
    pairs = [(score[j], score[picks[-1]]) for picks, score in ((f1, mass), (f2, pert), (q1, mass), (q2, pert))
             if len(picks)]
    return any(abs(a - c) <= TIE_TOL * max(abs(c), 1e-30) for a, c in pairs)


def run_global(cfgs, F_total, Q_total, steps, route_every, alpha=0.5):
    from kv_cache_eviction_gqa_b200.binding import ContextShape, QEvictContext, route_windows_global
    from tests.parity_helpers import torch_dtype
    c0 = cfgs[0]
    B, Hkv, G, w = c0.B, c0.Hkv, c0.G, c0.window
    tdt = torch_dtype(c0.dtype)
    max_ctx = c0.ctx + steps
    n_win = -(-max_ctx // w)
    ctxs, inps, units = [], [], {}
    for l, cfg in enumerate(cfgs):
        inp = W.draw_decode_inputs(cfg)
        inps.append(inp)
        K = torch.from_numpy(inp.K).view(B, Hkv, cfg.ctx, cfg.D).to("cuda", tdt)
        V = torch.from_numpy(inp.V).view(B, Hkv, cfg.ctx, cfg.D).to("cuda", tdt)
        Wo = torch.from_numpy(inp.W_O).to("cuda", tdt)
        shape = ContextShape(B, cfg.Hq, Hkv, cfg.D, w, cfg.full_windows, cfg.int2_windows, 0, cfg.hidden,
                             max_ctx, alpha, slots_per_unit=n_win)
        ctx = QEvictContext(shape, Wo)
        ctx.load_prefill(K, V)
        ctxs.append(ctx)
        for u in range(B * Hkv):
            units[l, u] = O.QEvictUnit(inp.K[u], inp.V[u], inp.W_O, u % Hkv, G, w, cfg.full_windows,
                                       cfg.int2_windows, alpha, cfg.dtype, max_ctx)
    states = [c.state() for c in ctxs]
    scratch = None
    rep = dict(events=0, near_ties=0, codes=0, max_out=0.0, max_mass=0.0)
    for s in range(steps):
        outs = []
        for l, (ctx, inp) in enumerate(zip(ctxs, inps)):
            q = torch.from_numpy(inp.q[s]).to("cuda", tdt)
            k = torch.from_numpy(inp.k_new[s]).to("cuda", tdt)
            v = torch.from_numpy(inp.v_new[s]).to("cuda", tdt)
            outs.append(ctx.decode_step(q, k, v))
        torch.cuda.synchronize()
        for l, inp in enumerate(inps):
            o_gpu = outs[l].cpu().numpy()
            g_mass = states[l]["mass"].cpu().numpy()
            for u in range(B * Hkv):
                b, h = divmod(u, Hkv)
                unit = units[l, u]
                unit.append(inp.k_new[s, b, h].astype(np.float64), inp.v_new[s, b, h].astype(np.float64))
                o_ref, _ = unit.attend_and_score(inp.q[s, b, h * G:(h + 1) * G].astype(np.float64))
                for j in range(G):
                    err = np.abs(o_gpu[b, h * G + j] - o_ref[j]).max() / np.abs(o_ref[j]).max()
                    rep["max_out"] = max(rep["max_out"], err)
                    assert err <= OUT_TOL, f"step {s} layer {l} unit {u}: output err {err:.2e}"
                live = np.nonzero(unit.tier != O.EVICTED)[0]
                rm = np.abs(g_mass[u, live] - unit.mass[live]) / np.maximum(np.abs(unit.mass[live]), 1e-30)
                rep["max_mass"] = max(rep["max_mass"], rm.max())
                assert rm.max() <= SCORE_TOL, f"step {s} layer {l} unit {u}: mass err {rm.max():.2e}"
        if s % route_every:
            continue
        scratch = route_windows_global(ctxs, F_total, Q_total, alpha, scratch)
        torch.cuda.synchronize()
        for l, ctx in enumerate(ctxs):
            assert ctx.status() == (0, 0), f"layer {l}: device status {ctx.status()}"
        rep["events"] += 1
        for b in range(B):
            group = [units[l, b * Hkv + h] for l in range(len(cfgs)) for h in range(Hkv)]
            ledgers = [set(u.ledger) for u in group]
            _, info = O.route_global(group, F_total, Q_total, alpha)
            for k, unit in enumerate(group):
                l, h = divmod(k, Hkv)
                g_tier = states[l]["win_tier"][b * Hkv + h].cpu().numpy()
                live = np.nonzero((unit.tier == O.FULL) | (unit.tier == O.INT2) |
                                  ((g_tier[:len(unit.tier)] == W.TIER_FULL) | (g_tier[:len(unit.tier)] == W.TIER_INT2)))[0]
                mism = [int(x) for x in live if int(g_tier[x]) != int(unit.tier[x])
                        and not (unit.tier[x] == O.TAIL and g_tier[x] in (W.TIER_TAIL, W.TIER_FULL))]
                if mism:
                    bad = [x for x in mism if not _near_cut(info, k * info["W"] + x)]
                    assert not bad, f"step {s} b {b} layer {l} kvh {h}: tiers differ on windows {bad}"
                    rep["near_ties"] += len(mism)
                    unit.apply({x: int(g_tier[x]) for x in mism})
                for x in sorted(set(unit.ledger) - ledgers[k]):
                    e = ctxs[l].ledger_entry(b * Hkv + h, x)
                    assert e is not None, f"layer {l} unit {b * Hkv + h} window {x}: no ledger slot"
                    (ck, _, _), (cv, _, _) = unit.ledger[x]
                    np.testing.assert_array_equal(e[0], ck)
                    np.testing.assert_array_equal(e[3], cv)
                    rep["codes"] += 1
    return rep


CASES = [
    ("bf16_3layers", [W.C2.scaled(name=f"g{l}", B=2, Hkv=2, Hq=8, ctx=1000, full_windows=6, int2_windows=10,
                                  steps=40, hidden=1024, seed=2100 + l) for l in range(3)], 30, 50, 40, 4),
    ("fp16_d64_2layers", [W.C1.scaled(name=f"h{l}", ctx=700, steps=30, seed=2200 + l) for l in range(2)],
     20, 30, 30, 5),
    ("g5_w64_2layers", [W.C5.scaled(name=f"k{l}", B=1, Hkv=2, Hq=10, ctx=2000, full_windows=5, int2_windows=8,
                                    steps=40, hidden=1280, seed=2300 + l) for l in range(2)], 12, 20, 40, 8),
]


@pytest.mark.parametrize("name,cfgs,F,Q,steps,R", CASES, ids=[c[0] for c in CASES])
def test_global_routing_matches_oracle(name, cfgs, F, Q, steps, R):
    rep = run_global(cfgs, F, Q, steps, R)
    assert rep["events"] == math.ceil(steps / R) and rep["codes"] > 0
    print(name, rep)


def test_global_budget_covering_everything_evicts_nothing():
    from kv_cache_eviction_gqa_b200.binding import ContextShape, QEvictContext, route_windows_global
    cfgs = [W.C1.scaled(name=f"e{l}", ctx=500, steps=1, seed=2400 + l) for l in range(2)]
    ctxs = []
    for cfg in cfgs:
        inp = W.draw_decode_inputs(cfg)
        K = torch.from_numpy(inp.K).view(cfg.B, cfg.Hkv, cfg.ctx, cfg.D).to("cuda", torch.float16)
        V = torch.from_numpy(inp.V).view(cfg.B, cfg.Hkv, cfg.ctx, cfg.D).to("cuda", torch.float16)
        Wo = torch.from_numpy(inp.W_O).to("cuda", torch.float16)
        shape = ContextShape(cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.window, 4, 4, 0, cfg.hidden, cfg.ctx + 1,
                             slots_per_unit=40)
        c = QEvictContext(shape, Wo)
        c.load_prefill(K, V)
        ctxs.append(c)
    route_windows_global(ctxs, 10_000, 0)
    torch.cuda.synchronize()
    for c in ctxs:
        t = c.state()["win_tier"].cpu().numpy()
        assert not (t[:, :cfgs[0].ctx // cfgs[0].window] == W.TIER_EVICTED).any()
    # mismatched contexts are refused on the host
    other = W.C1.scaled(B=1, Hkv=1, Hq=4, ctx=500)
    shape = ContextShape(1, 4, 1, 64, 16, 4, 4, 0, 512, 501)
    c3 = QEvictContext(shape, torch.zeros((4 * 64, 512), dtype=torch.float16, device="cuda"))
    c3.load_prefill(torch.zeros((1, 1, 500, 64), dtype=torch.float16, device="cuda"),
                    torch.zeros((1, 1, 500, 64), dtype=torch.float16, device="cuda"))
    with pytest.raises(RuntimeError, match="invalid"):
        route_windows_global([ctxs[0], c3], 4, 4)
    with pytest.raises(RuntimeError, match="invalid"):
        route_windows_global([ctxs[0], ctxs[0]], 4, 4)


def test_one_layer_one_kv_head_equals_per_unit_routing():
    """With one layer and one kv head per sequence the global candidates are exactly one unit's
    windows, so qe_route_windows_global must reproduce qe_route_windows tier for tier. Both
    contexts get the same prefill norms and no window completes during the run (the tail holds
    one token at the start), so every score is bit-identical."""
    from kv_cache_eviction_gqa_b200.binding import ContextShape, QEvictContext, route_windows_global, vwo_l1norm
    cfg = W.C2.scaled(name="one", B=3, Hkv=1, Hq=4, ctx=46 * 32 + 1, full_windows=7, int2_windows=12, steps=24,
                      hidden=512, seed=2500)
    inp = W.draw_decode_inputs(cfg)
    t = torch.bfloat16
    K = torch.from_numpy(inp.K).view(cfg.B, 1, cfg.ctx, cfg.D).to("cuda", t)
    V = torch.from_numpy(inp.V).view(cfg.B, 1, cfg.ctx, cfg.D).to("cuda", t)
    Wo = torch.from_numpy(inp.W_O).to("cuda", t)
    norms = vwo_l1norm(V.view(-1, cfg.ctx, cfg.D), Wo, cfg.Hq, 1).view(cfg.B, 1, cfg.ctx, cfg.G)
    ctxs = []
    for _ in range(2):
        shape = ContextShape(cfg.B, cfg.Hq, 1, cfg.D, cfg.window, cfg.full_windows, cfg.int2_windows, 0,
                             cfg.hidden, cfg.ctx + cfg.steps, slots_per_unit=80)
        c = QEvictContext(shape, Wo)
        c.workspace.zero_()
        c.load_prefill(K, V, norms)
        ctxs.append(c)
    local, glob = ctxs
    for s in range(cfg.steps):
        q = torch.from_numpy(inp.q[s]).to("cuda", t)
        k = torch.from_numpy(inp.k_new[s]).to("cuda", t)
        v = torch.from_numpy(inp.v_new[s]).to("cuda", t)
        o1, o2 = local.decode_step(q, k, v), glob.decode_step(q, k, v)
        if s % 4 == 0:
            local.route_windows()
            route_windows_global([glob], cfg.full_windows, cfg.int2_windows, cfg.alpha)
        torch.cuda.synchronize()
        assert local.status() == (0, 0) and glob.status() == (0, 0)
        assert torch.equal(o1, o2), f"step {s}: outputs differ"
        sl, sg = local.state(), glob.state()
        for name in ("win_tier", "win_slot", "mass", "pert", "stacks"):
            assert torch.equal(sl[name], sg[name]), f"step {s}: {name} differs"
