"""Lock-step comparison of the CUDA decode path with the CPU oracle.

Both sides take the same seeded inputs (kv_cache_eviction_gqa_b200.workloads). After
every decode step the checked units are compared:

* attention output: max |o_gpu - o_ref| / max |o_ref| per (batch, query head) <= 2e-3;
* cumulative window mass and perturbation: |d| / max(|ref|, 1e-30) <= 1e-4 per window
  (the tail window's perturbation is folded in when it completes, so it is compared then);
* routing: per-event counters (promotions, first and reused demotions, evictions, tier sizes,
  stage-1 share of the mass) equal those of the oracle's transitions;
* routing: tier decisions must match, except items whose score lies within 1e-4 relative
  of a selection boundary (near-ties: counted and reported). When every mismatch is a
  near-tie the oracle adopts the GPU's tiers for those windows so histories stay aligned;
  the GPU's decision is also checked to be exactly the two-stage selection of its own
  scores (a property of the selection, independent of the oracle);
* INT2 ledger codes and fp16 scale/zero of every newly demoted window: bit-exact;
* promoted pages: bit-exact dequant(ledger) in the cache dtype.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

import oracle as O
from kv_cache_eviction_gqa_b200 import workloads as W
from kv_cache_eviction_gqa_b200.binding import (TIER_EVICTED, TIER_FULL, TIER_INT2, TIER_TAIL,
                                                ContextShape, QEvictContext)

OUT_TOL = 2e-3
SCORE_TOL = 1e-4
TIE_TOL = 1e-4


def torch_dtype(name):
    return torch.bfloat16 if name == "bf16" else torch.float16


@dataclass
class ParityReport:
    steps: int = 0
    max_out_err: float = 0.0
    stats_checked: int = 0
    max_mass_err: float = 0.0
    max_pert_err: float = 0.0
    route_events: int = 0
    route_mismatch: int = 0
    near_ties: int = 0
    codes_checked: int = 0
    promoted_checked: int = 0
    max_fmm: float = 0.0
    diag: dict = field(default_factory=dict)
    notes: list = field(default_factory=list)


def _select_two_stage(ids, k1, k2, b, b1):
    """Independent restatement for the property check (lexsort on score desc, id asc)."""
    ids = np.asarray(ids)
    if ids.size <= b:
        return set(ids.tolist())
    o1 = np.lexsort((ids, -k1[ids]))
    s1 = ids[o1[:b1]]
    rest = np.setdiff1d(ids, s1)
    o2 = np.lexsort((rest, -k2[rest]))
    return set(s1.tolist()) | set(rest[o2[:b - b1]].tolist())


def _near_tie(unit: O.QEvictUnit, w: int) -> bool:
    """Is window w within TIE_TOL of any of the four selection boundaries of the last route?"""
    r = unit.last_route
    L = r["L"]
    mass, pert = unit.mass, unit.pert
    full = np.concatenate(r["full"])
    rest = np.setdiff1d(L, full)
    checks = [(L, mass, int(math.floor(unit.alpha * unit.F))),
              (np.setdiff1d(L, r["full"][0]), pert, unit.F - int(math.floor(unit.alpha * unit.F))),
              (rest, mass, int(math.floor(unit.alpha * unit.Q))),
              (np.setdiff1d(rest, r["int2"][0]), pert, unit.Q - int(math.floor(unit.alpha * unit.Q)))]
    for ids, key, k in checks:
        if ids.size == 0 or k <= 0 or k >= ids.size:
            continue
        srt = np.sort(key[ids])[::-1]
        for bnd in (srt[k - 1], srt[k]):
            if abs(key[w] - bnd) <= TIE_TOL * max(abs(bnd), 1e-30):
                return True
    return False


def run_decode_parity(cfg: W.DecodeConfig, check_units=None, steps=None, max_splits=32,
                      check_every=1, verbose=False, diag=False, fused=False) -> ParityReport:
    """Decode sequence on the GPU and in the oracle, compared step by step.

    With fused=True every step is one qe_decode_step call (the step's append inside the decode
    launch, routing on s % R == 0 in the same call): the call the bench times. The routing
    checks then take the candidates and the tiers before the event from the oracle's unit
    (the two sides' tiers agree before every event, which the previous event's checks assert).

    With diag=True the QEvict diagnostics ride along: after every routing event the context's
    tier map goes to qe_diag_tiers (the oracle's own tier history to tier_diagnostics, counts
    compared exactly at the end), and at every step qe_diag_fmm over a ghost cache of the
    seeded keys, with the tier map in force during that step's attention, is compared with
    future_missed_mass.
    """
    dev = "cuda"
    tdt = torch_dtype(cfg.dtype)
    steps = cfg.steps if steps is None else steps
    all_units = [(b, h) for b in range(cfg.B) for h in range(cfg.Hkv)]
    if check_units is None:
        check_units = list(range(len(all_units)))
    inp = W.draw_decode_inputs(cfg)
    K = torch.from_numpy(inp.K).view(cfg.B, cfg.Hkv, cfg.ctx, cfg.D).to(dev, tdt)
    V = torch.from_numpy(inp.V).view(cfg.B, cfg.Hkv, cfg.ctx, cfg.D).to(dev, tdt)
    W_O = torch.from_numpy(inp.W_O).to(dev, tdt)
    max_ctx = cfg.ctx + steps
    shape = ContextShape(cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.window, cfg.full_windows,
                         cfg.int2_windows, cfg.route_every, cfg.hidden, max_ctx, cfg.alpha,
                         max_splits=max_splits)
    ctx = QEvictContext(shape, W_O)
    ctx.load_prefill(K, V)
    G = cfg.G
    units = {}
    for u in check_units:
        b, h = all_units[u]
        units[u] = O.QEvictUnit(inp.K[u], inp.V[u], inp.W_O, h, G, cfg.window, cfg.full_windows,
                                cfg.int2_windows, cfg.alpha, cfg.dtype, max_ctx)
    rep = ParityReport()
    st = ctx.state()
    if diag:
        from kv_cache_eviction_gqa_b200.binding import TierDiagnostics, diag_fmm, trim_status
        Wn = st["win_tier"].shape[1]
        tdiag = TierDiagnostics(len(all_units), Wn, dev)
        tdiag.update(st["win_tier"])
        o_hist = {u: [unit.tier.copy()] for u, unit in units.items()}
        ghost = torch.zeros((cfg.B, cfg.Hkv, max_ctx, cfg.D), dtype=tdt, device=dev)
        ghost[:, :, :cfg.ctx] = K
        ghost_np = {u: np.concatenate([inp.K[u], np.zeros((steps, cfg.D), np.float32)]) for u in units}
    b1F = int(math.floor(cfg.alpha * cfg.full_windows))
    b1Q = int(math.floor(cfg.alpha * cfg.int2_windows))
    for s in range(steps):
        q = torch.from_numpy(inp.q[s]).to(dev, tdt)
        k = torch.from_numpy(inp.k_new[s]).to(dev, tdt)
        v = torch.from_numpy(inp.v_new[s]).to(dev, tdt)
        # scores before routing, for the selection-property check
        routing = s % cfg.route_every == 0
        if fused:
            out = ctx.decode_step(q, k, v)
        else:
            ctx.kv_append(k, v)
            out = ctx.decode_attend_and_score(q)
        if diag:
            ghost[:, :, cfg.ctx + s] = k
            fmm_g, fscr = diag_fmm(q, ghost, cfg.ctx + s + 1, st["win_tier"], cfg.window)
        torch.cuda.synchronize()
        if diag:
            assert trim_status(fscr) == (0, 0)
            fmm_g = fmm_g.cpu().numpy()
        g_mass = st["mass"].cpu().numpy().copy()
        g_pert = st["pert"].cpu().numpy().copy()
        g_tier_before = st["win_tier"].cpu().numpy().copy()
        if routing and not fused:
            ctx.route_windows()
        torch.cuda.synchronize()
        rc, det = ctx.status()
        assert rc == 0, f"device status {rc} detail {det} at step {s}"
        o_gpu = out.cpu().numpy()
        g_tier = st["win_tier"].cpu().numpy()
        for u, unit in units.items():
            b, h = all_units[u]
            unit.append(inp.k_new[s, b, h].astype(np.float64), inp.v_new[s, b, h].astype(np.float64))
            o_ref, _ = unit.attend_and_score(inp.q[s, b, h * G:(h + 1) * G].astype(np.float64))
            for j in range(G):
                og = o_gpu[b, h * G + j]
                err = np.abs(og - o_ref[j]).max() / np.abs(o_ref[j]).max()
                rep.max_out_err = max(rep.max_out_err, err)
                assert err <= OUT_TOL, f"step {s} unit {u} head {j}: output rel err {err:.3e}"
            if diag:
                ghost_np[u][cfg.ctx + s] = inp.k_new[s, b, h]
                ref = O.future_missed_mass(inp.q[s, b, h * G:(h + 1) * G], ghost_np[u][:cfg.ctx + s + 1],
                                           unit.tier, cfg.window)
                assert abs(fmm_g[u] - ref) <= 1e-6 + 1e-4 * ref, f"step {s} unit {u}: fmm {fmm_g[u]} vs {ref}"
                rep.max_fmm = max(rep.max_fmm, ref)
            if s % check_every == 0 or routing:
                live = np.nonzero(unit.tier != O.EVICTED)[0]
                tail = unit.n // cfg.window if unit.n % cfg.window else -1
                rm = np.abs(g_mass[u, live] - unit.mass[live]) / np.maximum(np.abs(unit.mass[live]), 1e-30)
                rep.max_mass_err = max(rep.max_mass_err, rm.max())
                assert rm.max() <= SCORE_TOL, f"step {s} unit {u}: mass rel err {rm.max():.3e} " \
                    f"at window {live[rm.argmax()]}"
                lp = live[live != tail]
                rp = np.abs(g_pert[u, lp] - unit.pert[lp]) / np.maximum(np.abs(unit.pert[lp]), 1e-30)
                if rp.size:
                    rep.max_pert_err = max(rep.max_pert_err, rp.max())
                    assert rp.max() <= SCORE_TOL, f"step {s} unit {u}: pert rel err {rp.max():.3e} " \
                        f"at window {lp[rp.argmax()]}"
            if routing:
                rep.route_events += 1
                if fused:
                    # tiers before the event, as the oracle holds them (routing already ran on the GPU)
                    tb = np.where(unit.tier == O.FULL, TIER_FULL, np.where(unit.tier == O.INT2, TIER_INT2,
                                  np.where(unit.tier == O.TAIL, TIER_TAIL, TIER_EVICTED)))
                    g_tier_before[u, :tb.size] = tb
                cands = np.nonzero((g_tier_before[u] == TIER_FULL) | (g_tier_before[u] == TIER_INT2))[0]
                # property: the GPU decision is the two-stage selection of its own scores
                full_g = _select_two_stage(cands, g_mass[u].astype(np.float64),
                                           g_pert[u].astype(np.float64), cfg.full_windows, b1F)
                rest = np.array(sorted(set(cands.tolist()) - full_g), dtype=np.int64)
                int2_g = _select_two_stage(rest, g_mass[u].astype(np.float64),
                                           g_pert[u].astype(np.float64), cfg.int2_windows, b1Q)
                got_full = set(np.nonzero(g_tier[u] == TIER_FULL)[0].tolist())
                got_int2 = set(np.nonzero(g_tier[u] == TIER_INT2)[0].tolist())
                assert got_full == full_g, f"step {s} unit {u}: full tier is not the two-stage pick"
                assert got_int2 == int2_g, f"step {s} unit {u}: INT2 tier is not the two-stage pick"
                ledger_before = set(unit.ledger.keys())
                tier_o_before = unit.tier.copy()
                new = unit.route()
                mism = [w for w, t in new.items() if int(g_tier[u, w]) != t]
                if mism:
                    ties = [w for w in mism if _near_tie(unit, w)]
                    rep.route_mismatch += len(mism)
                    rep.near_ties += len(ties)
                    assert len(ties) == len(mism), (
                        f"step {s} unit {u}: routing mismatch on windows "
                        f"{sorted(set(mism) - set(ties))} not near a selection boundary")
                    # replay: adopt the GPU's tiers for the near-tie windows
                    unit.apply({w: int(g_tier[u, w]) for w in mism})
                # INT2 codes of windows quantised at this event: bit-exact
                for w in sorted(set(unit.ledger.keys()) - ledger_before):
                    e = ctx.ledger_entry(u, w)
                    assert e is not None, f"unit {u} window {w}: no ledger slot on the GPU"
                    (ck, sk, zk), (cv, sv, zv) = unit.ledger[w]
                    gk, gsk, gzk, gv, gsv, gzv = e
                    for a_, b_, nm in ((gk, ck, "K codes"), (gv, cv, "V codes")):
                        np.testing.assert_array_equal(a_, b_, err_msg=f"unit {u} win {w} {nm}")
                    for a_, b_, nm in ((gsk, sk, "K scale"), (gzk, zk, "K zero"), (gsv, sv, "V scale"),
                                       (gzv, zv, "V zero")):
                        np.testing.assert_array_equal(a_.view(np.uint16), b_.view(np.uint16),
                                                      err_msg=f"unit {u} win {w} {nm}")
                    rep.codes_checked += 1
                # promoted windows: their pages hold dequant(ledger) in the cache dtype
                promoted = [w for w, t in new.items() if t == O.FULL and g_tier_before[u, w] == TIER_INT2]
                if promoted:
                    pages = st["pages"][u].float().cpu().numpy()
                    wp = st["win_pages"][u].cpu().numpy()
                    for w in promoted:
                        for t in range(cfg.window):
                            pg = wp[w, t // 16]
                            np.testing.assert_array_equal(pages[pg, 0, t % 16], unit.Kst[w * cfg.window + t])
                            np.testing.assert_array_equal(pages[pg, 1, t % 16], unit.Vst[w * cfg.window + t])
                        rep.promoted_checked += 1
                if diag:
                    o_hist[u].append(unit.tier.copy())
                # the event's counters (qe_route_windows' per-unit route_stats) against the
                # oracle's transitions: promotions, first demotions, demotions that reuse a
                # ledger entry, evictions, tier sizes, and the stage-1 share of the candidates'
                # mass (x 1e6) when the selection had no near-tie
                rs = st["route_stats"][u].cpu().numpy()
                ob, oa = tier_o_before, unit.tier
                live_b = (ob == O.FULL) | (ob == O.INT2)
                demoted = np.nonzero((ob == O.FULL) & (oa == O.INT2))[0]
                exp_stats = {
                    "promoted": int(np.sum((ob == O.INT2) & (oa == O.FULL))),
                    "first demotions": int(sum(1 for w in demoted if int(w) not in ledger_before)),
                    "reused demotions": int(sum(1 for w in demoted if int(w) in ledger_before)),
                    "evicted": int(np.sum(live_b & (oa == O.EVICTED))),
                    "full windows": int(np.sum(oa == O.FULL)),
                    "int2 windows": int(np.sum(oa == O.INT2)),
                }
                got_stats = dict(zip(exp_stats, (int(rs[0]), int(rs[1]), int(rs[2]), int(rs[3]), int(rs[4]),
                                                 int(rs[5]))))
                assert got_stats == exp_stats, f"step {s} unit {u}: route_stats {got_stats} vs {exp_stats}"
                if not mism:
                    L_ = unit.last_route["L"]
                    f1_ = unit.last_route["full"][0]
                    tot = float(np.sum(unit.mass[L_]))
                    share = round(1e6 * float(np.sum(unit.mass[f1_])) / tot) if tot > 0 else 0
                    # float32 sums of masses that match the oracle's to ~1e-6 relative
                    assert abs(int(rs[7]) - share) <= 2 + 1e-5 * share, \
                        f"step {s} unit {u}: stage-1 share {rs[7]} vs {share}"
                rep.stats_checked += 1
                # tiers agree after replay
                live_o = {int(w): int(unit.tier[w]) for w in np.nonzero(unit.tier != O.EVICTED)[0]}
                for w, t in live_o.items():
                    gt = int(g_tier[u, w])
                    assert gt == t or (t in (O.TAIL, O.FULL) and gt in (TIER_TAIL, TIER_FULL)), \
                        f"unit {u} window {w}: tier {gt} vs oracle {t}"
        if diag and routing:
            tdiag.update(st["win_tier"])
        ctx._steps_done = s + 1
        rep.steps += 1
        if verbose and (s % 8 == 0):
            print(f"step {s}: out {rep.max_out_err:.2e} mass {rep.max_mass_err:.2e} "
                  f"pert {rep.max_pert_err:.2e} ties {rep.near_ties}")
    if diag:
        got = tdiag.counters.cpu().numpy()
        for u in units:
            ref = O.tier_diagnostics(o_hist[u])["per_unit"][0]
            np.testing.assert_array_equal(got[u], ref, err_msg=f"unit {u}: tier diagnostics")
        rep.diag = tdiag.summary()
    return rep
