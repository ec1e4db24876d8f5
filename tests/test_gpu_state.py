"""Checkpoint and restore of a decode context (qe_state_export / qe_state_import) and the pooled
tier diagnostics (qe_diag_summary).

The checkpoint carries the state "Resumo Técnico: QEvict" makes persistent - the write-once INT2
ledger (Hierarquia Recuperável) and the cumulative window scores (Pontuação Cumulativa) - with
the pages, tiers and counters around them. A context restored mid-sequence from a checkpoint must
continue exactly as the original does (bit for bit) and as the oracle does (the parity
tolerances), across routing events and window completions after the restore.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle as O
from kv_cache_eviction_gqa_b200 import workloads as W

pytestmark = pytest.mark.gpu

OUT_TOL, SCORE_TOL = 2e-3, 1e-4


@pytest.mark.parametrize("where", ["host", "device"])
def test_export_import_continues_like_the_original_and_the_oracle(where):
    from kv_cache_eviction_gqa_b200.binding import ContextShape, QEvictContext
    cfg = W.C2.scaled(name="state", B=2, Hkv=2, Hq=8, ctx=1000, full_windows=6, int2_windows=10,
                      route_every=4, steps=40, hidden=1024)
    cut = 18  # after routing events 0, 4, ..., 16, mid-window
    dev, t = "cuda", torch.bfloat16
    inp = W.draw_decode_inputs(cfg)
    K = torch.from_numpy(inp.K).view(cfg.B, cfg.Hkv, cfg.ctx, cfg.D).to(dev, t)
    V = torch.from_numpy(inp.V).view(cfg.B, cfg.Hkv, cfg.ctx, cfg.D).to(dev, t)
    Wo = torch.from_numpy(inp.W_O).to(dev, t)
    shape = ContextShape(cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.window, cfg.full_windows, cfg.int2_windows,
                         cfg.route_every, cfg.hidden, cfg.ctx + cfg.steps, cfg.alpha)
    a = QEvictContext(shape, Wo)
    a.load_prefill(K, V)
    u, (b, h) = 3, (1, 1)
    unit = O.QEvictUnit(inp.K[u], inp.V[u], inp.W_O, h, cfg.G, cfg.window, cfg.full_windows,
                        cfg.int2_windows, cfg.alpha, cfg.dtype, cfg.ctx + cfg.steps)
    G = cfg.G
    restored = None
    for s in range(cfg.steps):
        if s == cut:
            if where == "host":
                ck = torch.empty(a.state_bytes(), dtype=torch.uint8, pin_memory=True)
                a.export_state(ck)
            else:
                ck = a.export_state()
            torch.cuda.synchronize()
            restored = QEvictContext(shape, Wo)
            restored.import_state(ck)
            assert restored.step_index == a.step_index == cut and restored.length == a.length
        q = torch.from_numpy(inp.q[s]).to(dev, t)
        k = torch.from_numpy(inp.k_new[s]).to(dev, t)
        v = torch.from_numpy(inp.v_new[s]).to(dev, t)
        o1 = a.decode_step(q, k, v)
        o2 = restored.decode_step(q, k, v) if restored is not None else None
        o_ref, _ = unit.step(s, inp.q[s, b, h * G:(h + 1) * G].astype(np.float64),
                             inp.k_new[s, b, h].astype(np.float64), inp.v_new[s, b, h].astype(np.float64),
                             cfg.route_every)
        torch.cuda.synchronize()
        assert a.status() == (0, 0)
        if restored is None:
            continue
        assert restored.status() == (0, 0)
        assert torch.equal(o1, o2), f"step {s}: outputs differ after the restore"
        sa, sb = a.state(), restored.state()
        for name in sa:  # bitwise: free pages and slots hold whatever the allocator left (NaN too)
            assert torch.equal(sa[name].contiguous().view(torch.uint8), sb[name].contiguous().view(torch.uint8)), \
                f"step {s}: {name} differs after the restore"
        # the restored context against the oracle (routing on this unit matches: no near-ties)
        og = o2.cpu().numpy()[b, h * G:(h + 1) * G]
        err = (np.abs(og - o_ref).max(axis=-1) / np.abs(o_ref).max(axis=-1)).max()
        assert err <= OUT_TOL, f"step {s}: output rel err {err:.3e}"
        gm = sb["mass"][u].cpu().numpy()
        gt = sb["win_tier"][u].cpu().numpy()
        live = np.nonzero(unit.tier != O.EVICTED)[0]
        assert np.array_equal(np.where(unit.tier[live] == O.TAIL, 3, unit.tier[live]), gt[live]), f"step {s}: tiers"
        rm = np.abs(gm[live] - unit.mass[live]) / np.maximum(np.abs(unit.mass[live]), 1e-30)
        assert rm.max() <= SCORE_TOL, f"step {s}: mass rel err {rm.max():.3e}"


def test_diag_summary_pools_the_counters():
    from kv_cache_eviction_gqa_b200.binding import QeDiagStats, lib
    r = np.random.default_rng(7)
    cnt = r.integers(0, 1000, size=(37, 6)).astype(np.int64)
    cnt[:, 0] += 1000
    d = torch.from_numpy(cnt).cuda()
    st = QeDiagStats()
    assert lib().qe_diag_summary(C.c_void_p(d.data_ptr()), 37, C.byref(st), None) == 0
    tot = cnt.sum(axis=0)
    assert [st.live_prev, st.changed, st.exits, st.reentries, st.windows_exited, st.windows_reentered] == tot.tolist()
    assert st.churn == tot[1] / tot[0] and st.lir == tot[5] / tot[4]
    z = torch.zeros((3, 6), dtype=torch.int64, device="cuda")
    assert lib().qe_diag_summary(C.c_void_p(z.data_ptr()), 3, C.byref(st), None) == 0
    assert np.isnan(st.churn) and np.isnan(st.lir)
