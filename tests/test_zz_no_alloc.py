"""The allocation-free decode entry point gives the same results as the regular one.

qe_decode_attend_and_score_noalloc serves callers that may not hand the library any device
memory beyond their inputs and outputs while a step runs (for instance an engine that
gives a plugin only its buffers). It keeps the decode kernel's per-call scratch in a fixed
array inside the library. This test drives two identical contexts, one through each entry
point, for two decode calls in a row and compares outputs and cumulative window scores
with the tolerances the other parity tests use. It lives in its own file so that pytest
collects it last.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from kv_cache_eviction_gqa_b200 import workloads as W

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3
SCORE_TOL = 1e-4


def test_noalloc_matches_regular_entry_point():
    from kv_cache_eviction_gqa_b200 import binding as Bd

    cfg = W.C2.scaled(name="noalloc", B=2, Hkv=2, Hq=8, ctx=700, full_windows=6, int2_windows=10,
                      route_every=4, steps=3, hidden=512)
    inp = W.draw_decode_inputs(cfg)
    tdt = torch.bfloat16
    K = torch.from_numpy(inp.K).view(cfg.B, cfg.Hkv, cfg.ctx, cfg.D).to("cuda", tdt)
    V = torch.from_numpy(inp.V).view(cfg.B, cfg.Hkv, cfg.ctx, cfg.D).to("cuda", tdt)
    Wo = torch.from_numpy(inp.W_O).to("cuda", tdt)
    shape = Bd.ContextShape(cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.window, cfg.full_windows,
                            cfg.int2_windows, cfg.route_every, cfg.hidden, cfg.ctx + cfg.steps)
    regular, noalloc = Bd.QEvictContext(shape, Wo), Bd.QEvictContext(shape, Wo)
    for ctx in (regular, noalloc):
        ctx.load_prefill(K, V)
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    for s in range(cfg.steps):
        q = torch.from_numpy(inp.q[s]).to("cuda", tdt)
        k = torch.from_numpy(inp.k_new[s]).to("cuda", tdt)
        v = torch.from_numpy(inp.v_new[s]).to("cuda", tdt)
        for ctx in (regular, noalloc):
            ctx.kv_append(k, v)
        out_r = regular.decode_attend_and_score(q)
        out_n = torch.empty_like(out_r)
        rc = Bd.lib().qe_decode_attend_and_score_noalloc(noalloc._h, C.c_void_p(q.data_ptr()),
                                                         C.c_void_p(out_n.data_ptr()), stream)
        assert rc == 0, Bd.strerror(rc)
        if s == 0:  # create INT2 windows so later calls read both tiers
            regular.route_windows()
            noalloc.route_windows()
        torch.cuda.synchronize()
        assert regular.status()[0] == 0 and noalloc.status()[0] == 0
        a, b = out_r.cpu().numpy(), out_n.cpu().numpy()
        err = (np.abs(a - b).max(axis=-1) / np.abs(a).max(axis=-1)).max()
        assert err <= OUT_TOL, f"call {s}: output rel err {err:.3e}"
        for key in ("mass", "pert"):
            x = regular.state()[key].cpu().numpy()
            y = noalloc.state()[key].cpu().numpy()
            rel = np.abs(x - y) / np.maximum(np.abs(x), 1e-30)
            assert rel.max() <= SCORE_TOL, f"call {s}: {key} rel err {rel.max():.3e}"
    n_full, n_int2 = C.c_int(), C.c_int()
    Bd.lib().qe_list_counts(noalloc._h, C.byref(n_full), C.byref(n_int2))
    assert n_int2.value > 0
