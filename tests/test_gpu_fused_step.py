"""qe_decode_step appends the step's token inside the decode launch. Its results must equal
those of the separate calls (qe_kv_append, qe_decode_attend_and_score, qe_route_windows),
whose parity with the oracle the decode tests establish: outputs and every state array after
every step, across routing events and window completions, bit for bit (the norms of windows
completed during the run included: every output element of the tensor-core norm GEMM is
written by one CTA, so they do not depend on scheduling)."""
from __future__ import annotations

import pytest
import torch

from kv_cache_eviction_gqa_b200 import workloads as W

pytestmark = pytest.mark.gpu

CASES = [
    W.C2.scaled(name="fused_c2_small", B=2, Hkv=2, Hq=8, ctx=1000, full_windows=6, int2_windows=10,
                route_every=4, steps=70, hidden=1024),
    W.C1.scaled(name="fused_c1", steps=40),
    W.C5.scaled(name="fused_g5_w64", B=1, Hkv=2, Hq=10, ctx=700, full_windows=3, int2_windows=6,
                route_every=5, steps=140, hidden=1280),
]


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_fused_step_matches_separate_calls(cfg):
    from kv_cache_eviction_gqa_b200.binding import ContextShape, QEvictContext
    from tests.parity_helpers import torch_dtype
    dev, t = "cuda", torch_dtype(cfg.dtype)
    inp = W.draw_decode_inputs(cfg)
    K = torch.from_numpy(inp.K).view(cfg.B, cfg.Hkv, cfg.ctx, cfg.D).to(dev, t)
    V = torch.from_numpy(inp.V).view(cfg.B, cfg.Hkv, cfg.ctx, cfg.D).to(dev, t)
    Wo = torch.from_numpy(inp.W_O).to(dev, t)
    shape = ContextShape(cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.window, cfg.full_windows, cfg.int2_windows,
                         cfg.route_every, cfg.hidden, cfg.ctx + cfg.steps, cfg.alpha)
    from kv_cache_eviction_gqa_b200.binding import vwo_l1norm
    norms = vwo_l1norm(V.view(-1, cfg.ctx, cfg.D), Wo, cfg.Hq, cfg.Hkv).view(cfg.B, cfg.Hkv, cfg.ctx, cfg.G)
    sep, fus = QEvictContext(shape, Wo), QEvictContext(shape, Wo)
    # free pages and ledger slots hold whatever the allocator left: start both from zeros so
    # that whole pools can be compared byte by byte
    sep.workspace.zero_()
    fus.workspace.zero_()
    sep.load_prefill(K, V, norms)
    fus.load_prefill(K, V, norms)
    ss, sf = sep.state(), fus.state()
    for s in range(cfg.steps):
        q = torch.from_numpy(inp.q[s]).to(dev, t)
        k = torch.from_numpy(inp.k_new[s]).to(dev, t)
        v = torch.from_numpy(inp.v_new[s]).to(dev, t)
        sep.kv_append(k, v)
        o1 = sep.decode_attend_and_score(q)
        if s % cfg.route_every == 0:
            sep.route_windows()
        o2 = fus.decode_step(q, k, v)
        torch.cuda.synchronize()
        assert sep.status() == (0, 0) and fus.status() == (0, 0)
        assert torch.equal(o1, o2), f"step {s}: outputs differ"
        for name in ss:
            assert torch.equal(ss[name], sf[name]), f"step {s}: state {name} differs"
    assert sep.length == fus.length == cfg.ctx + cfg.steps
