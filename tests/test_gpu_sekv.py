"""SEKV mixed-resolution attention on the GPU against the oracle ("Resumo Técnico: SEKV",
Metodologia 1-3).

Segmentation (anchors, span bounds, counts) is integer work decided by float32 comparisons of
the same float32 surprisal on both sides: bit-exact. Span summaries are float32 sums on the GPU
against float64 in the oracle: |delta| <= 1e-5 x the largest |value| of the row. The expansion
of a span is decided by comparing a float32 score with theta: the GPU's decisions must equal
the oracle's except where the oracle's score lies within 1e-4 of theta (near-ties, counted);
the oracle then attends with the GPU's decisions, and the outputs must agree to the decode
tolerance, max |delta o| / max |o| <= 2e-3 per head.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle as O
from kv_cache_eviction_gqa_b200 import workloads as W

pytestmark = pytest.mark.gpu

OUT_TOL, SUM_TOL, GATE_TOL = 2e-3, 1e-5, 1e-4


def _tdt(dtype):
    return torch.bfloat16 if dtype == "bf16" else torch.float16


def run_case(base, n, tau, theta_mode):
    from kv_cache_eviction_gqa_b200 import binding as Bd
    t = _tdt(base.dtype)
    cfg = base.scaled(ctx=n)
    B, Hq, Hkv, D, G = cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.G
    Ks, Vs = {}, {}
    for b in range(B):
        for h in range(Hkv):
            Ks[b, h], Vs[b, h] = W.draw_unit_cache(cfg, b, h)
    H = W.draw_surprisal(cfg, n)
    q = W.draw_step_inputs(cfg.scaled(steps=1))[0][0]
    K = torch.stack([torch.from_numpy(Ks[b, h]) for b in range(B) for h in range(Hkv)]).view(B, Hkv, n, D)
    V = torch.stack([torch.from_numpy(Vs[b, h]) for b in range(B) for h in range(Hkv)]).view(B, Hkv, n, D)
    K, V = K.to("cuda", t), V.to("cuda", t)
    Hd = torch.from_numpy(H).cuda()
    state = Bd.sekv_build(K, V, Hd, tau, Hq)
    views = Bd.sekv_views(state, B, Hq, Hkv, n, D)
    torch.cuda.synchronize()
    counts = views["counts"].cpu().numpy()
    ref = {}
    for b in range(B):
        anchors, spans = O.sekv_segment(H[b], tau)
        assert counts[b].tolist() == [len(anchors), len(spans)], f"b {b}: counts"
        np.testing.assert_array_equal(views["anchor_pos"][b, :len(anchors)].cpu().numpy(), anchors)
        np.testing.assert_array_equal(views["span_start"][b, :len(spans)].cpu().numpy(), [s for s, _ in spans])
        np.testing.assert_array_equal(views["span_end"][b, :len(spans)].cpu().numpy(), [e for _, e in spans])
        for h in range(Hkv):
            kb, vb, _ = O.sekv_summaries(Ks[b, h], Vs[b, h], H[b], spans)
            for name, refv in (("kbar", kb), ("vbar", vb)):
                got = views[name][b, h, :len(spans)].cpu().numpy()
                scale = np.maximum(np.abs(refv).max(axis=1, keepdims=True), 1e-30)
                err = (np.abs(got - refv) / scale).max() if len(spans) else 0.0
                assert err <= SUM_TOL, f"b {b} kvh {h}: {name} err {err:.2e}"
            ref[b, h] = (spans, kb)
    # theta: a fixed value, or the 90th percentile of the oracle's gates (about 10 % expanded)
    if theta_mode == "q90":
        gates = [O.sekv_gates(q[b, h * G:(h + 1) * G], ref[b, h][1])
                 for b in range(B) for h in range(Hkv) if len(ref[b, h][1])]
        theta = float(np.quantile(np.concatenate(gates), 0.9)) if gates else 0.0
    else:
        theta = float(theta_mode)
    out = Bd.sekv_attend(torch.from_numpy(q).to("cuda", t), K, V, theta, state)
    torch.cuda.synchronize()
    o_gpu = out.cpu().numpy()
    flags = views["expanded"].cpu().numpy()
    near, expanded = 0, 0
    for b in range(B):
        for h in range(Hkv):
            spans, kb = ref[b, h]
            qg = q[b, h * G:(h + 1) * G]
            g = O.sekv_gates(qg, kb)
            e_gpu = flags[b, h, :len(spans)].astype(bool)
            diff = np.nonzero(e_gpu != (g >= theta))[0]
            bad = [int(i) for i in diff if abs(g[i] - theta) > GATE_TOL * max(1.0, abs(theta))]
            assert not bad, f"b {b} kvh {h}: expansion differs away from theta on spans {bad[:5]}"
            near += len(diff)
            expanded += int(e_gpu.sum())
            o_ref, _ = O.sekv_attend(qg, Ks[b, h], Vs[b, h], H[b], tau, theta, expand=e_gpu)
            for j in range(G):
                err = np.abs(o_gpu[b, h * G + j] - o_ref[j]).max() / np.abs(o_ref[j]).max()
                assert err <= OUT_TOL, f"b {b} head {h * G + j}: output err {err:.2e}"
    return dict(anchors=int(counts[:, 0].sum()), spans=int(counts[:, 1].sum()), expanded=expanded, near=near,
                theta=theta)


CASES = [
    ("c1_fp16_d64", W.C1, 2053, W.SEKV_TAU, "q90"),
    ("g5_d128", W.C5.scaled(B=1, Hkv=2, Hq=10), 1500, W.SEKV_TAU, "q90"),
    ("g1_b2", W.C2.scaled(B=2, Hq=2, Hkv=2), 777, W.SEKV_TAU, "q90"),
    ("g8_d64", W.C1.scaled(Hq=16, Hkv=2), 999, 1.0, "q90"),
    ("g2_fp16_d128", W.C2.scaled(B=1, Hq=4, Hkv=2, dtype="fp16"), 640, W.SEKV_TAU, "q90"),
    # every token an anchor (surprisal >= 0): plain attention
    ("all_anchors", W.C2.scaled(B=1, Hq=4, Hkv=1), 300, 0.0, "q90"),
    # no anchor: one span over everything, summarised (theta = +inf) or expanded (theta = -inf)
    ("one_span_summary", W.C2.scaled(B=1, Hq=4, Hkv=1), 300, math.inf, "inf"),
    ("one_span_expanded", W.C2.scaled(B=1, Hq=4, Hkv=1), 300, math.inf, "-inf"),
    ("single_token", W.C1.scaled(B=1, Hkv=1, Hq=4), 1, W.SEKV_TAU, "q90"),
]


@pytest.mark.parametrize("name,base,n,tau,theta", CASES, ids=[c[0] for c in CASES])
def test_sekv_matches_oracle(name, base, n, tau, theta):
    rep = run_case(base, n, tau, theta)
    print(name, rep)


def test_sekv_host_errors():
    from kv_cache_eviction_gqa_b200 import binding as Bd
    K = torch.zeros((1, 1, 16, 96), dtype=torch.bfloat16, device="cuda")
    H = torch.zeros((1, 16), dtype=torch.float32, device="cuda")
    with pytest.raises(ValueError):
        Bd.sekv_build(K, K, H, 1.0, 4)  # D = 96 is not supported
    K = torch.zeros((1, 1, 16, 128), dtype=torch.bfloat16, device="cuda")
    small = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(RuntimeError, match="workspace"):
        Bd.sekv_build(K, K, H, 1.0, 4, state=small)


@pytest.mark.slow
def test_sekv_full_c2_sampled():
    rep = run_case(W.C2.scaled(B=2), 32768, W.SEKV_TAU, "q90")
    assert rep["expanded"] > 0 and rep["anchors"] > 0
    print("c2 32K, 2 sequences:", rep)
