"""GPU parity of the decode hot path (attention + scoring + routing + ledger) with the oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from kv_cache_eviction_gqa_b200 import workloads as W

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from kv_cache_eviction_gqa_b200 import binding as Bd
    from tests.parity_helpers import run_decode_parity, torch_dtype


# tiny config of the pages' settings: fp16, GQA 4, D 64, 2K context, w 16, 25 % / 25 %
def test_c1_full_sequence_all_units():
    rep = run_decode_parity(W.C1)
    assert rep.steps == W.C1.steps and rep.route_events == 4 * W.C1.units and rep.codes_checked > 0
    print(rep)


# several tiles + ragged tails: prefill not a multiple of the page or window
SMALL = [
    W.C2.scaled(name="c2_small", B=2, Hkv=2, Hq=8, ctx=1000, full_windows=6, int2_windows=10,
                route_every=4, steps=40, hidden=1024),
    W.C5.scaled(name="c5_small", B=1, Hkv=2, Hq=10, ctx=3000, full_windows=5, int2_windows=20,
                route_every=8, steps=70, hidden=1280),
    W.C1.scaled(name="mha_small", Hq=2, Hkv=2, ctx=517, full_windows=4, int2_windows=4,
                route_every=3, steps=30, hidden=128, kind="plain"),
    W.C2.scaled(name="g2_bf16_d64", B=3, Hkv=1, Hq=2, D=64, ctx=700, window=64, full_windows=2,
                int2_windows=3, route_every=5, steps=60, hidden=128),
]


@pytest.mark.parametrize("cfg", SMALL, ids=[c.name for c in SMALL])
def test_small_sequences(cfg):
    rep = run_decode_parity(cfg)
    assert rep.steps == cfg.steps
    print(rep)


# full sizes, through the call and launch configuration the bench times (qe_decode_step: the
# append inside the decode launch, routing in the same call); the oracle follows sampled units
@pytest.mark.slow
def test_c2_full_size_sampled_units():
    """The benched call (qe_decode_step: append fused into the decode launch, routing every 16
    steps) at full c2 size, all 64 steps, on eight units spread over every batch row and kv head
    (unit 9k: batch k, kv head k mod 8)."""
    cfg = W.C2
    units = [9 * k for k in range(8) if 9 * k < cfg.units]
    rep = run_decode_parity(cfg, check_units=units, fused=True)
    assert rep.steps == cfg.steps and rep.route_events == 4 * len(units) and rep.codes_checked > 0
    print(rep)


@pytest.mark.slow
def test_c5_full_size_sampled_units():
    """All 256 drift steps of the long-context stress (16 routing events, 8 focus rotations that
    force repeated promotions and demotions through the write-once ledger) on two kv heads."""
    cfg = W.C5
    units = [3, 6]
    rep = run_decode_parity(cfg, check_units=units, fused=True)
    assert rep.steps == cfg.steps == 256 and rep.route_events == 16 * len(units)
    assert rep.codes_checked > 0 and rep.promoted_checked > 0
    print(rep)


@pytest.mark.parametrize("splits", [1, 3, 64])
def test_split_counts_agree(splits):
    cfg = SMALL[0].scaled(steps=9)
    rep = run_decode_parity(cfg, max_splits=splits)
    assert rep.steps == 9


def test_budget_covers_everything_is_plain_attention():
    cfg = W.C1.scaled(name="nobudget", ctx=256, full_windows=1000, int2_windows=0, steps=12)
    rep = run_decode_parity(cfg)
    assert rep.codes_checked == 0


def test_int2_quantizer_bit_exact():
    r = np.random.default_rng(5)
    for D, dt in ((128, "bf16"), (64, "fp16"), (128, "fp16")):
        x = W.to_dtype_values((r.standard_normal((1000, D)) * r.uniform(0.01, 10, (1000, 1))).astype(np.float32), dt)
        x[3] = 0.25  # constant row: scale 0
        xt = torch.from_numpy(x).to("cuda", torch_dtype(dt))
        codes, meta = Bd.int2_quantize(xt)
        ck, sk, zk = O.int2_quantize(x.astype(np.float64))
        c = codes.cpu().numpy()
        gc = np.stack([(c >> (2 * e)) & 3 for e in range(4)], -1).reshape(1000, D)
        np.testing.assert_array_equal(gc, ck)
        m = meta.cpu().numpy().view(np.uint32)
        np.testing.assert_array_equal((m & 0xFFFF).astype(np.uint16), sk.view(np.uint16))
        np.testing.assert_array_equal((m >> 16).astype(np.uint16), zk.view(np.uint16))


def test_vwo_l1norm_matches_oracle():
    r = np.random.default_rng(6)
    for (G, Hkv, D, hidden, rows, dt) in ((4, 2, 128, 512, 300, "bf16"), (5, 1, 128, 640, 129, "bf16"),
                                          (4, 2, 64, 512, 77, "fp16")):
        Hq = G * Hkv
        V = W.to_dtype_values(r.standard_normal((3, rows, D)).astype(np.float32), dt)
        Wo = W.to_dtype_values((r.standard_normal((Hq * D, hidden)) / np.sqrt(Hq * D)).astype(np.float32), dt)
        out = Bd.vwo_l1norm(torch.from_numpy(V).to("cuda", torch_dtype(dt)),
                            torch.from_numpy(Wo).to("cuda", torch_dtype(dt)), Hq, Hkv).cpu().numpy()
        for g in range(3):
            kvh = g % Hkv
            ref = O.vwo_l1norm(V[g], Wo, [kvh * G + j for j in range(G)], D)
            np.testing.assert_allclose(out[g], ref, rtol=1e-4)


def test_write_once_through_the_abi():
    """quantize_once -> promote -> quantize_once keeps the first ledger entry; the promoted
    pages hold dequant(codes) in the cache dtype."""
    cfg = W.C1.scaled(name="wo", ctx=128, full_windows=100, int2_windows=100, steps=0)
    inp = W.draw_decode_inputs(cfg)
    tdt = torch.float16
    K = torch.from_numpy(inp.K).view(1, 2, 128, 64).to("cuda", tdt)
    V = torch.from_numpy(inp.V).view(1, 2, 128, 64).to("cuda", tdt)
    Wo = torch.from_numpy(inp.W_O).to("cuda", tdt)
    shape = Bd.ContextShape(1, 8, 2, 64, 16, 100, 100, 4, 512, 160)
    ctx = Bd.QEvictContext(shape, Wo)
    ctx.load_prefill(K, V)
    ctx.quantize_once(1, [2, 5])
    torch.cuda.synchronize()
    e1 = ctx.ledger_entry(1, 2)
    ck, sk, zk = O.int2_quantize(inp.K[1][32:48].astype(np.float64))
    np.testing.assert_array_equal(e1[0], ck)
    ctx.promote(1, [2])
    ctx.quantize_once(1, [2])
    torch.cuda.synchronize()
    assert ctx.status()[0] == 0
    e2 = ctx.ledger_entry(1, 2)
    for a, b in zip(e1, e2):
        np.testing.assert_array_equal(np.asarray(a).view(np.uint8), np.asarray(b).view(np.uint8))
    st = ctx.state()
    assert int(st["win_tier"][1, 2]) == Bd.TIER_INT2 and int(st["win_tier"][1, 5]) == Bd.TIER_INT2
    # promoted values: check a promotion of window 5
    ctx.promote(1, [5])
    torch.cuda.synchronize()
    st = ctx.state()
    pg = st["win_pages"][1, 5, 0].item()
    got = st["pages"][1, pg, 0].float().cpu().numpy()
    cks, sks, zks = O.int2_quantize(inp.K[1][80:96].astype(np.float64))
    np.testing.assert_array_equal(got, O.int2_promote_values(cks, sks, zks, "fp16"))


def test_errors_are_reported_not_trapped():
    cfg = W.C1.scaled(name="err", ctx=64, steps=0)
    inp = W.draw_decode_inputs(cfg)
    Wo = torch.from_numpy(inp.W_O).to("cuda", torch.float16)
    # a page pool too small for the first appended page: the device records the error
    shape = Bd.ContextShape(1, 8, 2, 64, 16, 2, 2, 4, 512, 80, pages_per_unit=4)
    ctx = Bd.QEvictContext(shape, Wo)
    K = torch.from_numpy(inp.K).view(1, 2, 64, 64).to("cuda", torch.float16)
    ctx.load_prefill(K, K.clone())
    k = torch.zeros((1, 2, 64), dtype=torch.float16, device="cuda")
    ctx.kv_append(k, k)
    rc, _ = ctx.status()
    assert rc == -3  # QE_ERR_POOL_EXHAUSTED
    # invalid demotion request (window not in the full tier): reported, state unchanged
    ctx2 = Bd.QEvictContext(Bd.ContextShape(1, 8, 2, 64, 16, 2, 2, 4, 512, 80), Wo)
    ctx2.load_prefill(K, K.clone())
    ctx2.promote(0, [1])
    assert ctx2.status()[0] == -1
    with pytest.raises(RuntimeError):
        ctx2.quantize_once(0, [10 ** 6])
