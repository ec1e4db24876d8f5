"""DBTrimKV global top-M trim on the GPU against the oracle ("Make Each Token Count",
Metodologia 2-4).

Both sides rank log r = (t - pos) * ln(beta) in float64. The oracle's ln is numpy's and the
kernel's is CUDA's; both are within an ulp of the exact value, so an entry whose oracle key
lies within a few ulps of the M-th key may land on either side of the cut. Such entries are
near-ties: counted and reported, never failed. Everything else is bit-exact: the kept set,
the new lengths (up to the near-ties), the survivors' order, and the bytes moved (K/V rows,
beta, pos).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from kv_cache_eviction_gqa_b200 import workloads as W

pytestmark = pytest.mark.gpu

NEAR_ULPS = 8


def _device_inputs(cfg, lay, dtype=torch.bfloat16):
    from kv_cache_eviction_gqa_b200 import binding as B  # noqa: F401  (loads the library)
    dev = torch.device("cuda")
    kv = W.draw_trim_kv_pool(cfg, lay.n_pages, dev, dtype)
    return dict(
        beta=torch.from_numpy(lay.beta_pages).to(dev),
        pos=torch.from_numpy(lay.pos_pages).to(dev),
        page_table=torch.from_numpy(lay.page_table).to(dev),
        lengths=torch.from_numpy(lay.lengths).to(dev),
        kv=kv,
    )


def run_trim_parity(cfg, lay, M, dtype=torch.bfloat16):
    from kv_cache_eviction_gqa_b200 import binding as B
    d = _device_inputs(cfg, lay, dtype)
    kv_out = torch.zeros_like(d["kv"])
    beta_out = torch.zeros_like(d["beta"])
    pos_out = torch.full_like(d["pos"], -1)
    _, _, _, new_len, scratch = B.trim_global_topm(d["beta"], d["pos"], d["page_table"], d["lengths"],
                                                   cfg.t, M, d["kv"], kv_out, beta_out, pos_out)
    torch.cuda.synchronize()
    assert B.trim_status(scratch) == (0, 0)

    masks, lens, keys = O.trim_global_topm(lay.betas, lay.poss, cfg.t, M)
    total = keys.size
    near = np.zeros(total, dtype=bool)
    if 0 < M < total:
        kth = np.sort(keys)[::-1][M - 1]
        near = np.abs(keys - kth) <= NEAR_ULPS * np.spacing(np.abs(kth))

    new_len = new_len.cpu().numpy()
    bo, po = beta_out.cpu().numpy(), pos_out.cpu().numpy()
    table = lay.page_table
    kv_in, kv_o = d["kv"], kv_out
    src_pages, src_slots, dst_pages, dst_slots = [], [], [], []
    mismatch = near_count = 0
    a = 0
    for h in range(len(lay.lengths)):
        n = int(lay.lengths[h])
        L = int(new_len[h])
        assert 0 <= L <= n
        dst = np.arange(L)
        dpg, dsl = table[h, dst // 16], dst % 16
        got_pos = po[dpg, dsl]
        # survivors keep their order and are entries of this head: positions are distinct
        # and sorted within a head, so they identify the entries
        assert np.all(np.diff(got_pos) > 0), f"head {h}: survivors out of order"
        idx = np.searchsorted(lay.poss[h], got_pos)
        assert np.all(idx < n) and np.array_equal(lay.poss[h][idx], got_pos), f"head {h}"
        got = np.zeros(n, dtype=bool)
        got[idx] = True
        diff = got != masks[h]
        hn = near[a:a + n]
        assert not np.any(diff & ~hn), (
            f"head {h}: {int(np.sum(diff & ~hn))} entries differ away from the cut")
        mismatch += int(diff.sum())
        near_count += int(hn.sum())
        np.testing.assert_array_equal(bo[dpg, dsl], lay.betas[h][idx])
        spg, ssl = table[h, idx // 16], idx % 16
        src_pages.append(spg), src_slots.append(ssl), dst_pages.append(dpg), dst_slots.append(dsl)
        a += n
    if mismatch == 0:
        np.testing.assert_array_equal(new_len, lens)
    else:
        assert abs(int(new_len.sum()) - min(M, total)) == 0
    # K/V rows: byte-exact copies of the kept entries' rows
    cat = lambda xs: torch.from_numpy(np.concatenate(xs).astype(np.int64)).cuda()
    sp, ss, dp, ds = map(cat, (src_pages, src_slots, dst_pages, dst_slots))
    for part in (0, 1):
        want = kv_in[sp, part, ss].view(torch.int16)
        have = kv_o[dp, part, ds].view(torch.int16)
        assert torch.equal(want, have), f"kv part {part} differs"
    return dict(mismatch=mismatch, near=near_count, kept=int(new_len.sum()), total=total)


def small_cfg(**kw):
    base = dict(layers=2, Hkv=3, len_lo=1, len_hi=5000, t=8192, M=4000, seed=77)
    base.update(kw)
    return W.C4.scaled(**base)


@pytest.mark.parametrize("frac", [0.05, 0.37, 0.9])
def test_trim_small_random(frac):
    cfg = small_cfg()
    lay = W.trim_layout(cfg)
    total = int(lay.lengths.sum())
    r = run_trim_parity(cfg, lay, int(frac * total))
    assert r["kept"] == int(frac * total)


@pytest.mark.parametrize("M", ["zero", "all", "all_plus", "all_minus_one", "one"])
def test_trim_budget_edges(M):
    cfg = small_cfg(seed=78)
    lay = W.trim_layout(cfg)
    total = int(lay.lengths.sum())
    m = {"zero": 0, "all": total, "all_plus": total + 1000, "all_minus_one": total - 1, "one": 1}[M]
    r = run_trim_parity(cfg, lay, m)
    assert r["kept"] == min(m, total)


def test_trim_ties_across_heads_go_to_lower_flat_index():
    # every head holds the same positions and one shared beta: each key appears once per head,
    # so the cut falls inside a block of exact ties that only the flat index can order
    cfg = small_cfg(layers=1, Hkv=5, len_lo=3000, len_hi=3000, t=4096, seed=79)
    pos = np.sort(W._rng(5).choice(cfg.t, size=3000, replace=False)).astype(np.int32)
    betas = [np.full(3000, 0.93, np.float32) for _ in range(5)]
    lay = W.trim_layout(cfg, np.full(5, 3000), betas, [pos] * 5)
    r = run_trim_parity(cfg, lay, 5 * 1000 + 2)
    assert r["mismatch"] == 0


def test_trim_ragged_heads_with_empty_and_full():
    cfg = small_cfg(layers=1, Hkv=4, len_lo=0, len_hi=4096, seed=80)
    lengths = np.array([0, 4096, 17, 2049], dtype=np.int32)
    r = W._rng(6)
    betas = [r.beta(8.0, 1.0, size=n).astype(np.float32) for n in lengths]
    poss = [np.sort(r.choice(cfg.t, size=n, replace=False)).astype(np.int32) for n in lengths]
    lay = W.trim_layout(cfg, lengths, betas, poss)
    run_trim_parity(cfg, lay, 3000)


def test_trim_fp16_and_d64():
    cfg = small_cfg(D=64, seed=81, dtype="fp16")
    lay = W.trim_layout(cfg)
    run_trim_parity(cfg, lay, int(0.4 * lay.lengths.sum()), dtype=torch.float16)


def test_trim_reports_bad_page_table_entry():
    from kv_cache_eviction_gqa_b200 import binding as B
    cfg = small_cfg(seed=82)
    lay = W.trim_layout(cfg)
    lay.page_table[1, 0] = lay.n_pages + 5  # out of range: recorded, never dereferenced
    d = _device_inputs(cfg, lay)
    *_, scratch = B.trim_global_topm(d["beta"], d["pos"], d["page_table"], d["lengths"], cfg.t,
                                     100, d["kv"])
    torch.cuda.synchronize()
    code, detail = B.trim_status(scratch)
    assert code == B.QE_ERR_DEVICE_FAULT and detail == 1


@pytest.mark.slow
def test_trim_full_c4():
    cfg = W.C4
    lay = W.trim_layout(cfg)
    r = run_trim_parity(cfg, lay, cfg.M)
    assert r["kept"] == cfg.M
    print("c4 trim:", r)
