"""The allocation-free decode entry point gives the same results as the regular one.

qe_decode_attend_and_score_noalloc serves callers that may not hand the library any device
memory beyond their inputs and outputs while a step runs (for instance an engine that
gives a plugin only its buffers). It keeps the decode kernel's per-call scratch in a fixed
array inside the library. The GPU test drives two identical contexts, one through each
entry point, for two decode calls in a row (and one more after routing), with a third
context of another shape using the same array in between, and requires identical outputs
and cumulative window scores: both entry points run the same deterministic kernel on the
same inputs. A CPU test checks that a context whose scratch does not fit the array is
refused before anything is enqueued. The file is collected last.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from kv_cache_eviction_gqa_b200 import workloads as W


def _noalloc(Bd, ctx, q, out, stream):
    return Bd.lib().qe_decode_attend_and_score_noalloc(ctx._h, C.c_void_p(q.data_ptr()),
                                                       C.c_void_p(out.data_ptr()), stream)


@pytest.mark.gpu
def test_noalloc_matches_regular_entry_point():
    from kv_cache_eviction_gqa_b200 import binding as Bd

    cfg = W.C2.scaled(name="noalloc", B=2, Hkv=2, Hq=8, ctx=700, full_windows=6, int2_windows=10,
                      route_every=4, steps=3, hidden=512)
    # another shape that shares the static array between the calls above
    other = W.C1.scaled(name="noalloc_other", B=1, Hkv=2, Hq=4, ctx=300, full_windows=4, int2_windows=4,
                        route_every=4, steps=3, hidden=256)
    inp = W.draw_decode_inputs(cfg)
    inp2 = W.draw_decode_inputs(other)
    tdt = torch.bfloat16
    K = torch.from_numpy(inp.K).view(cfg.B, cfg.Hkv, cfg.ctx, cfg.D).to("cuda", tdt)
    V = torch.from_numpy(inp.V).view(cfg.B, cfg.Hkv, cfg.ctx, cfg.D).to("cuda", tdt)
    Wo = torch.from_numpy(inp.W_O).to("cuda", tdt)
    shape = Bd.ContextShape(cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.window, cfg.full_windows,
                            cfg.int2_windows, cfg.route_every, cfg.hidden, cfg.ctx + cfg.steps)
    regular, noalloc = Bd.QEvictContext(shape, Wo), Bd.QEvictContext(shape, Wo)
    for ctx in (regular, noalloc):
        ctx.load_prefill(K, V)
    t2 = torch.float16
    K2 = torch.from_numpy(inp2.K).view(other.B, other.Hkv, other.ctx, other.D).to("cuda", t2)
    V2 = torch.from_numpy(inp2.V).view(other.B, other.Hkv, other.ctx, other.D).to("cuda", t2)
    Wo2 = torch.from_numpy(inp2.W_O).to("cuda", t2)
    shape2 = Bd.ContextShape(other.B, other.Hq, other.Hkv, other.D, other.window, other.full_windows,
                             other.int2_windows, other.route_every, other.hidden, other.ctx + other.steps)
    third = Bd.QEvictContext(shape2, Wo2)
    third.load_prefill(K2, V2)
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    for s in range(cfg.steps):
        q = torch.from_numpy(inp.q[s]).to("cuda", tdt)
        k = torch.from_numpy(inp.k_new[s]).to("cuda", tdt)
        v = torch.from_numpy(inp.v_new[s]).to("cuda", tdt)
        for ctx in (regular, noalloc):
            ctx.kv_append(k, v)
        out_r = regular.decode_attend_and_score(q)
        out_n = torch.empty_like(out_r)
        rc = _noalloc(Bd, noalloc, q, out_n, stream)
        assert rc == 0, Bd.strerror(rc)
        # the other context's call reuses the array on the same stream
        q2 = torch.from_numpy(inp2.q[s]).to("cuda", t2)
        third.kv_append(torch.from_numpy(inp2.k_new[s]).to("cuda", t2),
                        torch.from_numpy(inp2.v_new[s]).to("cuda", t2))
        out3 = torch.empty((other.B, other.Hq, other.D), dtype=torch.float32, device="cuda")
        assert _noalloc(Bd, third, q2, out3, stream) == 0
        if s == 0:  # create INT2 windows so later calls read both tiers
            regular.route_windows()
            noalloc.route_windows()
            third.route_windows()
        torch.cuda.synchronize()
        assert regular.status()[0] == 0 and noalloc.status()[0] == 0 and third.status()[0] == 0
        np.testing.assert_array_equal(out_r.cpu().numpy(), out_n.cpu().numpy(),
                                      err_msg=f"call {s}: outputs differ")
        for key in ("mass", "pert", "tail_p"):
            np.testing.assert_array_equal(regular.state()[key].cpu().numpy(), noalloc.state()[key].cpu().numpy(),
                                          err_msg=f"call {s}: {key} differs")
    n_full, n_int2 = C.c_int(), C.c_int()
    Bd.lib().qe_list_counts(noalloc._h, C.byref(n_full), C.byref(n_int2))
    assert n_int2.value > 0


def test_noalloc_rejects_oversized_scratch():
    """A context whose decode scratch exceeds the static array is refused with
    QE_ERR_INVALID_ARG before anything is enqueued (no device memory is touched, so the
    workspace and tensors here are stand-in addresses)."""
    from kv_cache_eviction_gqa_b200 import binding as Bd

    cfg = Bd.QeConfig(64, 32, 8, 128, Bd.QE_BF16, 16, 16, 64, 128, 0.5, 16, 4096, 131072,
                      131072 // 16 + 8, 192, 16)
    lay = Bd.QeLayout()
    assert Bd.lib().qe_plan(C.byref(cfg), C.byref(lay)) == 0
    # decode scratch of this shape: per-window partials alone are U * W * 3G floats
    assert lay.units * lay.max_windows * 3 * 4 * 4 > 16 << 20
    h = C.c_void_p()
    fake = C.c_void_p(1 << 40)  # 256-byte aligned, never dereferenced by these calls
    assert Bd.lib().qe_create(C.byref(cfg), fake, C.c_size_t(lay.total), fake, C.byref(h)) == 0
    try:
        rc = Bd.lib().qe_decode_attend_and_score_noalloc(h, fake, fake, None)
        assert rc == Bd.QE_ERR_INVALID_ARG, rc
    finally:
        Bd.lib().qe_destroy(h)
