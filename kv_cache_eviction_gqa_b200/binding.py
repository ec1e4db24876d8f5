"""Python binding of libqevict (argument marshalling only).

Every function here forwards to the C ABI declared in ``include/qevict.h``; all
computation runs in the library's CUDA kernels. PyTorch supplies device memory
(the context workspace and the inputs/outputs) and the current CUDA stream.
If the shared library is missing, every call raises RuntimeError: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqevict.so")
_lib = None

QE_FP16, QE_BF16 = 0, 1
(QE_OK, QE_ERR_INVALID_ARG, QE_ERR_UNSUPPORTED_SHAPE, QE_ERR_POOL_EXHAUSTED, QE_ERR_LEDGER_FULL,
 QE_ERR_CUDA, QE_ERR_TIMEOUT, QE_ERR_DEVICE_FAULT, QE_ERR_WORKSPACE, QE_ERR_STATE) = range(0, -10, -1)
TIER_EVICTED, TIER_INT2, TIER_FULL, TIER_TAIL = 0, 1, 2, 3


class QeConfig(C.Structure):
    _fields_ = [(n, C.c_int) for n in ("B", "Hq", "Hkv", "D", "dtype", "page", "window",
                                        "full_windows", "int2_windows")] + \
               [("alpha", C.c_float)] + \
               [(n, C.c_int) for n in ("route_every", "hidden", "max_ctx", "pages_per_unit",
                                        "slots_per_unit", "max_splits")]


class QeDiagStats(C.Structure):
    _fields_ = [(n, C.c_longlong) for n in ("live_prev", "changed", "exits", "reentries", "windows_exited",
                                            "windows_reentered")] + [("churn", C.c_double), ("lir", C.c_double)]


class QeLayout(C.Structure):
    _fields_ = [(n, C.c_size_t) for n in ("total", "pages", "page_free", "win_pages", "win_tier",
                                           "win_slot", "slots", "slot_free", "mass", "pert", "norms",
                                           "full_list", "int2_list", "tail_p", "stacks", "route_stats",
                                           "status", "scratch", "scratch_bytes")] + \
               [("max_windows", C.c_int), ("units", C.c_int)]


def lib():
    """Load libqevict.so (raises RuntimeError if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"libqevict.so not found at {_LIB_PATH}; build it with "
                               "`python -m kv_cache_eviction_gqa_b200.build`")
        L = C.CDLL(_LIB_PATH)
        vp, i, sz, f, ll = C.c_void_p, C.c_int, C.c_size_t, C.c_float, C.c_longlong
        sig = {
            "qe_plan": (i, [C.POINTER(QeConfig), C.POINTER(QeLayout)]),
            "qe_workspace_bytes": (sz, [C.POINTER(QeConfig)]),
            "qe_create": (i, [C.POINTER(QeConfig), vp, sz, vp, C.POINTER(vp)]),
            "qe_destroy": (i, [vp]),
            "qe_load_prefill": (i, [vp, vp, vp, i, vp, vp]),
            "qe_kv_append": (i, [vp, vp, vp, vp]),
            "qe_decode_attend_and_score": (i, [vp, vp, vp, vp]),
            "qe_decode_attend_and_score_noalloc": (i, [vp, vp, vp, vp]),
            "qe_route_windows": (i, [vp, vp]),
            "qe_decode_step": (i, [vp, vp, vp, vp, vp, vp]),
            "qe_quantize_once": (i, [vp, i, vp, i, vp]),
            "qe_promote": (i, [vp, i, vp, i, vp]),
            "qe_int2_quantize": (i, [vp, i, i, i, vp, vp, vp]),
            "qe_vwo_l1norm": (i, [vp, i, i, i, i, vp, i, i, i, vp, ll, vp]),
            "qe_criticalkv_scratch_bytes": (sz, [i, i, i, i, i]),
            "qe_criticalkv_select": (i, [vp, i, vp, vp, vp, i, i, i, i, i, i, i, i, f, vp, vp, vp,
                                         vp, sz, vp]),
            "qe_trim_scratch_bytes": (sz, [i, i]),
            "qe_trim_global_topm": (i, [vp, vp, vp, vp, i, i, i, i, i, i, ll, vp, vp, vp, vp, vp,
                                        vp, sz, vp]),
            "qe_route_global_scratch_bytes": (sz, [i, i, i, i]),
            "qe_route_windows_global": (i, [vp, i, i, i, f, vp, sz, vp]),
            "qe_sekv_state_bytes": (sz, [i, i, i, i, i]),
            "qe_sekv_state_offsets": (i, [i, i, i, i, i, C.POINTER(C.c_size_t)]),
            "qe_sekv_build": (i, [vp, vp, vp, i, i, i, i, i, i, f, vp, sz, vp]),
            "qe_sekv_attend": (i, [vp, vp, vp, i, i, i, i, i, i, f, vp, sz, vp, vp]),
            "qe_diag_tiers": (i, [vp, vp, vp, i, i, i, vp, vp]),
            "qe_diag_fmm_scratch_bytes": (sz, [i, i]),
            "qe_diag_fmm": (i, [vp, vp, ll, i, vp, i, i, i, i, i, i, i, vp, vp, sz, vp]),
            "qe_ledger_read": (i, [vp, i, i, vp, vp, vp, vp, vp, vp]),
            "qe_state_bytes": (sz, [vp]),
            "qe_state_export": (i, [vp, vp, sz, vp]),
            "qe_state_import": (i, [vp, vp, sz, vp]),
            "qe_diag_summary": (i, [vp, i, C.POINTER(QeDiagStats), vp]),
            "qe_status": (i, [vp, C.POINTER(C.c_int)]),
            "qe_step_index": (i, [vp]),
            "qe_length": (i, [vp]),
            "qe_list_counts": (i, [vp, C.POINTER(C.c_int), C.POINTER(C.c_int)]),
            "qe_strerror": (C.c_char_p, [i]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name, None)
            if fn is None:
                continue
            fn.restype, fn.argtypes = res, args
        _lib = L
    return _lib


def strerror(code: int) -> str:
    return lib().qe_strerror(code).decode()


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"{what} failed: {strerror(rc)} ({rc})")


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _ptr(t: torch.Tensor):
    return C.c_void_p(t.data_ptr())


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return QE_BF16
    if dt == torch.float16:
        return QE_FP16
    raise ValueError(f"unsupported cache dtype {dt}")


def _need(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


@dataclass
class ContextShape:
    B: int
    Hq: int
    Hkv: int
    D: int
    window: int
    full_windows: int
    int2_windows: int
    route_every: int
    hidden: int
    max_ctx: int
    alpha: float = 0.5
    pages_per_unit: int = 0  # 0: ceil(max_ctx / 16) + 2 * window / 16
    slots_per_unit: int = 0  # 0: full_windows + int2_windows
    max_splits: int = 32


class QEvictContext:
    """One decode context (one attention layer) bound to a torch-allocated workspace."""

    def __init__(self, shape: ContextShape, W_O: torch.Tensor):
        self.shape = shape
        self.dtype = W_O.dtype
        _need(W_O, "W_O", shape=(shape.Hq * shape.D, shape.hidden))
        ppu = shape.pages_per_unit or (-(-shape.max_ctx // 16) + 2 * shape.window // 16)
        spu = shape.slots_per_unit or (shape.full_windows + shape.int2_windows)
        self.cfg = QeConfig(shape.B, shape.Hq, shape.Hkv, shape.D, dtype_code(W_O.dtype), 16,
                            shape.window, shape.full_windows, shape.int2_windows, shape.alpha,
                            shape.route_every, shape.hidden, shape.max_ctx, ppu, spu, shape.max_splits)
        self.layout = QeLayout()
        _check(lib().qe_plan(C.byref(self.cfg), C.byref(self.layout)), "qe_plan")
        self.W_O = W_O
        self.workspace = torch.empty(self.layout.total, dtype=torch.uint8, device=W_O.device)
        h = C.c_void_p()
        _check(lib().qe_create(C.byref(self.cfg), _ptr(self.workspace), self.layout.total, _ptr(W_O),
                               C.byref(h)), "qe_create")
        self._h = h
        self.G = shape.Hq // shape.Hkv
        self.units = shape.B * shape.Hkv

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and _lib is not None:
            _lib.qe_destroy(h)
            self._h = None

    # -- the hot path -------------------------------------------------------------
    def load_prefill(self, K: torch.Tensor, V: torch.Tensor, norms: torch.Tensor = None, stream=None):
        """Load a prefill cache K, V [B][Hkv][ctx][D]; norms [B][Hkv][ctx][G] float32 or None."""
        s = self.shape
        _need(K, "K", self.dtype)
        _need(V, "V", self.dtype, K.shape)
        if K.dim() != 4 or K.shape[:2] != (s.B, s.Hkv) or K.shape[3] != s.D:
            raise ValueError("K, V must be [B][Hkv][ctx][D]")
        if norms is not None:
            _need(norms, "norms", torch.float32, (s.B, s.Hkv, K.shape[2], self.G))
        _check(lib().qe_load_prefill(self._h, _ptr(K), _ptr(V), K.shape[2],
                                     _ptr(norms) if norms is not None else None, _stream(stream)),
               "qe_load_prefill")

    def kv_append(self, k: torch.Tensor, v: torch.Tensor, stream=None):
        s = self.shape
        _need(k, "k_new", self.dtype, (s.B, s.Hkv, s.D))
        _need(v, "v_new", self.dtype, (s.B, s.Hkv, s.D))
        _check(lib().qe_kv_append(self._h, _ptr(k), _ptr(v), _stream(stream)), "qe_kv_append")

    def decode_attend_and_score(self, q: torch.Tensor, out: torch.Tensor = None, stream=None):
        s = self.shape
        _need(q, "q", self.dtype, (s.B, s.Hq, s.D))
        if out is None:
            out = torch.empty((s.B, s.Hq, s.D), dtype=torch.float32, device=q.device)
        _need(out, "out", torch.float32, (s.B, s.Hq, s.D))
        _check(lib().qe_decode_attend_and_score(self._h, _ptr(q), _ptr(out), _stream(stream)),
               "qe_decode_attend_and_score")
        return out

    def route_windows(self, stream=None):
        _check(lib().qe_route_windows(self._h, _stream(stream)), "qe_route_windows")

    def decode_step(self, q, k, v, out=None, stream=None):
        s = self.shape
        _need(q, "q", self.dtype, (s.B, s.Hq, s.D))
        _need(k, "k_new", self.dtype, (s.B, s.Hkv, s.D))
        _need(v, "v_new", self.dtype, (s.B, s.Hkv, s.D))
        if out is None:
            out = torch.empty((s.B, s.Hq, s.D), dtype=torch.float32, device=q.device)
        _need(out, "out", torch.float32, (s.B, s.Hq, s.D))
        _check(lib().qe_decode_step(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(out), _stream(stream)),
               "qe_decode_step")
        return out

    def quantize_once(self, unit: int, win_ids, stream=None):
        ids = (C.c_int32 * len(win_ids))(*[int(x) for x in win_ids])
        _check(lib().qe_quantize_once(self._h, unit, ids, len(win_ids), _stream(stream)),
               "qe_quantize_once")

    def promote(self, unit: int, win_ids, stream=None):
        ids = (C.c_int32 * len(win_ids))(*[int(x) for x in win_ids])
        _check(lib().qe_promote(self._h, unit, ids, len(win_ids), _stream(stream)), "qe_promote")

    # -- status and state -----------------------------------------------------------
    def status(self):
        d = C.c_int()
        rc = lib().qe_status(self._h, C.byref(d))
        return rc, d.value

    @property
    def step_index(self) -> int:
        return lib().qe_step_index(self._h)

    @property
    def length(self) -> int:
        return lib().qe_length(self._h)

    def _view(self, off: int, count: int, dtype, shape):
        nbytes = count * torch.tensor([], dtype=dtype).element_size()
        return self.workspace[off:off + nbytes].view(dtype).view(*shape)

    def state(self) -> dict:
        """Views (no copies) of the context's state arrays inside the workspace."""
        L, s, U, W = self.layout, self.shape, self.units, self.layout.max_windows
        ppu, spu = self.cfg.pages_per_unit, self.cfg.slots_per_unit
        pitch = -(-s.max_ctx // 16) * 16
        return {
            "pages": self._view(L.pages, U * ppu * 2 * 16 * s.D, self.dtype, (U, ppu, 2, 16, s.D)),
            "win_pages": self._view(L.win_pages, U * W * (s.window // 16), torch.int32,
                                    (U, W, s.window // 16)),
            "win_tier": self._view(L.win_tier, U * W, torch.uint8, (U, W)),
            "win_slot": self._view(L.win_slot, U * W, torch.int32, (U, W)),
            "slots": self._view(L.slots, U * spu * s.window * s.D, torch.uint8, (U, spu, s.window * s.D)),
            "mass": self._view(L.mass, U * W, torch.float32, (U, W)),
            "pert": self._view(L.pert, U * W, torch.float32, (U, W)),
            "norms": self._view(L.norms, U * pitch * self.G, torch.float32, (U, pitch, self.G)),
            "full_list": self._view(L.full_list, U * W, torch.int32, (U, W)),
            "int2_list": self._view(L.int2_list, U * W, torch.int32, (U, W)),
            "tail_p": self._view(L.tail_p, U * s.window * self.G, torch.float32, (U, s.window, self.G)),
            "stacks": self._view(L.stacks, U * 4, torch.int32, (U, 4)),
            "route_stats": self._view(L.route_stats, U * 8, torch.int32, (U, 8)),
        }

    def state_bytes(self) -> int:
        return int(lib().qe_state_bytes(self._h))

    def export_state(self, dst: torch.Tensor = None, stream=None) -> torch.Tensor:
        """Checkpoint of the context (qe_state_export) into a uint8 tensor (host or device)."""
        n = self.state_bytes()
        if dst is None:
            dst = torch.empty(n, dtype=torch.uint8, device=self.workspace.device)
        if dst.dtype != torch.uint8 or not dst.is_contiguous() or dst.numel() < n:
            raise ValueError(f"dst must be a contiguous uint8 tensor of at least {n} bytes")
        _check(lib().qe_state_export(self._h, _ptr(dst), n, _stream(stream)), "qe_state_export")
        return dst

    def import_state(self, src: torch.Tensor, stream=None):
        """Restore a checkpoint taken from a context of the same configuration (qe_state_import)."""
        if src.dtype != torch.uint8 or not src.is_contiguous():
            raise ValueError("src must be a contiguous uint8 tensor")
        _check(lib().qe_state_import(self._h, _ptr(src), src.numel(), _stream(stream)), "qe_state_import")

    def ledger_entry(self, unit: int, win: int, stream=None):
        """One window's INT2 ledger entry as (codes_K, s_K, z_K, codes_V, s_V, z_V) NumPy arrays
        (codes [window][D] in 0..3, scales and zeros [window][D/16] float16), read through
        qe_ledger_read; None when the window has no entry."""
        import numpy as np
        w, D = self.shape.window, self.shape.D
        dev = self.workspace.device
        ck = torch.empty((w, D // 4), dtype=torch.uint8, device=dev)
        cv = torch.empty_like(ck)
        mk = torch.empty((w, D // 16), dtype=torch.int32, device=dev)
        mv = torch.empty_like(mk)
        found = torch.zeros(1, dtype=torch.int32, device=dev)
        _check(lib().qe_ledger_read(self._h, unit, win, _ptr(ck), _ptr(mk), _ptr(cv), _ptr(mv), _ptr(found),
                                    _stream(stream)), "qe_ledger_read")
        if stream is None:
            torch.cuda.synchronize(dev)
        else:
            stream.synchronize()
        if int(found.item()) == 0:
            return None

        def codes(b):
            b = b.cpu().numpy()
            return np.stack([(b >> (2 * e)) & 3 for e in range(4)], -1).reshape(w, D)

        def meta(m):
            m = m.cpu().numpy().view(np.uint32)
            return ((m & 0xFFFF).astype(np.uint16).view(np.float16),
                    (m >> 16).astype(np.uint16).view(np.float16))
        sk, zk = meta(mk)
        sv, zv = meta(mv)
        return codes(ck), sk, zk, codes(cv), sv, zv


# ---------------------------------------------------------------------------------
# standalone kernels
# ---------------------------------------------------------------------------------


def int2_quantize(x: torch.Tensor, stream=None):
    """INT2 group quantiser: x [T][D] -> (codes uint8 [T][D/4], meta int32 [T][D/16])."""
    _need(x, "x")
    T, D = x.shape
    codes = torch.empty((T, D // 4), dtype=torch.uint8, device=x.device)
    meta = torch.empty((T, D // 16), dtype=torch.int32, device=x.device)
    _check(lib().qe_int2_quantize(_ptr(x), T, D, dtype_code(x.dtype), _ptr(codes), _ptr(meta),
                                  _stream(stream)), "qe_int2_quantize")
    return codes, meta


def vwo_l1norm(V: torch.Tensor, W_O: torch.Tensor, Hq: int, Hkv: int, out=None, stream=None):
    """N[g][r][j] = ||V[g][r] @ W_O^{(g % Hkv)*G + j}||_1 for V [n_groups][rows][D]."""
    _need(V, "V")
    _need(W_O, "W_O", V.dtype)
    n_groups, rows, D = V.shape
    G = Hq // Hkv
    if out is None:
        out = torch.empty((n_groups, rows, G), dtype=torch.float32, device=V.device)
    _need(out, "out", torch.float32)
    _check(lib().qe_vwo_l1norm(_ptr(V), n_groups, rows, D, dtype_code(V.dtype), _ptr(W_O), Hq, Hkv,
                               W_O.shape[1], _ptr(out), rows * G, _stream(stream)), "qe_vwo_l1norm")
    return out


def trim_scratch_bytes(n_heads: int, max_pages_per_head: int) -> int:
    return int(lib().qe_trim_scratch_bytes(n_heads, max_pages_per_head))


def trim_global_topm(beta: torch.Tensor, pos: torch.Tensor, page_table: torch.Tensor,
                     lengths: torch.Tensor, t: int, M: int, kv_in: torch.Tensor, kv_out=None,
                     beta_out=None, pos_out=None, new_lengths=None, scratch=None, stream=None):
    """DBTrimKV global top-M trim with stable per-head compaction (qe_trim_global_topm).

    beta [P][16] float32, pos [P][16] int32, page_table [H][max_pages] int32, lengths [H] int32,
    kv_in [P][2][16][D] fp16/bf16. Returns (kv_out, beta_out, pos_out, new_lengths, scratch);
    the device status word is scratch[:8] (see trim_status).
    """
    _need(beta, "beta", torch.float32)
    P = beta.shape[0]
    _need(pos, "pos", torch.int32, beta.shape)
    _need(page_table, "page_table", torch.int32)
    H, max_pages = page_table.shape
    _need(lengths, "lengths", torch.int32, (H,))
    _need(kv_in, "kv_in")
    D = kv_in.shape[-1]
    dev = kv_in.device
    kv_out = torch.empty_like(kv_in) if kv_out is None else kv_out
    beta_out = torch.empty_like(beta) if beta_out is None else beta_out
    pos_out = torch.empty_like(pos) if pos_out is None else pos_out
    new_lengths = torch.empty(H, dtype=torch.int32, device=dev) if new_lengths is None else new_lengths
    for name, x, y in (("kv_out", kv_out, kv_in), ("beta_out", beta_out, beta), ("pos_out", pos_out, pos)):
        _need(x, name, y.dtype, y.shape)
    nbytes = trim_scratch_bytes(H, max_pages)
    if scratch is None:
        scratch = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    _check(lib().qe_trim_global_topm(_ptr(beta), _ptr(pos), _ptr(page_table), _ptr(lengths), H,
                                     max_pages, P, D, dtype_code(kv_in.dtype), int(t), int(M),
                                     _ptr(kv_in), _ptr(kv_out), _ptr(beta_out), _ptr(pos_out),
                                     _ptr(new_lengths), _ptr(scratch), scratch.numel(),
                                     _stream(stream)), "qe_trim_global_topm")
    return kv_out, beta_out, pos_out, new_lengths, scratch


def trim_status(scratch: torch.Tensor):
    """(code, detail) of the device status word a trim call left in its scratch."""
    w = scratch[:8].view(torch.int32).cpu()
    return int(w[0]), int(w[1])


def criticalkv_select(q_obs: torch.Tensor, K: torch.Tensor, V: torch.Tensor, W_O: torch.Tensor,
                      budget: int, alpha: float = 0.5, A=None, N=None, idx=None, scratch=None,
                      stream=None):
    """CriticalKV two-stage selection with an observation window (qe_criticalkv_select).

    q_obs [B][Hq][n_obs][D], K and V [B][Hkv][n][D], W_O [Hq*D][hidden], all one cache dtype.
    Returns (A [B][Hkv][G][n] fp32, N [B][Hkv][n][G] fp32, idx [B][Hkv][budget] int32, scratch);
    the device status word is scratch[:8] (see trim_status).
    """
    _need(q_obs, "q_obs")
    B, Hq, n_obs, D = q_obs.shape
    _need(K, "K", q_obs.dtype)
    _, Hkv, n, _ = K.shape
    _need(V, "V", q_obs.dtype, K.shape)
    _need(W_O, "W_O", q_obs.dtype)
    G = Hq // Hkv
    dev = K.device
    A = torch.empty((B, Hkv, G, n), dtype=torch.float32, device=dev) if A is None else A
    N = torch.empty((B, Hkv, n, G), dtype=torch.float32, device=dev) if N is None else N
    idx = torch.empty((B, Hkv, budget), dtype=torch.int32, device=dev) if idx is None else idx
    _need(A, "A", torch.float32, (B, Hkv, G, n))
    _need(N, "N", torch.float32, (B, Hkv, n, G))
    _need(idx, "idx", torch.int32, (B, Hkv, budget))
    nbytes = int(lib().qe_criticalkv_scratch_bytes(B, Hq, Hkv, n, n_obs))
    if scratch is None:
        scratch = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    _check(lib().qe_criticalkv_select(_ptr(q_obs), n_obs, _ptr(K), _ptr(V), _ptr(W_O), B, Hq, Hkv, n, D,
                                      W_O.shape[1], dtype_code(K.dtype), budget, float(alpha), _ptr(A),
                                      _ptr(N), _ptr(idx), _ptr(scratch), scratch.numel(),
                                      _stream(stream)), "qe_criticalkv_select")
    return A, N, idx, scratch


class TierDiagnostics:
    """Selection churn and global LIR over the routing events of a run (qe_diag_tiers).

    Holds the previous tier map, the per-window history flags and the int64 counters
    [units][6] (live_prev, changed, exits, reentries, windows_exited, windows_reentered) on the
    device. Call ``update(tiers)`` after every routing event with the [units][W] uint8 tier map
    (e.g. ``QEvictContext.state()["win_tier"]``); the first call only records the map.
    """

    def __init__(self, units: int, W: int, device):
        self.units, self.W = units, W
        self.prev = torch.zeros((units, W), dtype=torch.uint8, device=device)
        self.flags = torch.zeros((units, W), dtype=torch.uint8, device=device)
        self.counters = torch.zeros((units, 6), dtype=torch.int64, device=device)
        self.events = 0

    def update(self, tiers: torch.Tensor, stream=None):
        _need(tiers, "tiers", torch.uint8, (self.units, self.W))
        _check(lib().qe_diag_tiers(_ptr(tiers), _ptr(self.prev), _ptr(self.flags), self.units, self.W,
                                   1 if self.events == 0 else 0, _ptr(self.counters), _stream(stream)),
               "qe_diag_tiers")
        self.events += 1

    def summary(self, stream=None) -> dict:
        """Pooled counts and the two ratios (nan when a denominator is 0), from qe_diag_summary;
        synchronises."""
        st = QeDiagStats()
        _check(lib().qe_diag_summary(_ptr(self.counters), self.units, C.byref(st), _stream(stream)),
               "qe_diag_summary")
        return {name: getattr(st, name) for name, _ in QeDiagStats._fields_}


def diag_fmm_scratch_bytes(units: int, G: int) -> int:
    return int(lib().qe_diag_fmm_scratch_bytes(units, G))


def diag_fmm(q: torch.Tensor, K_ghost: torch.Tensor, n: int, tiers: torch.Tensor, window: int,
             out=None, scratch=None, stream=None):
    """Future missed mass of one step (qe_diag_fmm).

    q [B][Hq][D], K_ghost [B][Hkv][n_stride][D] (same dtype; the first n rows of each unit are
    used), tiers [B*Hkv][W] uint8. Returns (fmm [B*Hkv] float32, scratch); the device status
    word is scratch[:8] (see trim_status).
    """
    _need(q, "q")
    B, Hq, D = q.shape
    _need(K_ghost, "K_ghost", q.dtype)
    _, Hkv, n_stride, _ = K_ghost.shape
    _need(tiers, "tiers", torch.uint8)
    U, W = tiers.shape
    if U != B * Hkv:
        raise ValueError(f"tiers must have {B * Hkv} rows, got {U}")
    dev = q.device
    out = torch.empty(U, dtype=torch.float32, device=dev) if out is None else out
    _need(out, "out", torch.float32, (U,))
    if scratch is None:
        scratch = torch.empty(diag_fmm_scratch_bytes(U, Hq // Hkv), dtype=torch.uint8, device=dev)
    _check(lib().qe_diag_fmm(_ptr(q), _ptr(K_ghost), n_stride, int(n), _ptr(tiers), W, int(window), B, Hq,
                             Hkv, D, dtype_code(q.dtype), _ptr(out), _ptr(scratch), scratch.numel(),
                             _stream(stream)), "qe_diag_fmm")
    return out, scratch


def route_global_scratch_bytes(n_layers: int, B: int, Hkv: int, max_windows: int) -> int:
    return int(lib().qe_route_global_scratch_bytes(n_layers, B, Hkv, max_windows))


def route_windows_global(ctxs, full_windows: int, int2_windows: int, alpha: float = 0.5, scratch=None,
                         stream=None):
    """One routing event under budgets shared by every layer (context) and kv head of each
    sequence (qe_route_windows_global). ``ctxs``: the layers' QEvictContext, in layer order.
    Returns the scratch buffer (reuse it across events)."""
    if not ctxs:
        raise ValueError("no contexts")
    c0 = ctxs[0]
    W = c0.layout.max_windows
    if scratch is None:
        nbytes = route_global_scratch_bytes(len(ctxs), c0.shape.B, c0.shape.Hkv, W)
        scratch = torch.empty(nbytes, dtype=torch.uint8, device=c0.workspace.device)
    arr = (C.c_void_p * len(ctxs))(*[c._h.value for c in ctxs])
    _check(lib().qe_route_windows_global(arr, len(ctxs), int(full_windows), int(int2_windows), float(alpha),
                                         _ptr(scratch), scratch.numel(), _stream(stream)),
           "qe_route_windows_global")
    return scratch


def sekv_state_bytes(B: int, Hq: int, Hkv: int, n: int, D: int) -> int:
    return int(lib().qe_sekv_state_bytes(B, Hq, Hkv, n, D))


def sekv_build(K: torch.Tensor, V: torch.Tensor, H: torch.Tensor, tau: float, Hq: int, state=None, stream=None):
    """SEKV segmentation and span summaries (qe_sekv_build). K, V [B][Hkv][n][D] fp16/bf16,
    H [B][n] float32 surprisal. Returns the state buffer for sekv_attend."""
    _need(K, "K")
    B, Hkv, n, D = K.shape
    _need(V, "V", K.dtype, K.shape)
    _need(H, "H", torch.float32, (B, n))
    nbytes = sekv_state_bytes(B, Hq, Hkv, n, D)
    if nbytes == 0:
        raise ValueError("unsupported SEKV shape")
    if state is None:
        state = torch.empty(nbytes, dtype=torch.uint8, device=K.device)
    _check(lib().qe_sekv_build(_ptr(K), _ptr(V), _ptr(H), B, Hq, Hkv, n, D, dtype_code(K.dtype), float(tau),
                               _ptr(state), state.numel(), _stream(stream)), "qe_sekv_build")
    return state


def sekv_attend(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, theta: float, state: torch.Tensor, out=None,
                stream=None):
    """SEKV mixed-resolution attention of one step (qe_sekv_attend). q [B][Hq][D]; K, V and
    state as given to sekv_build. Returns out [B][Hq][D] float32."""
    _need(q, "q", K.dtype)
    B, Hq, D = q.shape
    _, Hkv, n, _ = K.shape
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, (B, Hq, D))
    _check(lib().qe_sekv_attend(_ptr(q), _ptr(K), _ptr(V), B, Hq, Hkv, n, D, dtype_code(q.dtype), float(theta),
                                _ptr(state), state.numel(), _ptr(out), _stream(stream)), "qe_sekv_attend")
    return out


def sekv_views(state: torch.Tensor, B: int, Hq: int, Hkv: int, n: int, D: int) -> dict:
    """Views of the SEKV state arrays (counts, anchors, span bounds, summaries, expansion flags)."""
    off = (C.c_size_t * 8)()
    _check(lib().qe_sekv_state_offsets(B, Hq, Hkv, n, D, off), "qe_sekv_state_offsets")
    cap = int(off[7])

    def view(o, count, dtype, shape):
        nb = count * torch.tensor([], dtype=dtype).element_size()
        return state[o:o + nb].view(dtype).view(*shape)

    return {"counts": view(off[0], B * 2, torch.int32, (B, 2)),
            "anchor_pos": view(off[1], B * n, torch.int32, (B, n)),
            "span_start": view(off[2], B * cap, torch.int32, (B, cap)),
            "span_end": view(off[3], B * cap, torch.int32, (B, cap)),
            "kbar": view(off[4], B * Hkv * cap * D, torch.float32, (B, Hkv, cap, D)),
            "vbar": view(off[5], B * Hkv * cap * D, torch.float32, (B, Hkv, cap, D)),
            "expanded": view(off[6], B * Hkv * cap, torch.uint8, (B, Hkv, cap)),
            "cap": cap}
