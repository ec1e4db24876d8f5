"""Seeded synthetic inputs for the tiered-KV decode path.

This module only draws and encodes data. It holds none of the method's
arithmetic (no attention, no scoring, no quantisation, no selection), so both
the CUDA path and the CPU oracle may take their inputs from it.

Every random draw goes through ``numpy.random.Generator(PCG64(SeedSequence(...)))``
with the config's base seed (1000 + config index) and, for cache tensors, the
(batch, kv-head) unit as extra entropy words, so that one unit can be drawn
without drawing the others. Values are drawn in float32 and rounded once to the
cache dtype (fp16 or bf16, round-to-nearest-even); the arrays returned are
float32 arrays that hold those exact dtype values.

Workload shapes follow the pages' long-context decode settings: QEvict
("Resumo Técnico: QEvict", Resultados: 32K-context RULER, 5-20 % budgets),
CriticalKV ("Resumo Técnico: CriticalKV", Algoritmo: two-stage selection with
alpha = 0.5) and DBTrimKV ("Make Each Token Count", Metodologia 2-3: retention
beta^(t-i) with a global budget M).
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass

import numpy as np

# --------------------------------------------------------------------------
# dtype encoding (data representation only)
# --------------------------------------------------------------------------


def to_bf16_values(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest-even); return them as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def to_fp16_values(x: np.ndarray) -> np.ndarray:
    """Round float32 values to IEEE half (nearest-even); return them as float32."""
    return np.asarray(x, dtype=np.float32).astype(np.float16).astype(np.float32)


def to_dtype_values(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return to_bf16_values(x)
    if dtype == "fp16":
        return to_fp16_values(x)
    raise ValueError(f"unknown cache dtype {dtype!r}")


def _rng(*words: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(w) for w in words])))


# --------------------------------------------------------------------------
# decode workloads (windowed three-tier cache)
# --------------------------------------------------------------------------


@dataclass(frozen=True)
class DecodeConfig:
    """One decode workload: a single attention layer, ``steps`` decode steps."""

    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    ctx: int
    window: int
    full_windows: int  # budget F, in windows, per (batch, kv-head)
    int2_windows: int  # budget Q, in windows, per (batch, kv-head)
    route_every: int  # R: route after attention on every step s with s % R == 0
    steps: int
    dtype: str  # cache dtype: "fp16" or "bf16"
    hidden: int  # columns of W_O
    seed: int
    kind: str  # "heavy" | "outlier" | "drift" | "plain"
    alpha: float = 0.5
    page: int = 16

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def units(self) -> int:
        return self.B * self.Hkv

    def scaled(self, **kw) -> "DecodeConfig":
        return dataclasses.replace(self, **kw)


# Tiny single-layer decode (fp16, GQA 4, 2K context, 25 % full + 25 % INT2).
C1 = DecodeConfig("c1_tiny_2k", B=1, Hq=8, Hkv=2, D=64, ctx=2048, window=16,
                  full_windows=32, int2_windows=32, route_every=4, steps=16,
                  dtype="fp16", hidden=512, seed=1000, kind="heavy")
# Llama-3-8B-shaped layer, 32K context, batch 8: 2048 full + 4096 INT2 tokens per head.
C2 = DecodeConfig("c2_llama8b_32k_b8", B=8, Hq=32, Hkv=8, D=128, ctx=32768, window=32,
                  full_windows=64, int2_windows=128, route_every=16, steps=64,
                  dtype="bf16", hidden=4096, seed=1001, kind="outlier")
# Long-context drift stress: 128K context, GQA 5, tiers 10 % / 65 % / 25 % of 2048 windows.
C5 = DecodeConfig("c5_drift_128k", B=1, Hq=40, Hkv=8, D=128, ctx=131072, window=64,
                  full_windows=205, int2_windows=1331, route_every=16, steps=256,
                  dtype="bf16", hidden=5120, seed=1004, kind="drift")

DECODE_CONFIGS = {c.name: c for c in (C1, C2, C5)}


@dataclass
class DecodeInputs:
    """Prefill cache, output projection and the per-step decode inputs."""

    cfg: DecodeConfig
    units: list  # list of (b, kvh) drawn, in order
    K: np.ndarray  # [n_units][ctx][D] float32 (dtype-exact)
    V: np.ndarray  # [n_units][ctx][D]
    W_O: np.ndarray  # [Hq*D][hidden] float32 (dtype-exact)
    q: np.ndarray  # [steps][B][Hq][D]
    k_new: np.ndarray  # [steps][B][Hkv][D]
    v_new: np.ndarray  # [steps][B][Hkv][D]


def _drift_directions(cfg: DecodeConfig, kvh: int):
    """Eight unit directions d_k = normalize(0.5*g + n_k) and their centre windows."""
    r = _rng(cfg.seed, 0xD1F7, kvh)
    g = r.standard_normal(cfg.D)
    n = r.standard_normal((8, cfg.D))
    d = 0.5 * g[None, :] + n
    d /= np.linalg.norm(d, axis=1, keepdims=True)
    n_win = cfg.ctx // cfg.window
    centres = r.choice(n_win, size=8, replace=False)
    return d.astype(np.float32), centres


def draw_unit_cache(cfg: DecodeConfig, b: int, kvh: int):
    """Prefill K and V of one (batch, kv-head) unit: two [ctx][D] float32 arrays."""
    r = _rng(cfg.seed, 0xCAC4E, b, kvh)
    K = r.standard_normal((cfg.ctx, cfg.D), dtype=np.float32)
    V = r.standard_normal((cfg.ctx, cfg.D), dtype=np.float32)
    if cfg.kind == "heavy":
        # 32 random "heavy" key positions scaled x4.
        heavy = r.choice(cfg.ctx, size=min(32, cfg.ctx), replace=False)
        K[heavy] *= 4.0
    elif cfg.kind == "outlier":
        # 4 seeded outlier channels scaled x8 on K and on V.
        ch = r.choice(cfg.D, size=4, replace=False)
        K[:, ch] *= 8.0
        V[:, ch] *= 8.0
    elif cfg.kind == "drift":
        d, centres = _drift_directions(cfg, kvh)
        for k, c in enumerate(centres):
            K[c * cfg.window:(c + 1) * cfg.window] += 4.0 * d[k][None, :]
    elif cfg.kind != "plain":
        raise ValueError(cfg.kind)
    return to_dtype_values(K, cfg.dtype), to_dtype_values(V, cfg.dtype)


def draw_w_o(cfg: DecodeConfig) -> np.ndarray:
    """Output projection W_O [Hq*D][hidden], N(0, 1/(Hq*D)), rounded to the cache dtype."""
    r = _rng(cfg.seed, 0x3A0)
    rows = cfg.Hq * cfg.D
    w = r.standard_normal((rows, cfg.hidden), dtype=np.float32) * np.float32(1.0 / math.sqrt(rows))
    return to_dtype_values(w, cfg.dtype)


def draw_step_inputs(cfg: DecodeConfig):
    """Per-step query [S][B][Hq][D] and new key/value [S][B][Hkv][D]."""
    r = _rng(cfg.seed, 0x57E9)
    S = cfg.steps
    q = r.standard_normal((S, cfg.B, cfg.Hq, cfg.D), dtype=np.float32)
    k = r.standard_normal((S, cfg.B, cfg.Hkv, cfg.D), dtype=np.float32)
    v = r.standard_normal((S, cfg.B, cfg.Hkv, cfg.D), dtype=np.float32)
    if cfg.kind == "drift":
        # q_h = 24 * d_{c(s)} + N(0, I), c(s) = floor(s / 32) mod 8, per kv-head group.
        for kvh in range(cfg.Hkv):
            d, _ = _drift_directions(cfg, kvh)
            for s in range(S):
                c = (s // 32) % 8
                q[s, :, kvh * cfg.G:(kvh + 1) * cfg.G, :] += 24.0 * d[c][None, None, :]
    return (to_dtype_values(q, cfg.dtype), to_dtype_values(k, cfg.dtype),
            to_dtype_values(v, cfg.dtype))


def draw_decode_inputs(cfg: DecodeConfig, units=None) -> DecodeInputs:
    """Draw the prefill cache for ``units`` (default: all) plus W_O and step inputs."""
    if units is None:
        units = [(b, h) for b in range(cfg.B) for h in range(cfg.Hkv)]
    K = np.empty((len(units), cfg.ctx, cfg.D), np.float32)
    V = np.empty_like(K)
    for i, (b, h) in enumerate(units):
        K[i], V[i] = draw_unit_cache(cfg, b, h)
    q, k, v = draw_step_inputs(cfg)
    return DecodeInputs(cfg, list(units), K, V, draw_w_o(cfg), q, k, v)


# --------------------------------------------------------------------------
# CriticalKV one-shot selection workload
# --------------------------------------------------------------------------


@dataclass(frozen=True)
class CriticalConfig:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    n: int  # context length
    n_obs: int  # observation window (last positions used as queries)
    budget: int  # b per (batch, kv-head)
    hidden: int
    seed: int
    alpha: float = 0.5
    zipf: float = 1.1
    dtype: str = "bf16"

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def scaled(self, **kw) -> "CriticalConfig":
        return dataclasses.replace(self, **kw)


C3 = CriticalConfig("c3_criticalkv_64k", B=4, Hq=32, Hkv=8, D=128, n=65536, n_obs=32,
                    budget=2048, hidden=4096, seed=1002)


def draw_critical_unit(cfg: CriticalConfig, b: int, kvh: int):
    """K [n][D], V [n][D] and observation queries [G][n_obs][D] of one unit.

    Keys carry Zipf(1.1) relevance along a unit direction u:
    K_i = z_i - (u.z_i) u + ln(w_i) u with w_i = (pi_i + 1)^-1.1 for a random
    permutation pi, so that softmax(q.K/sqrt(D)) with q ~ sqrt(D) u follows the
    Zipf weights. Queries: q = sqrt(D) u + 0.05 N(0, I).
    """
    r = _rng(cfg.seed, 0xC817, b, kvh)
    D = cfg.D
    u = r.standard_normal(D)
    u /= np.linalg.norm(u)
    perm = r.permutation(cfg.n)
    lw = -cfg.zipf * np.log(perm.astype(np.float64) + 1.0)
    z = r.standard_normal((cfg.n, D), dtype=np.float32).astype(np.float64)
    K = z - np.outer(z @ u, u) + np.outer(lw, u)
    V = r.standard_normal((cfg.n, D), dtype=np.float32)
    q = math.sqrt(D) * u[None, None, :] + 0.05 * r.standard_normal((cfg.G, cfg.n_obs, D))
    return (to_dtype_values(K.astype(np.float32), cfg.dtype), to_dtype_values(V, cfg.dtype),
            to_dtype_values(q.astype(np.float32), cfg.dtype))


def draw_critical_w_o(cfg: CriticalConfig) -> np.ndarray:
    r = _rng(cfg.seed, 0x3A0)
    rows = cfg.Hq * cfg.D
    w = r.standard_normal((rows, cfg.hidden), dtype=np.float32) * np.float32(1.0 / math.sqrt(rows))
    return to_dtype_values(w, cfg.dtype)


# --------------------------------------------------------------------------
# DBTrimKV global top-M workload
# --------------------------------------------------------------------------


@dataclass(frozen=True)
class TrimConfig:
    name: str
    layers: int
    Hkv: int
    D: int
    len_lo: int
    len_hi: int
    t: int
    M: int
    seed: int
    page: int = 16
    dtype: str = "bf16"

    @property
    def heads(self) -> int:
        return self.layers * self.Hkv

    def scaled(self, **kw) -> "TrimConfig":
        return dataclasses.replace(self, **kw)


C4 = TrimConfig("c4_dbtrim_32x8", layers=32, Hkv=8, D=128, len_lo=8192, len_hi=24576,
                t=32768, M=1048576, seed=1003)


def draw_trim_meta(cfg: TrimConfig):
    """Per-head lengths, retention betas and positions.

    Lengths ~ U[len_lo, len_hi]; beta ~ Beta(8, 1) in float32; each head's
    positions are sorted distinct integers drawn uniformly from [0, t).
    Returns (lengths [heads] int32, beta list of float32 arrays, pos list of int32 arrays).
    """
    r = _rng(cfg.seed, 0x7819)
    lengths = r.integers(cfg.len_lo, cfg.len_hi + 1, size=cfg.heads).astype(np.int32)
    betas, poss = [], []
    for h in range(cfg.heads):
        n = int(lengths[h])
        betas.append(r.beta(8.0, 1.0, size=n).astype(np.float32))
        poss.append(np.sort(r.choice(cfg.t, size=n, replace=False)).astype(np.int32))
    return lengths, betas, poss


def draw_trim_kv_page(cfg: TrimConfig, head: int, page: int):
    """K/V of one 16-entry page of one head: float32 arrays [2][page][D]."""
    r = _rng(cfg.seed, 0x7A6E, head, page)
    kv = r.standard_normal((2, cfg.page, cfg.D), dtype=np.float32)
    return to_dtype_values(kv, cfg.dtype)


@dataclass
class TrimLayout:
    """A paged cache for the trim: per-head entries scattered over physical pages.

    lengths [H] int32; page_table [H][max_pages] int32 (-1 past a head's pages);
    beta_pages [P][page] float32 and pos_pages [P][page] int32 by physical page and slot
    (slots past a head's length hold beta 1, pos 0); betas/poss the per-head arrays in
    logical order (the same values).
    """
    lengths: np.ndarray
    page_table: np.ndarray
    beta_pages: np.ndarray
    pos_pages: np.ndarray
    betas: list
    poss: list

    @property
    def n_pages(self) -> int:
        return self.beta_pages.shape[0]


def trim_layout(cfg: TrimConfig, lengths=None, betas=None, poss=None) -> TrimLayout:
    """Lay the (drawn or given) per-head metadata out over a seeded permutation of pages."""
    if lengths is None:
        lengths, betas, poss = draw_trim_meta(cfg)
    lengths = np.asarray(lengths, dtype=np.int32)
    pg = cfg.page
    max_pages = max(1, -(-cfg.len_hi // pg))
    n_pages = [-(-int(n) // pg) for n in lengths]
    P = max(1, sum(n_pages))
    perm = _rng(cfg.seed, 0x9A6E).permutation(P).astype(np.int32)
    table = np.full((len(lengths), max_pages), -1, dtype=np.int32)
    beta_pages = np.ones((P, pg), dtype=np.float32)
    pos_pages = np.zeros((P, pg), dtype=np.int32)
    a = 0
    for h, n in enumerate(lengths):
        k = n_pages[h]
        phys = perm[a:a + k]
        a += k
        table[h, :k] = phys
        pad = k * pg - int(n)
        b = np.concatenate([np.asarray(betas[h], dtype=np.float32), np.ones(pad, np.float32)])
        q = np.concatenate([np.asarray(poss[h], dtype=np.int32), np.zeros(pad, np.int32)])
        beta_pages[phys] = b.reshape(k, pg)
        pos_pages[phys] = q.reshape(k, pg)
    return TrimLayout(lengths, table, beta_pages, pos_pages, list(betas), list(poss))


def draw_trim_kv_pool(cfg: TrimConfig, n_pages: int, device, dtype):
    """K/V of the whole page pool [P][2][page][D], N(0, 1) drawn with a seeded torch generator
    on `device` (1M-row slabs, so that no float32 copy of the pool is held at once)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(cfg.seed * 7919 + 0x7A6E)
    out = torch.empty((n_pages, 2, cfg.page, cfg.D), dtype=dtype, device=device)
    flat = out.view(-1, cfg.D)
    step = 1 << 20
    for a in range(0, flat.shape[0], step):
        b = min(a + step, flat.shape[0])
        flat[a:b] = torch.randn((b - a, cfg.D), generator=g, device=device, dtype=torch.float32).to(dtype)
    return out


# --------------------------------------------------------------------------
# QEvict diagnostics workloads (routing histories and ghost caches)
# --------------------------------------------------------------------------

# tier encoding of a window (the library's QE_TIER_* values)
TIER_EVICTED, TIER_INT2, TIER_FULL, TIER_TAIL = 0, 1, 2, 3


@dataclass(frozen=True)
class DiagConfig:
    """Inputs of the QEvict diagnostics: a history of tier maps over ``events`` routing events
    and, at the last event, one decode step's queries over a ghost cache that holds every one
    of the ``n`` tokens' keys at their original precision. Shapes, dtype, key distribution
    and tier budgets come from ``base``."""

    name: str
    base: DecodeConfig
    n: int  # tokens at the last event (the tail window may be incomplete)
    events: int
    extra_windows: int = 3  # trailing windows never created: the map row is longer than needed
    n_pad: int = 0  # ghost-cache rows per unit beyond n (capacity for later tokens)

    @property
    def W(self) -> int:
        return -(-self.n // self.base.window) + self.extra_windows

    @property
    def n_stride(self) -> int:
        return self.n + self.n_pad

    def scaled(self, **kw) -> "DiagConfig":
        return dataclasses.replace(self, **kw)


# the c2 layer after 20 decode steps: 1024 complete windows of 32 plus a 20-token tail
DIAG_C2 = DiagConfig("diag_c2_llama8b_32k_b8", C2, n=32768 + 20, events=8)


def draw_tier_history(cfg: DiagConfig) -> np.ndarray:
    """Tier maps [events][B*Hkv][W] uint8 with the structure of a routing history.

    This draws data; it ranks windows by a random priority, not by any attention score. One
    window completes per event: at event e the first c_e = n // window - (events-1-e) windows
    are complete, window c_e is the tail (TAIL; at the last event only if n is not a multiple
    of the window) and later windows do not exist yet (EVICTED). Among the complete windows not
    evicted at an earlier event, the full_windows of highest priority are FULL, the next
    int2_windows INT2 and the rest EVICTED for good. A window's priority starts N(0, 1) and
    moves as p <- 0.8 p + 0.6 N(0, 1) between events, so windows leave and re-enter the full
    tier.
    """
    b = cfg.base
    U, W, w = b.units, cfg.W, b.window
    out = np.zeros((cfg.events, U, W), dtype=np.uint8)
    last_complete = cfg.n // w
    for u in range(U):
        r = _rng(b.seed, 0xD1A6, u)
        prio = r.standard_normal(W)
        gone = np.zeros(W, dtype=bool)
        for e in range(cfg.events):
            if e:
                prio = 0.8 * prio + 0.6 * r.standard_normal(W)
            c = max(0, last_complete - (cfg.events - 1 - e))
            cand = np.nonzero(~gone[:c])[0]
            order = cand[np.argsort(-prio[cand], kind="stable")]
            row = out[e, u]
            row[order[:b.full_windows]] = TIER_FULL
            row[order[b.full_windows:b.full_windows + b.int2_windows]] = TIER_INT2
            ev = order[b.full_windows + b.int2_windows:]
            row[ev] = TIER_EVICTED
            gone[ev] = True
            if c < W and (e < cfg.events - 1 or cfg.n % w):
                row[c] = TIER_TAIL
    return out


def draw_ghost_keys(cfg: DiagConfig, b: int, kvh: int) -> np.ndarray:
    """Ghost cache of one unit: the keys of all n tokens [n][D] (dtype-exact float32), drawn
    like the decode prefill cache of ``base`` at context n."""
    K, _ = draw_unit_cache(cfg.base.scaled(ctx=cfg.n), b, kvh)
    return K


def draw_diag_queries(cfg: DiagConfig) -> np.ndarray:
    """The step's queries [B][Hq][D]: the first decode step's q of ``base``."""
    return draw_step_inputs(cfg.base.scaled(steps=1))[0][0]


# --------------------------------------------------------------------------
# SEKV workloads (surprisal per token)
# --------------------------------------------------------------------------

# anchor threshold for Exponential(1) surprisal: P(H >= ln 10) = 1/10, so about 10 % of the
# tokens are anchors and spans average about 9 tokens
SEKV_TAU = math.log(10.0)


def draw_surprisal(cfg: DecodeConfig, n: int) -> np.ndarray:
    """Per-token surprisal [B][n] float32, Exponential(1): a stand-in for -log p(x_t | x_<t)
    of a language model, which needs trained weights."""
    r = _rng(cfg.seed, 0x5E4B)
    return r.exponential(size=(cfg.B, n)).astype(np.float32)
