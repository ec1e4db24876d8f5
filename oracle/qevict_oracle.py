"""Float64 CPU oracle of the tiered-KV decode path (TEST INFRASTRUCTURE ONLY).

Imported only by tests, ``__graft_entry__.smoke()`` and the CPU legs of
``bench.py``. It shares no code with the CUDA path and imports nothing from the
product package.

Everything is float64 except where floating point decides an integer: the INT2
code of an element and the fp16 scale/zero are decided in float32 with
round-to-nearest-even, exactly as written below, so that the CUDA path can take
the same decisions in the same precision.

Pins (tests that tie each function to something other than itself):

* attend -- brute force with scalar ``math.exp`` loops; uniform-key and
  single-token closed forms; G=1 reduces to plain multi-head attention.
* int2_quantize -- inputs already on the grid {z, z+s, z+2s, z+3s} round-trip
  exactly; a constant group gives s = 0 and all codes 0; hand-worked groups in
  ``tests/golden/int2_groups.txt``.
* vwo_l1norm -- W_O = identity reduces to ||V_i||_1; permutation/sign
  invariance; hand-worked case.
* two_stage -- exhaustive enumeration of subsets on small sets; hand-worked
  routing fixture in ``tests/golden/two_stage.txt``.
* QEvictUnit -- per-step mass invariant (sum over live windows = G);
  write-once ledger (demote -> promote -> demote yields identical codes);
  with budgets covering every window it reduces to plain attention; a hand-worked
  two-head, two-window step with a different W_O slice per head fixes the mass and the
  perturbation accumulation (``tests/golden/qevict_pert.txt``).
* observation_mass -- brute force; sum over keys of A = G * n_obs.
* trim_global_topm -- closed forms: constant beta keeps the most recent
  entries, equal age keeps the larger beta, beta = 1 everywhere ties and keeps
  the lowest flat indices; compared with ``np.argsort`` on tiny sets.
* output_perturbation -- a hand-worked three-token case, unprojected and projected
  through W_O^h (``tests/golden/output_perturbation.txt``); the full set gives 0.
* route_global -- one unit reduces to the unit's own routing; budgets covering
  every window evict nothing; equal scores across units go to the earlier unit;
  a hand-worked two-unit case (``tests/golden/route_global.txt``).
* sekv_segment / sekv_summaries / sekv_attend -- a hand-worked segmentation and a
  hand-worked weighted mean; a span of identical tokens, summarised with its size
  correction, gives exactly the attention of its tokens; every span expanded, or every
  token an anchor, is plain attention; a zero-surprisal span falls back to the plain mean;
  sekv_gates -- a hand-worked two-head case where the maximum over heads, the mean and
  the 1/sqrt(D) scale all differ (``tests/golden/sekv_gates.txt``).
* tier_diagnostics -- hand-worked two-unit event sequence in
  ``tests/golden/diag_tiers.txt``; a constant sequence has no change and no exit;
  a window alternating FULL/INT2 counts every exit and re-entry once per event and
  once per window; TAIL->FULL and first entries are not re-entries.
* future_missed_mass -- brute force with scalar ``math.exp`` loops; q = 0 gives
  the evicted share of tokens; no evicted window gives 0 and all evicted gives 1;
  a hand-worked four-token case with p proportional to 1:2:3:4.
"""
from __future__ import annotations

import math

import numpy as np

EVICTED, INT2, FULL, TAIL = 0, 1, 2, 3
GROUP = 16  # INT2 group: 16 consecutive head-dim elements of one token

# ---------------------------------------------------------------------------
# dtype helpers (oracle-private; not shared with any other module)
# ---------------------------------------------------------------------------


def _f32_to_bf16(x32: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 round-to-nearest-even, returned as float64 values."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def round_to_cache_dtype(x32: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values once to the cache dtype; float64 result."""
    x32 = np.asarray(x32, dtype=np.float32)
    if dtype == "bf16":
        return _f32_to_bf16(x32)
    if dtype == "fp16":
        return x32.astype(np.float16).astype(np.float64)
    raise ValueError(dtype)


# ---------------------------------------------------------------------------
# attention ("Resumo Técnico: QEvict", Implementação: GQA decode path)
# ---------------------------------------------------------------------------


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray):
    """Softmax attention of one query head over n keys.

    s_i = q.K_i / sqrt(D); p = softmax(s) (max-subtracted); o = sum_i p_i V_i.
    Returns (o [D], p [n]).
    """
    D = q.shape[-1]
    s = (K @ q) / math.sqrt(D)
    s = s - s.max()
    e = np.exp(s)
    p = e / e.sum()
    return p @ V, p


# ---------------------------------------------------------------------------
# INT2 recoverable tier ("Resumo Técnico: QEvict", Metodologia 2)
# ---------------------------------------------------------------------------


def int2_quantize(x: np.ndarray):
    """Asymmetric INT2 quantisation of [T][D] values in groups of 16 elements.

    Per group (16 consecutive head-dim elements of one token):
      mn, mx = min, max                          (exact)
      s = fp16( f32(mx - mn) / 3 )               (float32 ops, RNE to fp16)
      z = fp16( mn )
      code = clamp( rint( f32(x - z) / s ), 0, 3 ), code = 0 where s == 0
    All operations are float32 with round-to-nearest-even (rint: half to even).
    Returns (codes uint8 [T][D], s float16 [T][D/16], z float16 [T][D/16]).
    """
    T, D = x.shape
    g = np.asarray(x, dtype=np.float32).reshape(T, D // GROUP, GROUP)
    mn = g.min(axis=-1)
    mx = g.max(axis=-1)
    s16 = ((mx - mn) / np.float32(3.0)).astype(np.float16)
    z16 = mn.astype(np.float16)
    s32 = s16.astype(np.float32)[..., None]
    z32 = z16.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (g - z32) / s32
    codes = np.clip(np.rint(t), 0, 3)
    codes = np.where(s32 == 0, 0, codes).astype(np.uint8)
    return codes.reshape(T, D), s16, z16


def int2_dequantize(codes: np.ndarray, s16: np.ndarray, z16: np.ndarray) -> np.ndarray:
    """x_hat = code * s + z, exact in float64. Shapes as returned by int2_quantize."""
    T, D = codes.shape
    c = codes.reshape(T, D // GROUP, GROUP).astype(np.float64)
    x = c * s16.astype(np.float64)[..., None] + z16.astype(np.float64)[..., None]
    return x.reshape(T, D)


def int2_promote_values(codes, s16, z16, dtype: str) -> np.ndarray:
    """Values a promoted window holds in the full-precision tier.

    The full tier stores the cache dtype, so dequant(code) is rounded to it:
    first to float32 (one rounding of the exact code*s+z), then to fp16/bf16.
    """
    x32 = int2_dequantize(codes, s16, z16).astype(np.float32)
    return round_to_cache_dtype(x32, dtype)


# ---------------------------------------------------------------------------
# projected-value norms ("Resumo Técnico: CriticalKV", Framework Teórico)
# ---------------------------------------------------------------------------


def vwo_l1norm(V: np.ndarray, W_O: np.ndarray, heads, D: int, chunk: int = 4096) -> np.ndarray:
    """N[i, j] = || V_i @ W_O[h_j*D:(h_j+1)*D, :] ||_1 for each query head h_j.

    V: [n][D]; W_O: [Hq*D][hidden] with y = concat_h(o_h) @ W_O, so W_O^h is the
    row block h*D .. h*D+D-1. Returns [n][len(heads)] float64.
    """
    V = np.asarray(V, dtype=np.float64)
    out = np.empty((V.shape[0], len(heads)))
    for j, h in enumerate(heads):
        Wh = np.asarray(W_O[h * D:(h + 1) * D, :], dtype=np.float64)
        for a in range(0, V.shape[0], chunk):
            out[a:a + chunk, j] = np.abs(V[a:a + chunk] @ Wh).sum(axis=1)
    return out


# ---------------------------------------------------------------------------
# two-stage selection ("Resumo Técnico: CriticalKV", Algoritmo, Etapas 1 e 2)
# ---------------------------------------------------------------------------


def top_b(ids: np.ndarray, score: np.ndarray, b: int) -> np.ndarray:
    """The b ids with the highest score; ties go to the lower id."""
    ids = np.asarray(ids)
    if b <= 0 or ids.size == 0:
        return ids[:0]
    order = np.lexsort((ids, -score[ids]))
    return ids[order[:b]]


def two_stage(ids: np.ndarray, attn: np.ndarray, pert: np.ndarray, b: int, alpha: float):
    """Two-stage greedy selection of b items out of ``ids``.

    If |ids| <= b every item is kept. Otherwise b' = floor(alpha*b) items with
    the highest attention score are taken first, then b - b' items with the
    highest perturbation score among the rest. ``attn`` and ``pert`` are indexed
    by id. Returns (stage1 ids, stage2 ids).
    """
    ids = np.asarray(ids)
    if ids.size <= b:
        return ids.copy(), ids[:0]
    b1 = int(math.floor(alpha * b))
    s1 = top_b(ids, attn, b1)
    rest = np.setdiff1d(ids, s1, assume_unique=True)
    s2 = top_b(rest, pert, b - b1)
    return s1, s2


# ---------------------------------------------------------------------------
# QEvict unit ("Resumo Técnico: QEvict", Metodologia / Mecanismos Principais)
# ---------------------------------------------------------------------------


class QEvictUnit:
    """One (batch, kv-head) unit of the window-routed three-tier cache.

    State per window: tier (FULL / INT2 / EVICTED / TAIL), cumulative attention
    mass and cumulative perturbation score, and the write-once INT2 ledger entry.
    Per token: the values attention uses (``Keff``/``Veff``), the values the
    full tier stores (``Kst``/``Vst``) and the projected-value norms n[h].

    Readings where the pages are silent:
    the tail (newest, incomplete) window is always full precision, outside the
    budget and not routed; scores accumulate undecayed from step 0; evicted
    windows never return; routing runs after attention on steps s % R == 0;
    per-kv-head scores are sums over the G query heads of the group.
    """

    def __init__(self, K0, V0, W_O, kvh: int, G: int, window: int, full_windows: int,
                 int2_windows: int, alpha: float, dtype: str, max_tokens: int):
        K0 = np.asarray(K0, dtype=np.float64)
        V0 = np.asarray(V0, dtype=np.float64)
        n0, D = K0.shape
        self.D, self.G, self.w = D, G, window
        self.F, self.Q, self.alpha, self.dtype = full_windows, int2_windows, alpha, dtype
        self.heads = [kvh * G + j for j in range(G)]
        self.W_O = W_O
        nw = (max_tokens + window - 1) // window
        self.Kst = np.zeros((max_tokens, D))
        self.Vst = np.zeros((max_tokens, D))
        self.Keff = np.zeros((max_tokens, D))
        self.Veff = np.zeros((max_tokens, D))
        self.norms = np.zeros((max_tokens, G))
        self.tier = np.full(nw, EVICTED, dtype=np.int8)
        self.mass = np.zeros(nw)
        self.pert = np.zeros(nw)
        self.ledger = {}
        self.n = n0
        self.Kst[:n0], self.Vst[:n0] = K0, V0
        self.Keff[:n0], self.Veff[:n0] = K0, V0
        self.norms[:n0] = vwo_l1norm(V0, W_O, self.heads, D)
        self.tier[: n0 // window] = FULL
        if n0 % window:
            self.tier[n0 // window] = TAIL
        self.last_route = None

    # -- helpers --------------------------------------------------------------
    def tokens(self, w: int) -> slice:
        return slice(w * self.w, min((w + 1) * self.w, self.n))

    def live_windows(self) -> np.ndarray:
        # windows past the newest token are initialised EVICTED and become TAIL on append
        return np.nonzero(self.tier != EVICTED)[0]

    def live_tokens(self) -> np.ndarray:
        return np.concatenate([np.arange(self.tokens(w).start, self.tokens(w).stop)
                               for w in self.live_windows()])

    # -- one decode step ------------------------------------------------------
    def append(self, k, v):
        """Write the new token's K/V at position n and compute its norms n_h."""
        i = self.n
        self.Kst[i], self.Vst[i] = k, v
        self.Keff[i], self.Veff[i] = k, v
        self.norms[i] = vwo_l1norm(np.asarray(v, dtype=np.float64)[None, :], self.W_O,
                                   self.heads, self.D)[0]
        self.n += 1
        w = i // self.w
        self.tier[w] = FULL if self.n % self.w == 0 else TAIL

    def attend_and_score(self, qG):
        """Attention of the G query heads over every live token, plus scoring.

        mass_w += sum_h sum_{i in w} p_{h,i};  pert_w += sum_h sum_{i in w} p_{h,i} n_{h,i}.
        Returns o [G][D] and the per-window mass added at this step.
        """
        idx = self.live_tokens()
        K, V = self.Keff[idx], self.Veff[idx]
        win = idx // self.w
        o = np.empty((self.G, self.D))
        step_mass = np.zeros_like(self.mass)
        for j in range(self.G):
            o[j], p = attend(np.asarray(qG[j], dtype=np.float64), K, V)
            np.add.at(step_mass, win, p)
            np.add.at(self.pert, win, p * self.norms[idx, j])
        self.mass += step_mass
        return o, step_mass

    def route(self):
        """Full = TwoStage(L, F); INT2 = TwoStage(L minus Full, Q); the rest is evicted."""
        L = np.nonzero((self.tier == FULL) | (self.tier == INT2))[0]
        f1, f2 = two_stage(L, self.mass, self.pert, self.F, self.alpha)
        full = np.concatenate([f1, f2])
        rest = np.setdiff1d(L, full, assume_unique=True)
        q1, q2 = two_stage(rest, self.mass, self.pert, self.Q, self.alpha)
        int2 = np.concatenate([q1, q2])
        new = {int(w): EVICTED for w in L}
        new.update({int(w): FULL for w in full})
        new.update({int(w): INT2 for w in int2})
        self.last_route = dict(L=L, full=(f1, f2), int2=(q1, q2))
        self.apply(new)
        return new

    def apply(self, new: dict):
        """Tier transitions with the write-once ledger.

        FULL->INT2 quantises the stored values only if the window has no ledger
        entry yet; otherwise the entry is reused. INT2->FULL writes
        dequant(ledger) rounded to the cache dtype into the full tier and keeps
        the entry. ->EVICTED drops the data and the entry for good.
        """
        for w, t in sorted(new.items()):
            old = self.tier[w]
            sl = self.tokens(w)
            if old == FULL and t == INT2:
                if w not in self.ledger:
                    self.ledger[w] = (int2_quantize(self.Kst[sl]), int2_quantize(self.Vst[sl]))
                (ck, sk, zk), (cv, sv, zv) = self.ledger[w]
                self.Keff[sl] = int2_dequantize(ck, sk, zk)
                self.Veff[sl] = int2_dequantize(cv, sv, zv)
            elif old == INT2 and t == FULL:
                (ck, sk, zk), (cv, sv, zv) = self.ledger[w]
                self.Kst[sl] = int2_promote_values(ck, sk, zk, self.dtype)
                self.Vst[sl] = int2_promote_values(cv, sv, zv, self.dtype)
                self.Keff[sl], self.Veff[sl] = self.Kst[sl], self.Vst[sl]
            elif t == EVICTED:
                self.ledger.pop(w, None)
            self.tier[w] = t

    def step(self, s: int, qG, k, v, route_every: int):
        self.append(k, v)
        o, _ = self.attend_and_score(qG)
        routed = None
        if s % route_every == 0:
            routed = self.route()
        return o, routed


def route_global(units, full_windows: int, int2_windows: int, alpha: float):
    """One routing event of a sequence under global budgets across layers and kv heads.

    "Make Each Token Count", Metodologia 3 (Orçamento Global: one budget over every layer and
    head instead of a fixed share per head) applied to the window tiers of "Resumo Técnico:
    QEvict", Metodologia: the live (FULL or INT2) windows of all ``units`` compete together,
    Full = TwoStage(L, F); INT2 = TwoStage(L minus Full, Q); the rest is evicted, and each unit
    applies its part with the write-once ledger. ``units`` are the QEvictUnit of one sequence
    in flat order (layer-major, then kv head); window w of unit k has the flat id k * W + w
    (W windows per unit), and ties go to the lower flat id. Returns the per-unit assignments
    and the selection itself (candidates, the picks of each stage, the flat scores).
    """
    W = len(units[0].tier)
    mass = np.concatenate([u.mass for u in units])
    pert = np.concatenate([u.pert for u in units])
    tiers = np.concatenate([u.tier for u in units])
    L = np.nonzero((tiers == FULL) | (tiers == INT2))[0]
    f1, f2 = two_stage(L, mass, pert, full_windows, alpha)
    full = np.concatenate([f1, f2])
    rest = np.setdiff1d(L, full, assume_unique=True)
    q1, q2 = two_stage(rest, mass, pert, int2_windows, alpha)
    new = {int(j): EVICTED for j in L}
    new.update({int(j): FULL for j in full})
    new.update({int(j): INT2 for j in np.concatenate([q1, q2])})
    per_unit = [dict() for _ in units]
    for j, t in new.items():
        per_unit[j // W][j % W] = t
    for k, u in enumerate(units):
        u.apply(per_unit[k])
    return per_unit, dict(L=L, full=(f1, f2), int2=(q1, q2), mass=mass, pert=pert, W=W)


# ---------------------------------------------------------------------------
# CriticalKV with an observation window ("Resumo Técnico: CriticalKV", Algoritmo)
# ---------------------------------------------------------------------------


def observation_mass(q_obs: np.ndarray, K: np.ndarray) -> np.ndarray:
    """A[h, i] = sum_j softmax_j(q_{h,j}.K / sqrt(D))_i over the observation queries.

    q_obs [G][n_obs][D]: the queries at the last n_obs context positions; query j
    sits at position n - n_obs + j and attends causally to keys 0..n-n_obs+j.
    Returns A [G][n].
    """
    G, n_obs, D = q_obs.shape
    n = K.shape[0]
    K = np.asarray(K, dtype=np.float64)
    A = np.zeros((G, n))
    for h in range(G):
        for j in range(n_obs):
            last = n - n_obs + j + 1
            s = (K[:last] @ np.asarray(q_obs[h, j], dtype=np.float64)) / math.sqrt(D)
            e = np.exp(s - s.max())
            A[h, :last] += e / e.sum()
    return A


def criticalkv_select(A: np.ndarray, N: np.ndarray, b: int, alpha: float):
    """Stage 1 on sum_h A[h,i]; stage 2 on sum_h A[h,i] * N[i,h]. Returns (s1, s2, a, p)."""
    a = A.sum(axis=0)
    p = (A * N.T).sum(axis=0)
    ids = np.arange(a.size)
    s1, s2 = two_stage(ids, a, p, b, alpha)
    return s1, s2, a, p


# ---------------------------------------------------------------------------
# DBTrimKV global top-M ("Make Each Token Count", Metodologia 2-4)
# ---------------------------------------------------------------------------


def retention_log(beta: np.ndarray, pos: np.ndarray, t: int) -> np.ndarray:
    """log r_{t,i} = (t - i) * ln(beta_i), float64."""
    return (t - np.asarray(pos, dtype=np.float64)) * np.log(np.asarray(beta, dtype=np.float64))


def trim_global_topm(betas, poss, t: int, M: int):
    """Keep the M entries with the highest log r over all heads (ties: lower flat index).

    betas/poss: per-head arrays in head order; the flat index runs over heads
    first, then entries. Returns (keep masks per head, new lengths, all keys).
    """
    keys = np.concatenate([retention_log(b, p, t) for b, p in zip(betas, poss)])
    flat = np.arange(keys.size)
    order = np.lexsort((flat, -keys))
    keep = np.zeros(keys.size, dtype=bool)
    keep[order[:M]] = True
    masks, lens, a = [], [], 0
    for b in betas:
        m = keep[a:a + b.size]
        masks.append(m)
        lens.append(int(m.sum()))
        a += b.size
    return masks, np.array(lens, dtype=np.int64), keys


# ---------------------------------------------------------------------------
# output perturbation ("Resumo Técnico: CriticalKV", Definição de Perturbação)
# ---------------------------------------------------------------------------


def output_perturbation(q, K, V, subset, W_O_h=None) -> float:
    """L = ||o - o_hat||_1 between full-cache and subset attention (optionally projected)."""
    o, _ = attend(q, K, V)
    oh, _ = attend(q, K[subset], V[subset])
    d = o - oh
    if W_O_h is not None:
        d = d @ np.asarray(W_O_h, dtype=np.float64)
    return float(np.abs(d).sum())


# ---------------------------------------------------------------------------
# QEvict diagnostics ("Resumo Técnico: QEvict", Principais Contribuições 1:
# Massa Perdida Futura, LIR Global, Churn de Seleção)
# ---------------------------------------------------------------------------

# per-unit counter order shared by the tier diagnostics' results
DIAG_COUNTERS = ("live_prev", "changed", "exits", "reentries", "windows_exited", "windows_reentered")


def tier_diagnostics(tier_maps) -> dict:
    """Selection churn and latent importance reactivation over consecutive routing events.

    tier_maps: sequence of E integer arrays [U][W] (or [W]), the tier of every window
    after routing events 0..E-1 (EVICTED also marks windows that do not exist yet).
    Between events e-1 and e, per unit:
      live_prev  += #windows live (FULL or INT2) at e-1
      changed    += #of those whose tier at e differs from their tier at e-1
      exits      += #windows FULL at e-1 and not FULL at e  (leaving the active set)
      reentries  += #windows not FULL at e-1, FULL at e, that exited at an earlier event
      windows_exited / windows_reentered: windows whose first exit / first re-entry this is.
    churn = changed / live_prev and lir = windows_reentered / windows_exited, both pooled
    over every unit (nan when the denominator is 0). Returns {"per_unit": int64 [U][6] in
    DIAG_COUNTERS order, "churn": float, "lir": float}.
    """
    maps = [np.atleast_2d(np.asarray(m, dtype=np.int64)) for m in tier_maps]
    U, W = maps[0].shape
    counts = np.zeros((U, len(DIAG_COUNTERS)), dtype=np.int64)
    for u in range(U):
        exited = [False] * W
        reentered = [False] * W
        for e in range(1, len(maps)):
            for w in range(W):
                before, now = int(maps[e - 1][u, w]), int(maps[e][u, w])
                if before in (FULL, INT2):
                    counts[u, 0] += 1
                    if now != before:
                        counts[u, 1] += 1
                if before == FULL and now != FULL:
                    counts[u, 2] += 1
                    if not exited[w]:
                        exited[w] = True
                        counts[u, 4] += 1
                elif before != FULL and now == FULL and exited[w]:
                    counts[u, 3] += 1
                    if not reentered[w]:
                        reentered[w] = True
                        counts[u, 5] += 1
    tot = counts.sum(axis=0)
    churn = tot[1] / tot[0] if tot[0] else float("nan")
    lir = tot[5] / tot[4] if tot[4] else float("nan")
    return {"per_unit": counts, "churn": float(churn), "lir": float(lir)}


def future_missed_mass(qG: np.ndarray, K: np.ndarray, tiers: np.ndarray, window: int) -> float:
    """Share of the ghost attention that falls on evicted windows, averaged over the G heads.

    qG [G][D]: the step's query heads of one kv head; K [n][D]: the keys of every token so far
    at their original precision (the ghost cache: evicted windows included); tiers [W]: the
    tier of each window, token i lying in window i // window. For each head the ghost
    attention is the softmax of q.K_i / sqrt(D) over all n tokens; the result is
    (1/G) sum_h sum_{i in an EVICTED window} p_{h,i}, and 0 when n = 0.
    """
    K = np.asarray(K, dtype=np.float64)
    n = K.shape[0]
    if n == 0:
        return 0.0
    evicted = np.asarray(tiers)[np.arange(n) // window] == EVICTED
    G = len(qG)
    total = 0.0
    for h in range(G):
        _, p = attend(np.asarray(qG[h], dtype=np.float64), K, K)
        total += p[evicted].sum()
    return total / G


# ---------------------------------------------------------------------------
# SEKV mixed-resolution attention ("Resumo Técnico: SEKV", Metodologia 1-3)
# ---------------------------------------------------------------------------


def sekv_segment(H: np.ndarray, tau: float):
    """Entropy-guided segmentation (Metodologia 1): tokens whose surprisal H_t >= tau are
    anchors (kept at full resolution); every maximal run of non-anchor tokens is a span.
    Returns (anchor positions, spans as (start, end) pairs, end exclusive)."""
    H = np.asarray(H, dtype=np.float32)
    anchor = H >= np.float32(tau)
    anchors = np.nonzero(anchor)[0]
    spans = []
    t, n = 0, len(H)
    while t < n:
        if anchor[t]:
            t += 1
            continue
        s = t
        while t < n and not anchor[t]:
            t += 1
        spans.append((s, t))
    return anchors, spans


def sekv_summaries(K: np.ndarray, V: np.ndarray, H: np.ndarray, spans):
    """Span summaries (Metodologia 2, GPU-side coarse representation): the surprisal-weighted,
    normalised mean of the span's keys, k_S = sum_t H_t K_t / sum_t H_t, and the same mean of
    its values; the plain mean when the span's surprisal sums to 0. Returns (kbar, vbar, sizes)."""
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    H = np.asarray(H, dtype=np.float64)
    kbar = np.zeros((len(spans), K.shape[1]))
    vbar = np.zeros_like(kbar)
    sizes = np.array([e - s for s, e in spans], dtype=np.int64)
    for i, (s, e) in enumerate(spans):
        w = H[s:e]
        if w.sum() == 0:
            w = np.ones(e - s)
        kbar[i] = w @ K[s:e] / w.sum()
        vbar[i] = w @ V[s:e] / w.sum()
    return kbar, vbar, sizes


def sekv_gates(qG: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """Relevance of each span to the step's query heads (Metodologia 3, Roteamento): the
    largest q_h . k_S / sqrt(D) over the G heads of the kv head."""
    qG = np.asarray(qG, dtype=np.float64)
    if len(kbar) == 0:
        return np.zeros(0)
    return (qG @ kbar.T / math.sqrt(qG.shape[1])).max(axis=0)


def sekv_attend(qG, K, V, H, tau: float, theta: float, expand=None):
    """Mixed-resolution attention (Metodologia 3, Atenção de Resolução Mista) of the G query
    heads of one kv head: anchors contribute their K/V; a span whose gate reaches theta is
    expanded and contributes its tokens; every other span contributes its summary with the
    size correction ln|S| added to its score (it stands for |S| tokens). ``expand`` may give
    the expansion decisions instead of the gate. Returns (o [G][D], expanded [n_spans])."""
    qG = np.asarray(qG, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    anchors, spans = sekv_segment(H, tau)
    kbar, vbar, sizes = sekv_summaries(K, V, H, spans)
    if expand is None:
        expand = sekv_gates(qG, kbar) >= theta
    expand = np.asarray(expand, dtype=bool)
    keys, vals, bias = [K[anchors]], [V[anchors]], [np.zeros(len(anchors))]
    for i, (s, e) in enumerate(spans):
        if expand[i]:
            keys.append(K[s:e])
            vals.append(V[s:e])
            bias.append(np.zeros(e - s))
        else:
            keys.append(kbar[i:i + 1])
            vals.append(vbar[i:i + 1])
            bias.append(np.array([math.log(sizes[i])]))
    Kx, Vx, bx = np.concatenate(keys), np.concatenate(vals), np.concatenate(bias)
    D = qG.shape[1]
    o = np.empty((len(qG), D))
    for h, q in enumerate(qG):
        s = Kx @ q / math.sqrt(D) + bx
        s = s - s.max()
        p = np.exp(s)
        o[h] = (p / p.sum()) @ Vx
    return o, expand
