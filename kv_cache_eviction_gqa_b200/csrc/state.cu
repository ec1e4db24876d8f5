// Cache-state kernels: prefill load, token append, tail-window finalisation, two-stage
// routing with its tier transitions, and the write-once quantise / promote pass.
//
// "Resumo Técnico: QEvict" - Metodologia (three tiers: full precision, recoverable INT2,
// evicted, under a fixed budget) and Mecanismos Principais (window-level routing,
// cumulative scores, Rebaixamento / Promoção, write-once quantisation ledger).
// "Resumo Técnico: CriticalKV" - Algoritmo (two-stage selection: b' = alpha*b by
// attention mass, b - b' by the perturbation score).
//
// Every unit (batch, kv-head) owns a private slice of the page pool and of the ledger,
// with its own free stacks; one CTA per unit does that unit's bookkeeping, so no
// cross-unit atomics are needed and allocation is deterministic.
#include <math.h>

#include "append.cuh"
#include "int2.cuh"
#include "int2_block.cuh"
#include "qe_internal.cuh"

namespace {

constexpr int kRouteThreads = 512;
constexpr int kRankMax = 384;  // candidate sets up to this size are ranked by counting

// ---------------------------------------------------------------------------
// block helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

// Exclusive scan of one int per thread over the block; returns the block total in *total.
// `buf` needs 33 ints of shared memory.
__device__ int block_excl_scan(int v, int* buf, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int inc = warp_incl_scan(v, lane);
  if (lane == 31) buf[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int x = lane < nw ? buf[lane] : 0;
    int xi = warp_incl_scan(x, lane);
    if (lane < nw) buf[lane] = xi - x;
    if (lane == 31) buf[32] = xi;
  }
  __syncthreads();
  const int r = buf[warp] + inc - v;
  *total = buf[32];
  __syncthreads();
  return r;
}

// Exclusive prefix sums of N per-thread counts at once (one pass of barriers for all of them);
// buf holds at least N * 33 ints.
template <int N>
__device__ void block_excl_scan_n(const int (&v)[N], int* buf, int (&excl)[N], int (&total)[N]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int inc[N];
#pragma unroll
  for (int j = 0; j < N; ++j) {
    inc[j] = warp_incl_scan(v[j], lane);
    if (lane == 31) buf[j * 33 + warp] = inc[j];
  }
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int j = 0; j < N; ++j) {
      const int x = lane < nw ? buf[j * 33 + lane] : 0;
      const int xi = warp_incl_scan(x, lane);
      if (lane < nw) buf[j * 33 + lane] = xi - x;
      if (lane == 31) buf[j * 33 + 32] = xi;
    }
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < N; ++j) {
    excl[j] = buf[j * 33 + warp] + inc[j] - v[j];
    total[j] = buf[j * 33 + 32];
  }
  __syncthreads();
}

__device__ float block_sum(float v, float* buf) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) buf[warp] = v;
  __syncthreads();
  float r = 0.f;
  if (threadIdx.x == 0)
    for (int i = 0; i < nw; ++i) r += buf[i];
  __syncthreads();
  return r;  // valid in thread 0
}

// float -> uint32 whose unsigned order is the float order
__device__ __forceinline__ uint32_t ordered_bits(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------------------
// prefill
// ---------------------------------------------------------------------------
// K, V: [U][ctx][D]. Page p of unit u receives tokens 16p..16p+15 (zero past ctx).
__global__ void prefill_pages_kernel(DevState st, const uint4* K, const uint4* V, int ctx) {
  const int p = blockIdx.x, u = blockIdx.y;
  const int vec_per_row = st.D * 2 / 16;  // 16-byte vectors per row
  uint4* page = reinterpret_cast<uint4*>(st.pages + ((size_t)u * st.P + p) * st.page_bytes);
  for (int i = threadIdx.x; i < 2 * QE_PAGE * vec_per_row; i += blockDim.x) {
    const int kv = i / (QE_PAGE * vec_per_row), rem = i % (QE_PAGE * vec_per_row);
    const int r = rem / vec_per_row, c = rem % vec_per_row;
    const int tok = p * QE_PAGE + r;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (tok < ctx) val = (kv ? V : K)[((size_t)u * ctx + tok) * vec_per_row + c];
    page[i] = val;
  }
}

__global__ void prefill_meta_kernel(DevState st, const uint4* V, int ctx, uint4* tailV) {
  const int u = blockIdx.x, b = u / st.Hkv, kvh = u % st.Hkv;
  const int w = st.window, complete = ctx / w, n_pages = (ctx + QE_PAGE - 1) / QE_PAGE;
  const int n_win = (ctx + w - 1) / w;
  for (int i = threadIdx.x; i < n_win; i += blockDim.x) {
    st.win_tier[(size_t)u * st.Wmax + i] = i < complete ? QE_TIER_FULL : QE_TIER_TAIL;
    for (int k = 0; k < st.ppw; ++k) {
      const int pg = i * st.ppw + k;
      st.win_pages[((size_t)u * st.Wmax + i) * st.ppw + k] = pg < n_pages ? pg : -1;
    }
    if (i < complete) st.full_list[(size_t)u * st.Wmax + i] = i;
  }
  for (int i = threadIdx.x; i < st.P - n_pages; i += blockDim.x)
    st.page_free[(size_t)u * st.P + i] = st.P - 1 - i;
  for (int i = threadIdx.x; i < st.S; i += blockDim.x) st.slot_free[(size_t)u * st.S + i] = st.S - 1 - i;
  if (threadIdx.x == 0) {
    st.stacks[u * 4 + 0] = st.P - n_pages;
    st.stacks[u * 4 + 1] = st.S;
    st.stacks[u * 4 + 2] = complete;
    st.stacks[u * 4 + 3] = 0;
  }
  // V of an incomplete last window, staged for its norms when it completes
  const int vec_per_row = st.D * 2 / 16, tail = ctx - complete * w;
  for (int i = threadIdx.x; i < tail * vec_per_row; i += blockDim.x) {
    const int t = i / vec_per_row, c = i % vec_per_row;
    tailV[(((size_t)kvh * st.B + b) * w + t) * vec_per_row + c] =
        V[((size_t)u * ctx + complete * w + t) * vec_per_row + c];
  }
}

// ---------------------------------------------------------------------------
// append one token per unit at position pos
// ---------------------------------------------------------------------------
__global__ void append_kernel(DevState st, const uint4* k_new, const uint4* v_new, int pos,
                              uint4* tailV) {
  __shared__ int s_page;
  append_token(st, blockIdx.x, pos, k_new, v_new, tailV, &s_page);
}

// ---------------------------------------------------------------------------
// the tail window completed: store its norms, fold the deferred perturbation score,
// and move it into the full tier as a routing candidate
// ---------------------------------------------------------------------------
__global__ void finalize_kernel(DevState st, const float* tail_norm, int nparts, long long pstride, int tw) {
  const int u = blockIdx.x, b = u / st.Hkv, kvh = u % st.Hkv, w = st.window, G = st.G;
  __shared__ float red[32];
  float acc = 0.f;
  for (int i = threadIdx.x; i < w * G; i += blockDim.x) {
    const int t = i / G, h = i % G;
    // the column parts' partial row sums, added in part order
    const float* tn = tail_norm + (((size_t)kvh * st.B + b) * w + t) * G + h;
    float nrm = tn[0];
    for (int pp = 1; pp < nparts; ++pp) nrm += tn[pp * pstride];
    st.norms[((size_t)u * st.norm_pitch + (size_t)tw * w + t) * G + h] = nrm;
    float* tp = st.tail_p + (size_t)u * w * G + i;
    acc += *tp * nrm;
    *tp = 0.f;
  }
  const float sum = block_sum(acc, red);
  if (threadIdx.x == 0) {
    const size_t wi = (size_t)u * st.Wmax + tw;
    st.pert[wi] += sum;
    st.win_tier[wi] = QE_TIER_FULL;
    const int nf = st.stacks[u * 4 + 2];
    if (nf >= st.Wmax) {
      qe_record_error(st.status, QE_ERR_DEVICE_FAULT, u);
    } else {
      st.full_list[(size_t)u * st.Wmax + nf] = tw;
      st.stacks[u * 4 + 2] = nf + 1;
    }
  }
}

// ---------------------------------------------------------------------------
// routing
// ---------------------------------------------------------------------------
struct RouteArgs {
  DevState st;
  int32_t* xlist;   // [U][Wmax] windows to quantise
  int32_t* plist;   // [U][Wmax] windows to promote
  int32_t* xcount;  // [U][4]
  int F, Q, F1, Q1; // budgets and their stage-1 shares floor(alpha*b)
  int mode;         // 0: two-stage routing; 1: explicit targets for one unit; 2: decided tiers
  int unit;         // mode 1
  const int32_t* ids;  // mode 1: window ids
  int n_ids;           // mode 1
  int target;          // mode 1: QE_TIER_INT2 or QE_TIER_FULL
  // mode 2: new tier of window w of unit (b, kvh) at decided[b * dec_stride + kvh * Wmax + w]
  const uint8_t* decided;
  size_t dec_stride;
};

// Selection key: higher score first, then the lower window id; the candidate index rides in
// the low 12 bits (window ids < 2^20, candidates < 4096). Every real key is non-zero and keys
// of distinct candidates differ.
__device__ __forceinline__ unsigned long long sel_key(float score, int win, int idx) {
  return ((unsigned long long)ordered_bits(score) << 32) |
         ((unsigned long long)(0xFFFFFu - (uint32_t)win) << 12) | (uint32_t)idx;
}

// Number of keys in key[0..n) larger than x. A warp scans together and stops once every lane's
// count has reached `stop` (those candidates are out either way).
__device__ __forceinline__ int rank_of(const unsigned long long* key, int n, unsigned long long x, int stop) {
  int r = 0;
  for (int j0 = 0; j0 < n; j0 += 64) {
    const int j1 = min(n, j0 + 64);
    for (int j = j0; j < j1; ++j) r += key[j] > x ? 1 : 0;
    if (__all_sync(0xffffffffu, r >= stop)) break;
  }
  return r;
}

// Marks mark[i] |= 1 for the b largest of the non-zero keys key[0..n) (keys distinct), by a radix
// select from the most significant byte: a 256-bin histogram of the next byte among the keys
// that share the digits chosen so far, the bin where the count from the top reaches b, and so on
// until that bin holds exactly the keys still needed. hist: 256 ints of shared memory.
__device__ void radix_top(const unsigned long long* key, int n, int b, uint8_t* mark, int* hist) {
  __shared__ int s_digit, s_above, s_in;
  unsigned long long prefix = 0ull, mask = 0ull;
  int remaining = b;
  bool inclusive = false;
  for (int shift = 56; shift >= 0 && remaining > 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const unsigned long long k = key[i];
      if (k != 0ull && (k & mask) == prefix) atomicAdd(&hist[(int)((k >> shift) & 255ull)], 1);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane l sums bins 255 - 8l .. 248 - 8l (top down); the first lane whose running total from
      // the top reaches `remaining` holds the crossing bin
      const int l = threadIdx.x;
      int part = 0;
      for (int q = 0; q < 8; ++q) part += hist[255 - 8 * l - q];
      int incl = part;
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (l >= o) incl += v;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, incl >= remaining);
      const int lw = __ffs(hit) - 1;
      if (l == lw) {
        int above = incl - part;
        for (int q = 0; q < 8; ++q) {
          const int d = 255 - 8 * l - q, c = hist[d];
          if (above + c >= remaining) {
            s_digit = d;
            s_above = above;
            s_in = c;
            break;
          }
          above += c;
        }
      }
    }
    __syncthreads();
    const int d = s_digit, above = s_above, in = s_in;
    __syncthreads();
    prefix |= (unsigned long long)d << shift;
    mask |= 255ull << shift;
    remaining -= above;
    if (remaining == in) {  // the crossing bin holds exactly the keys still needed
      inclusive = true;
      break;
    }
  }
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const unsigned long long k = key[i], km = k & mask;
    if (k != 0ull && (km > prefix || (inclusive && km == prefix))) mark[i] = 1;
  }
  __syncthreads();
}

// Two-stage selection among candidates with inset[i]; selected ones get sel[i] = 1 and the
// stage-1 picks s1mark[i] = 1. A candidate's rank in a set is the number of members with a
// larger key, so stage 1 keeps the inset members of rank < b1 by k1 and stage 2 the members of
// the rest of rank < b - b1 by k2: exactly the top-b1 and top-(b - b1) (keys are distinct).
// `key` holds at least n 64-bit keys.
__device__ void two_stage_select(int n, const int32_t* cand, const float* k1, const float* k2,
                                 const uint8_t* inset, uint8_t* sel, uint8_t* s1mark, int b, int b1,
                                 int* ibuf, unsigned long long* key, int* hist) {
  int cnt_local = 0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) cnt_local += inset[i];
  int cnt;
  block_excl_scan(cnt_local, ibuf, &cnt);
  if (cnt <= b) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      sel[i] = inset[i];
      s1mark[i] = inset[i];
    }
    __syncthreads();
    return;
  }
  if (n > kRankMax) {
    // many candidates: radix select (a few histogram passes) instead of n^2 rank counts
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      key[i] = inset[i] ? sel_key(k1[i], cand[i], i) : 0ull;
      s1mark[i] = 0;
    }
    __syncthreads();
    if (b1 > 0) radix_top(key, n, b1, s1mark, hist);
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      key[i] = (inset[i] && !s1mark[i]) ? sel_key(k2[i], cand[i], i) : 0ull;
      sel[i] = s1mark[i];
    }
    __syncthreads();
    if (b - b1 > 0) radix_top(key, n, b - b1, sel, hist);
    return;
  }
  // stage 1: the b1 largest k1 among inset
  for (int i = threadIdx.x; i < n; i += blockDim.x) key[i] = inset[i] ? sel_key(k1[i], cand[i], i) : 0ull;
  __syncthreads();
  const int nn = (n + 31) / 32 * 32;  // whole warps take part in every rank scan
  for (int i = threadIdx.x; i < nn; i += blockDim.x) {
    const unsigned long long x = i < n ? key[i] : 0ull;
    const int r = rank_of(key, n, x, b1);
    if (i < n) s1mark[i] = (x != 0ull && r < b1) ? 1 : 0;
  }
  __syncthreads();
  // stage 2: the b - b1 largest k2 among inset minus stage 1
  for (int i = threadIdx.x; i < n; i += blockDim.x)
    key[i] = (inset[i] && !s1mark[i]) ? sel_key(k2[i], cand[i], i) : 0ull;
  __syncthreads();
  for (int i = threadIdx.x; i < nn; i += blockDim.x) {
    const unsigned long long x = i < n ? key[i] : 0ull;
    const int r = rank_of(key, n, x, b - b1);
    if (i < n) sel[i] = s1mark[i] | ((x != 0ull && r < b - b1) ? 1 : 0);
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kRouteThreads) route_kernel(RouteArgs a) {
  const DevState& st = a.st;
  const int u = a.mode == 1 ? a.unit : blockIdx.x;
  extern __shared__ __align__(16) uint8_t sm[];
  const int nf = st.stacks[u * 4 + 2], nq = st.stacks[u * 4 + 3], n = nf + nq;
  int NW = 1;  // key buffer capacity (power of two >= Wmax)
  while (NW < st.Wmax) NW <<= 1;
  unsigned long long* key = reinterpret_cast<unsigned long long*>(sm);
  int32_t* cand = reinterpret_cast<int32_t*>(key + NW);
  float* km = reinterpret_cast<float*>(cand + st.Wmax);
  float* kp = km + st.Wmax;
  uint8_t* oldt = reinterpret_cast<uint8_t*>(kp + st.Wmax);
  uint8_t* newt = oldt + st.Wmax;
  uint8_t* inset = newt + st.Wmax;
  uint8_t* sel = inset + st.Wmax;
  uint8_t* s1 = sel + st.Wmax;
  __shared__ int ibuf[33];
  __shared__ int sbuf[9 * 33];
  __shared__ float fbuf[32];
  __shared__ int hist[256];
  __shared__ int s_abort;
  if (threadIdx.x == 0) s_abort = 0;
  if (n > st.Wmax) {
    if (threadIdx.x == 0) qe_record_error(st.status, QE_ERR_DEVICE_FAULT, u);
    return;
  }
  const size_t ub = (size_t)u * st.Wmax;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int win = i < nf ? st.full_list[ub + i] : st.int2_list[ub + i - nf];
    cand[i] = win;
    km[i] = st.mass[ub + win];
    kp[i] = st.pert[ub + win];
    oldt[i] = i < nf ? QE_TIER_FULL : QE_TIER_INT2;
    newt[i] = QE_TIER_EVICTED;
  }
  __syncthreads();

  float stage1_mass = 0.f, all_mass = 0.f;
  if (a.mode == 0) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) inset[i] = 1;
    __syncthreads();
    two_stage_select(n, cand, km, kp, inset, sel, s1, a.F, a.F1, ibuf, key, hist);
    float s1m = 0.f, am = 0.f;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      if (sel[i]) newt[i] = QE_TIER_FULL;
      if (s1[i]) s1m += km[i];
      am += km[i];
      inset[i] = !sel[i];
    }
    stage1_mass = block_sum(s1m, fbuf);
    all_mass = block_sum(am, fbuf);
    two_stage_select(n, cand, km, kp, inset, sel, s1, a.Q, a.Q1, ibuf, key, hist);
    for (int i = threadIdx.x; i < n; i += blockDim.x)
      if (sel[i]) newt[i] = QE_TIER_INT2;
  } else if (a.mode == 2) {
    // tiers decided by a selection over several contexts (global budgets)
    const uint8_t* dec = a.decided + (size_t)(u / st.Hkv) * a.dec_stride + (size_t)(u % st.Hkv) * st.Wmax;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const int t = dec[cand[i]];
      if (t == QE_TIER_FULL || t == QE_TIER_INT2 || t == QE_TIER_EVICTED) {
        newt[i] = (uint8_t)t;
      } else {
        newt[i] = oldt[i];
        qe_record_error(st.status, QE_ERR_DEVICE_FAULT, u);
      }
    }
  } else {
    for (int i = threadIdx.x; i < n; i += blockDim.x) newt[i] = oldt[i];
    __syncthreads();
    for (int k = threadIdx.x; k < a.n_ids; k += blockDim.x) {
      const int id = a.ids[k];
      int found = -1;
      for (int i = 0; i < n; ++i)
        if (cand[i] == id) found = i;
      const int want_old = a.target == QE_TIER_INT2 ? QE_TIER_FULL : QE_TIER_INT2;
      if (found < 0 || oldt[found] != want_old)
        qe_record_error(st.status, QE_ERR_INVALID_ARG, id);
      else
        newt[found] = (uint8_t)a.target;
    }
  }
  __syncthreads();

  // ---- transitions: counts, then allocation (pops), then frees (pushes) ----
  // each thread owns a contiguous run of candidates so prefix sums stay in candidate order
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int i0 = threadIdx.x * per, i1 = min(n, i0 + per);
  // counts per thread: pages taken, new ledger slots, pages given back, slots given back,
  // promotions, full, INT2, demotions (first or reused), evictions
  int cnt[9] = {0, 0, 0, 0, 0, 0, 0, 0, 0};
  for (int i = i0; i < i1; ++i) {
    const int o = oldt[i], t = newt[i];
    const int slot = st.win_slot[ub + cand[i]];
    cnt[0] += (o == QE_TIER_INT2 && t == QE_TIER_FULL) ? st.ppw : 0;
    cnt[1] += (o == QE_TIER_FULL && t == QE_TIER_INT2 && slot < 0);
    cnt[2] += (o == QE_TIER_FULL && t != QE_TIER_FULL) ? st.ppw : 0;
    cnt[3] += (t == QE_TIER_EVICTED && slot >= 0);
    cnt[4] += (o == QE_TIER_INT2 && t == QE_TIER_FULL);
    cnt[5] += (t == QE_TIER_FULL);
    cnt[6] += (t == QE_TIER_INT2);
    cnt[7] += (o == QE_TIER_FULL && t == QE_TIER_INT2);
    cnt[8] += (t == QE_TIER_EVICTED);
  }
  int ex[9], tot[9];
  block_excl_scan_n<9>(cnt, sbuf, ex, tot);
  const int o_tp = ex[0], o_ts = ex[1], o_gp = ex[2], o_gs = ex[3], o_pr = ex[4], o_nf = ex[5], o_nq = ex[6];
  const int T_tp = tot[0], T_ts = tot[1], T_gp = tot[2], T_gs = tot[3], T_pr = tot[4], T_nf = tot[5],
            T_nq = tot[6], T_re = tot[7], T_ev = tot[8];
  const int ptop = st.stacks[u * 4 + 0], stop = st.stacks[u * 4 + 1];
  if (threadIdx.x == 0) {
    if (T_tp > ptop) {
      qe_record_error(st.status, QE_ERR_POOL_EXHAUSTED, u);
      s_abort = 1;
    } else if (T_ts > stop) {
      qe_record_error(st.status, QE_ERR_LEDGER_FULL, u);
      s_abort = 1;
    }
  }
  __syncthreads();
  if (s_abort) return;  // nothing was modified yet

  // pops
  {
    int tp = o_tp, ts = o_ts, pr = o_pr;
    for (int i = i0; i < i1; ++i) {
      const int o = oldt[i], t = newt[i], win = cand[i];
      if (o == QE_TIER_INT2 && t == QE_TIER_FULL) {
        for (int k = 0; k < st.ppw; ++k) {
          const int page = st.page_free[(size_t)u * st.P + ptop - 1 - (tp + k)];
          st.win_pages[(ub + win) * st.ppw + k] = page;
        }
        tp += st.ppw;
        a.plist[ub + pr++] = win;
      }
      if (o == QE_TIER_FULL && t == QE_TIER_INT2 && st.win_slot[ub + win] < 0) {
        const int slot = st.slot_free[(size_t)u * st.S + stop - 1 - ts];
        st.win_slot[ub + win] = slot;
        a.xlist[ub + ts] = win;
        ++ts;
      }
    }
  }
  __syncthreads();
  // pushes (freed pages and slots) on top of the shrunken stacks
  {
    const int ntop = ptop - T_tp, nstop = stop - T_ts;
    int gp = o_gp, gs = o_gs, f = o_nf, q = o_nq;
    for (int i = i0; i < i1; ++i) {
      const int o = oldt[i], t = newt[i], win = cand[i];
      if (o == QE_TIER_FULL && t != QE_TIER_FULL) {
        for (int k = 0; k < st.ppw; ++k)
          st.page_free[(size_t)u * st.P + ntop + gp + k] = st.win_pages[(ub + win) * st.ppw + k];
        gp += st.ppw;
      }
      if (t == QE_TIER_EVICTED) {
        const int slot = st.win_slot[ub + win];
        if (slot >= 0) {
          st.slot_free[(size_t)u * st.S + nstop + gs++] = slot;
          st.win_slot[ub + win] = -1;
        }
      }
      if (t == QE_TIER_FULL) st.full_list[ub + f++] = win;
      if (t == QE_TIER_INT2) st.int2_list[ub + q++] = win;
      st.win_tier[ub + win] = (uint8_t)t;
    }
  }
  if (threadIdx.x == 0) {
    st.stacks[u * 4 + 0] = ptop - T_tp + T_gp;
    st.stacks[u * 4 + 1] = stop - T_ts + T_gs;
    st.stacks[u * 4 + 2] = T_nf;
    st.stacks[u * 4 + 3] = T_nq;
    a.xcount[u * 4 + 0] = T_ts;
    a.xcount[u * 4 + 1] = T_pr;
    int32_t* rs = st.route_stats + u * 8;
    rs[0] = T_pr;
    rs[1] = T_ts;
    rs[2] = 0;  // filled below (demotions that reused a ledger entry)
    rs[4] = T_nf;
    rs[5] = T_nq;
    rs[7] = all_mass > 0.f ? (int)llrintf(1e6f * stage1_mass / all_mass) : 0;
  }
  // demotions that reused an entry, evictions
  if (threadIdx.x == 0) {
    st.route_stats[u * 8 + 2] = T_re - T_ts;
    st.route_stats[u * 8 + 3] = T_ev;
  }
}

// ---------------------------------------------------------------------------
// quantise (first demotion only) and promote
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  const T lo = Elem<T>::from_f(a), hi = Elem<T>::from_f(b);
  return static_cast<uint32_t>(*reinterpret_cast<const unsigned short*>(&lo)) |
         (static_cast<uint32_t>(*reinterpret_cast<const unsigned short*>(&hi)) << 16);
}
// Quantise (first demotion) and promote, one item = one (window, page) = one 16-token block of
// the window's ledger entry. The items of all units form one list (unit u's nx quantisations
// then np promotions, ppw pages each); block b of the grid takes items b, b + gridDim, ... .
// Each block is a pair of warps, warp 0 on the item's K rows and warp 1 on its V rows; the item's
// source arrives and its result leaves by bulk copies, the next item's copy overlapping the
// store of the current one, and many blocks per SM keep enough copies in flight.
//
// Quantisation, pass A (natural layout): lane l takes the (token, group) pairs l, l + 32, ...
// of its warp's tensor, reads the group's 16 elements, forms min and max with packed 16-bit
// min/max and builds the group's parameters once: fp16 scale and zero into the block's meta
// arrays, (-z, 1/s) for pass B. Pass B (block placement, int2_block.cuh): lane (r, t) computes
// the codes of its own positions with int2_code2_fast and stores its code words; positions the
// fast path cannot decide are marked in a bit mask and recomputed afterwards by IEEE division.
// Promotion: pass A turns each group's fp16 (s, z) into floats once; pass B rebuilds each element
// as f32(code * s + z) rounded to the cache dtype, in row-major page order.
constexpr int kApplyThreads = 64;

__device__ __forceinline__ void bulk_s2g(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_u32(src)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

template <typename T> __device__ __forceinline__ uint32_t min2_u32(uint32_t a, uint32_t b);
template <typename T> __device__ __forceinline__ uint32_t max2_u32(uint32_t a, uint32_t b);
template <> __device__ __forceinline__ uint32_t min2_u32<__nv_bfloat16>(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("min.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
template <> __device__ __forceinline__ uint32_t max2_u32<__nv_bfloat16>(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
template <> __device__ __forceinline__ uint32_t min2_u32<__half>(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("min.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
template <> __device__ __forceinline__ uint32_t max2_u32<__half>(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// A page's 32 rows (16 K then 16 V) sit in shared memory with a stride of D + 8 elements, so that
// the placement passes (lanes of one quad column on eight different rows) hit distinct banks;
// the group parameters use a stride of D/16 + 1 per token for the same reason.
template <int D>
constexpr int apply_row() { return D + 8; }
template <int D>
constexpr size_t apply_buf_bytes() {  // a padded page image (a block image is smaller)
  return (size_t)2 * QE_PAGE * apply_row<D>() * 2;
}
template <int D>
size_t apply_smem_bytes(int units) {
  return apply_buf_bytes<D>() + Int2Block<D>::BYTES + 2 * QE_PAGE * (D / 16 + 1) * 8 + 32 + 4 * (size_t)(units + 1);
}

// Replace the codes of the elements marked in mask (bit e; elements 0..7 in a, 8..15 in b, pairs
// of 16-bit values) in n by IEEE division: the path taken where the fast one cannot decide.
template <typename T>
__device__ __noinline__ uint32_t int2_group_codes_exact(uint32_t n, uint32_t mask, uint4 a, uint4 b, float s,
                                                        float z) {
  const uint32_t e2[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  for (int e = 0; e < 16; ++e) {
    if (!((mask >> e) & 1u)) continue;
    const uint32_t w = e2[e >> 1];
    const float x = (e & 1) ? Elem<T>::hi(w) : Elem<T>::lo(w);
    n = (n & ~(3u << (2 * e))) | (int2_code_exact(x, s, z) << (2 * e));
  }
  return n;
}

template <typename T, int D>
__global__ void __launch_bounds__(kApplyThreads) apply_kernel(DevState st, const int32_t* xlist,
                                                              const int32_t* plist, const int32_t* xcount,
                                                              int unit_only) {
  using BL = Int2Block<D>;
  constexpr int G8 = BL::G8, WPL = BL::WPL;
  constexpr int RS = apply_row<D>();          // row stride in shared memory (elements)
  constexpr int PAGES = (int)apply_buf_bytes<D>();  // a padded page image
  constexpr int NG = QE_PAGE * G8;            // groups per tensor and block
  constexpr int PS = G8 + 1;                  // parameter stride per token
  extern __shared__ __align__(16) uint8_t sm[];
  const int lane = threadIdx.x & 31, wq = threadIdx.x >> 5;  // wq: 0 K rows, 1 V rows
  const int r = lane >> 2, t4 = lane & 3;
  constexpr int BUFS = PAGES + BL::BYTES;      // the page image, then the block image
  float2* prm = reinterpret_cast<float2*>(sm + BUFS) + wq * QE_PAGE * PS;  // this warp's [16][PS]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + BUFS + 2 * QE_PAGE * PS * 8);
  int* info = reinterpret_cast<int*>(bars + 1);  // kind of the item whose source is being copied
  int* pre = reinterpret_cast<int*>(sm + BUFS + 2 * QE_PAGE * PS * 8 + 32);  // [units + 1]
  const int units = unit_only >= 0 ? 1 : st.U;
  const int ppw = st.ppw;

  // item prefix over units
  if (wq == 0) {
    int carry = 0;
    for (int c0 = 0; c0 < units; c0 += 32) {
      const int uu = c0 + lane;
      const int uid = unit_only >= 0 ? unit_only : uu;
      int v = uu < units ? (xcount[uid * 4 + 0] + xcount[uid * 4 + 1]) * ppw : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
      }
      if (uu < units) pre[uu + 1] = carry + v;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) {
      pre[0] = 0;
      mbar_init(&bars[0], 1);
      fence_mbar_init();
    }
  }
  __syncthreads();
  const int total = pre[units];
  const int n_items = (int)blockIdx.x < total ? (total - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;

  // Warp 0's lane l holds the addresses of the block's item kb + l (reloaded every 32 items):
  // kind (0 quantise, 1 promote, -1 invalid), the page and the block.
  int e_kind = -1;
  uint4* e_page = nullptr;
  uint4* e_blk = nullptr;
  int kb = -32;
  auto load_items = [&](int base) {
    kb = base;
    e_kind = -1;
    if (base + lane >= n_items) return;
    const int it = (int)blockIdx.x + (base + lane) * (int)gridDim.x;
    int lo = 0, hi = units;  // pre[lo] <= it < pre[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pre[mid] <= it) lo = mid;
      else hi = mid;
    }
    const int u = unit_only >= 0 ? unit_only : lo;
    const int local = it - pre[lo], item = local / ppw, pg = local % ppw;
    const int nx = xcount[u * 4 + 0];
    const size_t ub = (size_t)u * st.Wmax;
    const int win = item < nx ? xlist[ub + item] : plist[ub + item - nx];
    if (win < 0 || win >= st.Wmax) {
      qe_record_error(st.status, QE_ERR_DEVICE_FAULT, u);
      return;
    }
    const int slot = st.win_slot[ub + win];
    const int page = st.win_pages[(ub + win) * ppw + pg];
    if (slot < 0 || slot >= st.S || page < 0 || page >= st.P) {
      qe_record_error(st.status, QE_ERR_DEVICE_FAULT, u);
      return;
    }
    e_kind = item < nx ? 0 : 1;
    e_blk = reinterpret_cast<uint4*>(st.slots + ((size_t)u * st.S + slot) * st.slot_bytes + (size_t)pg * BL::BYTES);
    e_page = reinterpret_cast<uint4*>(st.pages + ((size_t)u * st.P + page) * st.page_bytes);
  };
  // Two buffers, a padded page image and a block image: an item's source arrives by bulk copy in
  // one (the page to quantise, row by row into the padded layout, or the ledger block to
  // dequantise) and its result is built in the other, which the bulk store then reads. The next
  // item's copy is issued as soon as both warps are done with the current item, so it overlaps
  // the store; when its source buffer is the one the store is reading (the kinds differ), it
  // first waits for the store to have read it.
  uint4* dst = nullptr;  // warp 0: where the item's result goes
  uint4* dst_next = nullptr;
  uint32_t par = 0u;     // barrier parity (every thread; the control flow is uniform)
  bool pend = false;     // warp 0: a copy is in flight
  int store_kind = -1;   // warp 0: kind of the item whose store may still read its buffer
  uint8_t* pg_s = sm;           // the page image
  uint8_t* img = sm + PAGES;    // the block image
  auto issue = [&](int k) {  // warp 0
    if (k - kb >= 32) load_items(k - k % 32);
    const int src = k - kb;
    const int kind = __shfl_sync(0xffffffffu, e_kind, src);
    uint4* pgp = reinterpret_cast<uint4*>(__shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(e_page), src));
    uint4* blp = reinterpret_cast<uint4*>(__shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(e_blk), src));
    dst_next = kind == 0 ? blp : pgp;
    if (lane == 0) info[0] = kind;
    if (kind < 0) return;
    if (store_kind >= 0 && store_kind != kind) bulk_wait_read_all();  // the source buffer is free
    pend = true;
    fence_proxy_async_smem();
    if (kind == 0) {
      if (lane == 0) mbar_arrive_expect_tx(&bars[0], 2 * QE_PAGE * D * 2);
      __syncwarp();
      bulk_g2s(pg_s + lane * RS * 2, reinterpret_cast<const uint8_t*>(pgp) + lane * D * 2, D * 2, &bars[0]);
    } else if (lane == 0) {
      mbar_arrive_expect_tx(&bars[0], BL::BYTES);
      bulk_g2s(img, blp, BL::BYTES, &bars[0]);
    }
  };

  if (wq == 0 && n_items > 0) issue(0);
  bool ok = true;
  for (int k = 0; k < n_items; ++k) {
    __syncthreads();  // info[0] of item k is visible; both warps are past item k - 1
    const int kind = info[0];
    if (kind < 0) {  // uniform
      __syncthreads();  // every thread has read info[0] before the next issue rewrites it
      if (wq == 0 && k + 1 < n_items) issue(k + 1);
      continue;
    }
    const bool okw = mbar_wait_bounded(&bars[0], par, st.status, 3000);
    if (wq == 0) bulk_wait_read_all();  // the result buffer is free: the store of item k - 1 has read it
    ok = __syncthreads_and(okw ? 1 : 0) != 0;
    if (!ok) break;
    par ^= 1u;
    pend = false;
    dst = dst_next;
    T* rows = reinterpret_cast<T*>(pg_s) + wq * QE_PAGE * RS;  // this warp's 16 rows
    uint16_t* msc = reinterpret_cast<uint16_t*>(img + (wq ? BL::VS : BL::KS));  // scales
    uint16_t* mzr = reinterpret_cast<uint16_t*>(img + (wq ? BL::VZ : BL::KZ));  // zeros
    // position of a (token, group) scale / zero in the block's meta arrays
    auto s_at = [&](int tok, int g) { return g * QE_PAGE + (wq ? BL::fpos(tok) : BL::ppos(tok)); };
    auto z_at = [&](int tok, int g) { return wq ? g * QE_PAGE + BL::fpos(tok) : tok * G8 + g; };
    uint32_t* words = reinterpret_cast<uint32_t*>(img + (wq ? BL::VC : BL::KC)) + lane * WPL;
    if (kind == 0) {
      // ---- pass A: each group's min, max, parameters and 16 codes (natural order: element e
      // at bits 2e of the group's word), once ----
      uint32_t* nat = reinterpret_cast<uint32_t*>(prm);  // [16 tokens][PS] code words
#pragma unroll
      for (int k2 = 0; k2 < NG / 32; ++k2) {
        const int p = lane + 32 * k2, tok = p / G8, g = p % G8;
        // the two 16-byte halves, upper half first for g >= G8/2 so that a quarter-warp's loads
        // fall on distinct banks
        const uint4* src = reinterpret_cast<const uint4*>(rows + tok * RS + 16 * g);
        const int h = g >= G8 / 2 ? 1 : 0;
        const uint4 ha = src[h], hb = src[h ^ 1];
        const uint4 a = h ? hb : ha, b = h ? ha : hb;  // elements 0..7, 8..15
        const uint32_t mn = min2_u32<T>(min2_u32<T>(min2_u32<T>(a.x, a.y), min2_u32<T>(a.z, a.w)),
                                        min2_u32<T>(min2_u32<T>(b.x, b.y), min2_u32<T>(b.z, b.w)));
        const uint32_t mx = max2_u32<T>(max2_u32<T>(max2_u32<T>(a.x, a.y), max2_u32<T>(a.z, a.w)),
                                        max2_u32<T>(max2_u32<T>(b.x, b.y), max2_u32<T>(b.z, b.w)));
        const float fmn = fminf(Elem<T>::lo(mn), Elem<T>::hi(mn)), fmx = fmaxf(Elem<T>::lo(mx), Elem<T>::hi(mx));
        const Int2Group q(fmn, fmx);
        msc[s_at(tok, g)] = __half_as_ushort(q.sh);
        mzr[z_at(tok, g)] = __half_as_ushort(q.zh);
        const float2 pm = q.fast_params(fmn);
        const uint32_t e2[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint32_t n;
        uint32_t near = int2_group_codes_fast<T>(e2, pm, n);
        if (pm.x < 0.f) near = 0xFFFFu;
        if (near) n = int2_group_codes_exact<T>(n, near, a, b, q.s, q.z);
        nat[tok * PS + g] = n;
      }
      __syncwarp();
      // ---- pass B: the code words in block placement ----
      uint32_t w[WPL];
#pragma unroll
      for (int j = 0; j < WPL; ++j) w[j] = 0u;
      if (wq == 0) {
        // K: tokens r, 8 + r; elements 2t, 2t + 1, 8 + 2t, 9 + 2t of each group go to bits base,
        // 16 + base, base + 2, 18 + base of the word of the group pair
#pragma unroll
        for (int tb = 0; tb < 2; ++tb) {
#pragma unroll
          for (int g = 0; g < G8; ++g) {
            const uint32_t x = nat[(r + 8 * tb) * PS + g] >> (4 * t4);
            const uint32_t v = (x & 0x3u) | ((x >> 14) & 0xCu) | ((x << 14) & 0x30000u) | (x & 0xC0000u);
            w[g >> 1] |= v << (8 * (g & 1) + 4 * tb);
          }
        }
      } else {
        // V: tokens 2t + e + 8 kh; elements r, 8 + r of each group go to bits base, base + 4
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const int tk = 2 * t4 + (kk & 1) + 8 * (kk >> 1);
#pragma unroll
          for (int g = 0; g < G8; ++g) {
            const uint32_t y = (nat[tk * PS + g] >> (2 * r)) & 0x00030003u;
            w[g >> 1] |= ((y | (y >> 12)) & 0x33u) << (16 * (kk & 1) + 8 * (g & 1) + 2 * (kk >> 1));
          }
        }
      }
#pragma unroll
      for (int j = 0; j < WPL; ++j) words[j] = w[j];
    } else {
      // ---- pass A: each group's (s, z) as floats, once ----
#pragma unroll
      for (int k2 = 0; k2 < NG / 32; ++k2) {
        const int p = lane + 32 * k2, tok = p / G8, g = p % G8;
        prm[tok * PS + g] = make_float2(meta_scale(msc[s_at(tok, g)]), meta_scale(mzr[z_at(tok, g)]));
      }
      __syncwarp();
      // ---- pass B: f32(code * s + z) in the cache dtype, row-major ----
      // two codes c as floats: the low bits of 2^23 + c, minus 2^23
      auto cf2 = [](uint32_t x, int b0, int b1) {
        return __fadd2_rn(make_float2(__uint_as_float(0x4B000000u | ((x >> b0) & 3u)),
                                      __uint_as_float(0x4B000000u | ((x >> b1) & 3u))),
                          make_float2(-8388608.f, -8388608.f));
      };
      if (wq == 0) {
#pragma unroll
        for (int tb = 0; tb < 2; ++tb) {
          const int t = r + 8 * tb;
          uint32_t* row = reinterpret_cast<uint32_t*>(rows + t * RS);
#pragma unroll
          for (int g = 0; g < G8; ++g) {
            const uint32_t x = words[g >> 1];
            const int base = 8 * (g & 1) + 4 * tb;
            const float2 pm = prm[t * PS + g];
            const float2 s2 = make_float2(pm.x, pm.x), z2 = make_float2(pm.y, pm.y);
            const float2 va = __ffma2_rn(cf2(x, base, 16 + base), s2, z2);
            const float2 vb = __ffma2_rn(cf2(x, base + 2, 16 + base + 2), s2, z2);
            row[8 * g + t4] = pack2<T>(va.x, va.y);
            row[8 * g + 4 + t4] = pack2<T>(vb.x, vb.y);
          }
        }
      } else {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const int tk = 2 * t4 + (kk & 1) + 8 * (kk >> 1);
          const int e = kk & 1, kh = kk >> 1;
#pragma unroll
          for (int g = 0; g < G8; ++g) {
            const uint32_t x = words[g >> 1];
            const int base = 16 * e + 8 * (g & 1) + 2 * kh;
            const float2 pm = prm[tk * PS + g];
            const float2 v = __ffma2_rn(cf2(x, base, base + 4), make_float2(pm.x, pm.x), make_float2(pm.y, pm.y));
            rows[tk * RS + 16 * g + r] = Elem<T>::from_f(v.x);
            rows[tk * RS + 16 * g + 8 + r] = Elem<T>::from_f(v.y);
          }
        }
      }
    }
    // the result leaves by bulk stores once both warps' writes are visible to the async proxy;
    // then the source buffer is free for the next item's copy
    fence_proxy_async_smem();
    __syncthreads();
    if (wq == 0) {
      if (kind == 0) {
        if (lane == 0) bulk_s2g(dst, img, BL::BYTES);
      } else {
        bulk_s2g(reinterpret_cast<uint8_t*>(dst) + lane * D * 2, pg_s + lane * RS * 2, D * 2);
      }
      bulk_commit();
      store_kind = kind;
      if (k + 1 < n_items) issue(k + 1);
    }
  }
  if (!ok && wq == 0 && pend) mbar_wait_bounded(&bars[0], par, st.status, 3001);  // a copy still in flight
  bulk_wait_all();
}

// A window's ledger entry in the row-major form of qe_int2_quantize: one warp per 16-token
// block. found[0] = 1 when the window has an entry, else 0 (and nothing else is written).
template <int D>
__global__ void __launch_bounds__(128) ledger_read_kernel(DevState st, int u, int win, uint8_t* codes_k,
                                                          uint32_t* meta_k, uint8_t* codes_v, uint32_t* meta_v,
                                                          int32_t* found) {
  using BL = Int2Block<D>;
  constexpr int NAT = QE_PAGE * D / 4;
  __shared__ __align__(16) uint8_t sm_all[4][BL::BYTES];
  const int lane = threadIdx.x & 31, wq = threadIdx.x >> 5;
  const int slot = st.win_slot[(size_t)u * st.Wmax + win];
  if (slot < 0 || slot >= st.S) {
    if (threadIdx.x == 0) found[0] = 0;
    return;
  }
  if (threadIdx.x == 0) found[0] = 1;
  uint8_t* img = sm_all[wq];
  for (int bk = wq; bk < st.window / QE_PAGE; bk += 4) {
    const uint4* g = reinterpret_cast<const uint4*>(st.slots + ((size_t)u * st.S + slot) * st.slot_bytes +
                                                    (size_t)bk * BL::BYTES);
    __syncwarp();
    for (int i = lane; i < BL::BYTES / 16; i += 32) reinterpret_cast<uint4*>(img)[i] = g[i];
    __syncwarp();
    const uint32_t* kc = reinterpret_cast<const uint32_t*>(img + BL::KC);
    const uint32_t* vc = reinterpret_cast<const uint32_t*>(img + BL::VC);
    for (int n = lane; n < NAT; n += 32) {
      codes_k[(size_t)bk * NAT + n] = BL::template unpack_byte<false>(kc, n);
      codes_v[(size_t)bk * NAT + n] = BL::template unpack_byte<true>(vc, n);
    }
    const uint16_t* ks = reinterpret_cast<const uint16_t*>(img + BL::KS);
    const uint16_t* kz = reinterpret_cast<const uint16_t*>(img + BL::KZ);
    const uint16_t* vs = reinterpret_cast<const uint16_t*>(img + BL::VS);
    const uint16_t* vz = reinterpret_cast<const uint16_t*>(img + BL::VZ);
    for (int i = lane; i < QE_PAGE * BL::G8; i += 32) {
      const int t = i / BL::G8, gg = i % BL::G8;
      const size_t o = ((size_t)bk * QE_PAGE + t) * BL::G8 + gg;
      const int fp = BL::fpos(t);
      meta_k[o] = (uint32_t)ks[gg * QE_PAGE + BL::ppos(t)] | ((uint32_t)kz[t * BL::G8 + gg] << 16);
      meta_v[o] = (uint32_t)vs[gg * QE_PAGE + fp] | ((uint32_t)vz[gg * QE_PAGE + fp] << 16);
    }
  }
}

// standalone quantiser: one warp per row
template <typename T, int D>
__global__ void int2_quantize_kernel(const T* x, int rows, uint8_t* codes, uint32_t* meta) {
  constexpr int DPL = D / 32;
  using R = Int2Row<DPL>;
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  float xv[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) xv[e] = Elem<T>::to_f(x[(size_t)row * D + lane * DPL + e]);
  uint32_t m;
  const uint32_t bits = R::quantize(xv, &m);
  R::store_codes(codes + (size_t)row * D / 4, bits, lane);
  if (lane % R::LPG == 0) meta[(size_t)row * D / 16 + R::group_of(lane)] = m;
}

template <typename T, int D>
void launch_apply(const DevState& st, const qe_ctx* c, int unit_only, cudaStream_t s) {
  const int units = unit_only >= 0 ? 1 : st.U;
  // a routing event moves at most F + Q windows of a unit into a new tier (host-given
  // transitions at most Wmax): that bounds the items; the grid is one wave of resident blocks
  int wins = unit_only >= 0 ? st.Wmax : c->cfg.full_windows + c->cfg.int2_windows;
  if (wins > st.Wmax) wins = st.Wmax;
  const size_t smem = apply_smem_bytes<D>(units);
  static QeOnce once;
  static int wave_of[QE_MAX_DEVICES];
  int dev = 0;
  if (qe_once_per_device(once, &dev, [](int d) {
        QE_CUDA_TRY(cudaFuncSetAttribute(apply_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         96 * 1024));
        int sms = 0, per_sm = 0;
        QE_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, d));
        QE_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, apply_kernel<T, D>, kApplyThreads,
                                                                  apply_smem_bytes<D>(64)));
        wave_of[d] = sms * (per_sm > 0 ? per_sm : 1);
        return QE_OK;
      }) != QE_OK)
    wave_of[dev] = 148 * 8;
  const long long max_items = (long long)units * wins * st.ppw;
  int blocks = (int)(max_items < wave_of[dev] ? max_items : wave_of[dev]);
  if (blocks < 1) blocks = 1;
  apply_kernel<T, D><<<blocks, kApplyThreads, smem, s>>>(st, c->xlist, c->plist, c->xcount, unit_only);
}

int apply_dispatch(const qe_ctx* c, const DevState& st, int unit_only, cudaStream_t s) {
  const bool bf = c->cfg.dtype == QE_BF16;
  if (c->cfg.D == 128) {
    if (bf) launch_apply<__nv_bfloat16, 128>(st, c, unit_only, s);
    else launch_apply<__half, 128>(st, c, unit_only, s);
  } else {
    if (bf) launch_apply<__nv_bfloat16, 64>(st, c, unit_only, s);
    else launch_apply<__half, 64>(st, c, unit_only, s);
  }
  return cudaGetLastError() == cudaSuccess ? QE_OK : QE_ERR_CUDA;
}

size_t route_smem(const DevState& st) {
  size_t N = 1;
  while (N < (size_t)st.Wmax) N <<= 1;
  return N * 8 + (size_t)st.Wmax * (4 + 4 + 4 + 5) + 64;
}

// Raise the route kernel's dynamic shared-memory limit once per device (outside any graph
// capture).
int route_smem_attr(size_t smem, int Wmax) {
  if (smem > 200 * 1024 || Wmax > 4096) return QE_ERR_UNSUPPORTED_SHAPE;
  static QeOnce once;
  int dev = 0;
  return qe_once_per_device(once, &dev, [](int) {
    QE_CUDA_TRY(cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024));
    return QE_OK;
  });
}

}  // namespace

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
int launch_prefill(qe_ctx* c, const void* K, const void* V, int ctx, const float* norms,
                   cudaStream_t s) {
  DevState st = make_state(c);
  const qe_layout& L = c->lay;
  const size_t U = L.units, W = L.max_windows;
  QE_CUDA_TRY(cudaMemsetAsync(st.win_tier, 0, U * W, s));
  QE_CUDA_TRY(cudaMemsetAsync(st.win_slot, 0xff, U * W * 4, s));
  QE_CUDA_TRY(cudaMemsetAsync(st.win_pages, 0xff, U * W * st.ppw * 4, s));
  QE_CUDA_TRY(cudaMemsetAsync(st.mass, 0, U * W * 4, s));
  QE_CUDA_TRY(cudaMemsetAsync(st.pert, 0, U * W * 4, s));
  QE_CUDA_TRY(cudaMemsetAsync(st.tail_p, 0, U * st.window * st.G * 4, s));
  QE_CUDA_TRY(cudaMemsetAsync(st.route_stats, 0, U * 8 * 4, s));
  QE_CUDA_TRY(cudaMemsetAsync(st.status, 0, 16, s));
  QE_CUDA_TRY(cudaMemsetAsync(c->xcount, 0, U * 16, s));
  const int n_pages = (ctx + QE_PAGE - 1) / QE_PAGE;
  prefill_pages_kernel<<<dim3(n_pages, (unsigned)U), 256, 0, s>>>(st, (const uint4*)K, (const uint4*)V,
                                                                  ctx);
  prefill_meta_kernel<<<(unsigned)U, 256, 0, s>>>(st, (const uint4*)V, ctx, (uint4*)c->tailV);
  QE_CUDA_TRY(cudaGetLastError());
  if (norms) {
    const size_t row = (size_t)ctx * c->G * 4, pitch = (size_t)st.norm_pitch * c->G * 4;
    QE_CUDA_TRY(cudaMemcpy2DAsync(st.norms, pitch, norms, row, row, U, cudaMemcpyDeviceToDevice, s));
    return QE_OK;
  }
  return launch_vwo(V, (int)U, ctx, c->cfg.D, c->cfg.dtype, c->W_O, c->cfg.Hq, c->cfg.Hkv,
                    c->cfg.hidden, st.norms, (long long)st.norm_pitch * c->G, st.status, s);
}

int launch_append(qe_ctx* c, const void* k, const void* v, cudaStream_t s) {
  DevState st = make_state(c);
  append_kernel<<<st.U, 64, 0, s>>>(st, (const uint4*)k, (const uint4*)v, c->n, (uint4*)c->tailV);
  return cudaGetLastError() == cudaSuccess ? QE_OK : QE_ERR_CUDA;
}

int launch_finalize(qe_ctx* c, int tw, cudaStream_t s) {
  DevState st = make_state(c);
  const int rows = c->cfg.B * c->cfg.window;
  const long long gstride = (long long)rows * c->G, pstride = (long long)c->cfg.Hkv * gstride;
  // A completed window is a few row blocks: on the tensor-core path each head's hidden columns
  // are split into parts so that the launch covers the SMs; finalize adds the parts in order.
  int nparts = 1, e;
  if (c->cfg.hidden % 128 == 0) {
    static QeOnce once;
    static int sms_of[QE_MAX_DEVICES];
    int dev = 0;
    if (qe_once_per_device(once, &dev, [](int d) {
          QE_CUDA_TRY(cudaDeviceGetAttribute(&sms_of[d], cudaDevAttrMultiProcessorCount, d));
          return QE_OK;
        }) != QE_OK)
      sms_of[dev] = 148;
    nparts = vwo_tc_parts(c->cfg.Hkv, rows, c->cfg.Hq, c->cfg.Hkv, c->cfg.hidden, kTailNormParts, sms_of[dev]);
    e = launch_vwo_tc(c->tailV, c->cfg.Hkv, rows, c->cfg.D, c->cfg.dtype, c->W_O, c->cfg.Hq, c->cfg.Hkv,
                      c->cfg.hidden, c->tail_norm, gstride, st.status, s, nparts, pstride);
  } else {
    e = launch_vwo(c->tailV, c->cfg.Hkv, rows, c->cfg.D, c->cfg.dtype, c->W_O, c->cfg.Hq, c->cfg.Hkv,
                   c->cfg.hidden, c->tail_norm, gstride, st.status, s);
  }
  if (e) return e;
  finalize_kernel<<<st.U, 128, 0, s>>>(st, c->tail_norm, nparts, pstride, tw);
  return cudaGetLastError() == cudaSuccess ? QE_OK : QE_ERR_CUDA;
}

int launch_route(qe_ctx* c, cudaStream_t s) {
  DevState st = make_state(c);
  RouteArgs a{};
  a.st = st;
  a.xlist = c->xlist;
  a.plist = c->plist;
  a.xcount = c->xcount;
  a.F = c->cfg.full_windows;
  a.Q = c->cfg.int2_windows;
  a.F1 = (int)floor((double)c->cfg.alpha * a.F);
  a.Q1 = (int)floor((double)c->cfg.alpha * a.Q);
  a.mode = 0;
  a.unit = -1;
  const size_t smem = route_smem(st);
  if (int e = route_smem_attr(smem, st.Wmax)) return e;
  route_kernel<<<st.U, kRouteThreads, smem, s>>>(a);
  QE_CUDA_TRY(cudaGetLastError());
  return apply_dispatch(c, st, -1, s);
}

int launch_route_decided(qe_ctx* c, const uint8_t* decided, size_t dec_stride, cudaStream_t s) {
  DevState st = make_state(c);
  RouteArgs a{};
  a.st = st;
  a.xlist = c->xlist;
  a.plist = c->plist;
  a.xcount = c->xcount;
  a.mode = 2;
  a.unit = -1;
  a.decided = decided;
  a.dec_stride = dec_stride;
  const size_t smem = route_smem(st);
  if (int e = route_smem_attr(smem, st.Wmax)) return e;
  route_kernel<<<st.U, kRouteThreads, smem, s>>>(a);
  QE_CUDA_TRY(cudaGetLastError());
  return apply_dispatch(c, st, -1, s);
}

int launch_set_tier(qe_ctx* c, int unit, const int32_t* ids, int n, int tier, cudaStream_t s) {
  DevState st = make_state(c);
  QE_CUDA_TRY(cudaMemcpyAsync(c->host_ids, ids, (size_t)n * 4, cudaMemcpyHostToDevice, s));
  RouteArgs a{};
  a.st = st;
  a.xlist = c->xlist;
  a.plist = c->plist;
  a.xcount = c->xcount;
  a.mode = 1;
  a.unit = unit;
  a.ids = c->host_ids;
  a.n_ids = n;
  a.target = tier;
  const size_t smem = route_smem(st);
  if (int e = route_smem_attr(smem, st.Wmax)) return e;
  route_kernel<<<1, kRouteThreads, smem, s>>>(a);
  QE_CUDA_TRY(cudaGetLastError());
  return apply_dispatch(c, st, unit, s);
}

int launch_ledger_read(qe_ctx* c, int unit, int win, uint8_t* codes_k, uint32_t* meta_k, uint8_t* codes_v,
                       uint32_t* meta_v, int32_t* found, cudaStream_t s) {
  const DevState st = make_state(c);
  if (c->cfg.D == 128)
    ledger_read_kernel<128><<<1, 128, 0, s>>>(st, unit, win, codes_k, meta_k, codes_v, meta_v, found);
  else
    ledger_read_kernel<64><<<1, 128, 0, s>>>(st, unit, win, codes_k, meta_k, codes_v, meta_v, found);
  QE_CUDA_TRY(cudaGetLastError());
  return QE_OK;
}

int launch_int2_quantize(const void* x, int T, int D, int dtype, uint8_t* codes, uint32_t* meta,
                         cudaStream_t s) {
  const int blocks = (T + 7) / 8;
  if (D == 128) {
    if (dtype == QE_BF16)
      int2_quantize_kernel<__nv_bfloat16, 128><<<blocks, 256, 0, s>>>((const __nv_bfloat16*)x, T, codes, meta);
    else
      int2_quantize_kernel<__half, 128><<<blocks, 256, 0, s>>>((const __half*)x, T, codes, meta);
  } else if (D == 64) {
    if (dtype == QE_BF16)
      int2_quantize_kernel<__nv_bfloat16, 64><<<blocks, 256, 0, s>>>((const __nv_bfloat16*)x, T, codes, meta);
    else
      int2_quantize_kernel<__half, 64><<<blocks, 256, 0, s>>>((const __half*)x, T, codes, meta);
  } else {
    return QE_ERR_UNSUPPORTED_SHAPE;
  }
  return cudaGetLastError() == cudaSuccess ? QE_OK : QE_ERR_CUDA;
}
