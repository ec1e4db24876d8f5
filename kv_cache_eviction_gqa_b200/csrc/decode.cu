// Split-K GQA decode attention over the full-precision and INT2 tiers, fused with the
// cumulative window scores.
//
// "Resumo Técnico: QEvict" - Mecanismos Principais: window-level routing driven by
// attention accumulated over time (Pontuação Cumulativa); recoverable INT2 tier that
// attention still reads (Metodologia 2); GQA decode path (Implementação).
// "Resumo Técnico: CriticalKV" - Etapa 2: the perturbation score A_i * ||V_i W_O||_1.
//
// Per unit u = (b, g) the live windows form a list [full windows | INT2 windows | tail].
// The list is cut into `splits` contiguous, cost-balanced ranges, one CTA each. Inside a
// CTA every warp takes whole windows round-robin and streams them through its own ring of
// shared-memory stages with 1-D bulk copies (cp.async.bulk, completion on an mbarrier):
// one 16-token page (K rows then V rows) per stage for full windows, one ledger entry per
// stage for INT2 windows, each with the window's norms. Lanes split the head dimension
// (D/32 elements each); a token's G query-head dot products are reduced across the warp
// in batches of 8 tokens. Softmax runs online in the log2 domain.
//
// Scoring without a second pass: every warp records, per window and head, the partial
// (m, sum_i 2^(s_i-m), sum_i 2^(s_i-m) n_i) relative to its running max m. The last CTA of
// the unit to finish (atomic ticket, no spinning) combines the splits into the output and
// the per-head log-sum-exp, then adds each window's exact attention mass and perturbation
// to the cumulative scores. The tail window's norms are not known yet, so its per-token
// attention is accumulated instead (tail_p) and folded in when it completes.
#include <math.h>

#include "int2.cuh"
#include "qe_internal.cuh"

namespace {

constexpr int kNW = 4;   // warps per CTA
constexpr int kNST = 3;  // stages per warp

struct DecodeArgs {
  DevState st;
  const void* q;     // [B][Hq][D]
  float* out;        // [B][Hq][D]
  float* split_part; // [U][max_splits][G][D + 2]
  float* win_part;   // [U][Wmax][G][4]
  float* tail_s;     // [U][window][G]
  uint32_t* tickets; // [U]
  int splits, max_splits;
  int tail_win, tail_len;
  float scale_log2;  // log2(e) / sqrt(D)
};

// Sum a value per token over the warp, for 8 tokens at once. Lane l ends with the
// total of token (l >> 2) & 7 (each token replicated in 4 lanes).
__device__ __forceinline__ float reduce8(const float (&v)[8], int lane) {
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
  float r4[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float send = b4 ? v[i] : v[i + 4];
    const float keep = b4 ? v[i + 4] : v[i];
    r4[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
  float r2[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float send = b3 ? r4[i] : r4[i + 2];
    const float keep = b3 ? r4[i + 2] : r4[i];
    r2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  const float send = b2 ? r2[0] : r2[1];
  const float keep = b2 ? r2[1] : r2[0];
  float r = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  r += __shfl_xor_sync(0xffffffffu, r, 2);
  r += __shfl_xor_sync(0xffffffffu, r, 1);
  return r;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// First list index of split s: windows are weighted 4 (full, tail) and 1 (INT2).
__device__ __forceinline__ int split_begin(int s, int S, int nf, int nq, int has_tail) {
  const long long W = 4ll * nf + nq + 4ll * has_tail;
  const long long t = (s * W + S - 1) / S;
  if (t <= 4ll * nf) return (int)((t + 3) / 4);
  if (t <= 4ll * nf + nq) return nf + (int)(t - 4ll * nf);
  return nf + nq + 1;
}

template <typename T, int D>
__device__ __forceinline__ void load_row(const T* row, int lane, float (&x)[D / 32]) {
  constexpr int DPL = D / 32;
  if constexpr (DPL == 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(row + lane * 4);
    x[0] = Elem<T>::lo(w.x);
    x[1] = Elem<T>::hi(w.x);
    x[2] = Elem<T>::lo(w.y);
    x[3] = Elem<T>::hi(w.y);
  } else {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(row + lane * 2);
    x[0] = Elem<T>::lo(w);
    x[1] = Elem<T>::hi(w);
  }
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kNW * 32) decode_kernel(DecodeArgs a) {
  constexpr int DPL = D / 32;
  using R = Int2Row<DPL>;
  constexpr int PAGE_BYTES = 2 * QE_PAGE * D * 2;   // K rows then V rows
  constexpr int NORM_BYTES = 64 * G * 4;            // up to a 64-token window
  constexpr int STAGE = PAGE_BYTES + NORM_BYTES;
  extern __shared__ __align__(128) uint8_t smem[];
  const DevState& st = a.st;
  const int u = blockIdx.x / a.splits, split = blockIdx.x % a.splits;
  const int b = u / st.Hkv, kvh = u % st.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int w = st.window, ppw = st.ppw;
  const size_t ub = (size_t)u * st.Wmax;

  const int nf = st.stacks[u * 4 + 2], nq = st.stacks[u * 4 + 3];
  const int has_tail = a.tail_len > 0;
  const int nwin = nf + nq + has_tail;
  const int j0 = split_begin(split, a.splits, nf, nq, has_tail);
  const int j1 = split + 1 == a.splits ? nwin : split_begin(split + 1, a.splits, nf, nq, has_tail);

  uint8_t* ring = smem + warp * kNST * STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kNW * kNST * STAGE) + warp * kNST;
  if (lane == 0) {
    for (int s = 0; s < kNST; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();

  // query heads of this group, pre-scaled into the log2 domain
  float q[G][DPL], qsum[G];
  {
    const T* qb = reinterpret_cast<const T*>(a.q) + ((size_t)b * st.Hq + (size_t)kvh * G) * D;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      load_row<T, D>(qb + (size_t)h * D, lane, q[h]);
      qsum[h] = 0.f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) {
        q[h][e] *= a.scale_log2;
        qsum[h] += q[h][e];
      }
    }
  }
  float acc[G][DPL], zacc[G], m[G], lsum[G], lw[G], nw[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    zacc[h] = 0.f;
    m[h] = -INFINITY;
    lsum[h] = 0.f;
    lw[h] = 0.f;
    nw[h] = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[h][e] = 0.f;
  }

  // ---- task iteration: (window list index j, page index pg) ----
  auto kind_of = [&](int j) { return j < nf ? 0 : (j < nf + nq ? 1 : 2); };  // full, int2, tail
  auto n_tasks = [&](int j) {
    const int k = kind_of(j);
    return k == 0 ? ppw : (k == 1 ? 1 : (a.tail_len + QE_PAGE - 1) / QE_PAGE);
  };
  auto advance = [&](int& j, int& pg) {
    if (++pg >= n_tasks(j)) {
      pg = 0;
      j += kNW;
    }
  };
  // issue the bulk copies of task (j, pg) into stage s (lane 0 only)
  auto issue = [&](int j, int pg, int s) {
    uint8_t* dst = ring + s * STAGE;
    uint64_t* bar = &bars[s];
    const int k = kind_of(j);
    if (k == 1) {
      const int win = st.int2_list[ub + j - nf];
      const int slot = (win >= 0 && win < st.Wmax) ? st.win_slot[ub + win] : -1;
      if (slot < 0 || slot >= st.S) {
        qe_record_error(st.status, QE_ERR_DEVICE_FAULT, u);
        mbar_arrive_expect_tx(bar, 0);
        return;
      }
      const uint32_t nb = (uint32_t)(w * G * 4);
      mbar_arrive_expect_tx(bar, (uint32_t)st.slot_bytes + nb);
      bulk_g2s(dst, st.slots + ((size_t)u * st.S + slot) * st.slot_bytes, (uint32_t)st.slot_bytes, bar);
      bulk_g2s(dst + PAGE_BYTES, st.norms + ((size_t)u * st.norm_pitch + (size_t)win * w) * G, nb, bar);
    } else {
      const int win = k == 0 ? st.full_list[ub + j] : a.tail_win;
      const int page = (win >= 0 && win < st.Wmax) ? st.win_pages[(ub + win) * ppw + pg] : -1;
      if (page < 0 || page >= st.P) {
        qe_record_error(st.status, QE_ERR_DEVICE_FAULT, u);
        mbar_arrive_expect_tx(bar, 0);
        return;
      }
      const uint8_t* src = st.pages + ((size_t)u * st.P + page) * st.page_bytes;
      if (k == 0) {
        const uint32_t nb = QE_PAGE * G * 4;
        mbar_arrive_expect_tx(bar, PAGE_BYTES + nb);
        bulk_g2s(dst, src, PAGE_BYTES, bar);
        bulk_g2s(dst + PAGE_BYTES,
                 st.norms + ((size_t)u * st.norm_pitch + (size_t)win * w + pg * QE_PAGE) * G, nb, bar);
      } else {
        mbar_arrive_expect_tx(bar, PAGE_BYTES);
        bulk_g2s(dst, src, PAGE_BYTES, bar);
      }
    }
  };

  // online-softmax update with one batch of 8 scores (lane holds token (lane>>2)&7)
  auto online = [&](float (&s)[G], float (&p)[G]) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float mb = s[h];
      mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 4));
      mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 8));
      mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 16));
      const float mn = fmaxf(m[h], mb);
      if (mn == -INFINITY) {
        p[h] = 0.f;
        continue;
      }
      if (mn > m[h]) {
        const float sc = exp2f(m[h] - mn);
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[h][e] *= sc;
        zacc[h] *= sc;
        lsum[h] *= sc;
        lw[h] *= sc;
        nw[h] *= sc;
        m[h] = mn;
      }
      p[h] = exp2f(s[h] - mn);
    }
  };

  int j = j0 + warp, pg = 0;
  const bool any = j < j1;
  // prologue: fill kNST - 1 stages
  int ij = j, ipg = pg, issued = 0;
  if (lane == 0) {
    for (int s = 0; s < kNST - 1 && ij < j1; ++s) {
      issue(ij, ipg, s);
      advance(ij, ipg);
      ++issued;
    }
  }
  ij = __shfl_sync(0xffffffffu, ij, 0);
  ipg = __shfl_sync(0xffffffffu, ipg, 0);
  issued = __shfl_sync(0xffffffffu, issued, 0);
  int k = 0;  // tasks consumed
  bool ok = true;
  while (any && j < j1) {
    // keep kNST - 1 tasks in flight
    if (ij < j1) {
      if (lane == 0) {
        fence_proxy_async_smem();
        issue(ij, ipg, issued % kNST);
      }
      advance(ij, ipg);
      ++issued;
    }
    const int s = k % kNST;
    ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[s], (k / kNST) & 1, st.status, 1000 + u));
    if (!ok) break;
    const uint8_t* stage = ring + s * STAGE;
    const int kind = kind_of(j);
    const float* nrm = reinterpret_cast<const float*>(stage + PAGE_BYTES);
    if (kind != 1) {
      // ---- full-precision page (K rows then V rows) ----
      const T* Ks = reinterpret_cast<const T*>(stage);
      const T* Vs = Ks + QE_PAGE * D;
      const int valid = kind == 2 ? min(QE_PAGE, a.tail_len - pg * QE_PAGE) : QE_PAGE;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        if (half * 8 >= valid) break;
        float part[G][8];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          float kx[DPL];
          load_row<T, D>(Ks + (size_t)(half * 8 + t) * D, lane, kx);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            float d0 = 0.f;
#pragma unroll
            for (int e = 0; e < DPL; ++e) d0 = fmaf(q[h][e], kx[e], d0);
            part[h][t] = d0;
          }
        }
        const int tl = half * 8 + ((lane >> 2) & 7);
        const bool vt = tl < valid;
        float sc[G], p[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          sc[h] = reduce8(part[h], lane);
          if (!vt) sc[h] = -INFINITY;
        }
        online(sc, p);
        if ((lane & 3) == 0 && vt) {
#pragma unroll
          for (int h = 0; h < G; ++h) {
            lsum[h] += p[h];
            if (kind == 0) {
              lw[h] += p[h];
              nw[h] = fmaf(p[h], nrm[tl * G + h], nw[h]);  // this page's 16 tokens
            } else {
              a.tail_s[((size_t)u * w + pg * QE_PAGE + tl) * G + h] = sc[h];
            }
          }
        }
        const int nt = min(8, valid - half * 8);
        for (int t = 0; t < nt; ++t) {
          float vx[DPL];
          load_row<T, D>(Vs + (size_t)(half * 8 + t) * D, lane, vx);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float pt = __shfl_sync(0xffffffffu, p[h], t * 4);
#pragma unroll
            for (int e = 0; e < DPL; ++e) acc[h][e] = fmaf(pt, vx[e], acc[h][e]);
          }
        }
      }
    } else {
      // ---- INT2 ledger entry of a whole window: codes K | codes V | meta K | meta V ----
      const uint8_t* kc = stage;
      const uint8_t* vc = stage + w * D / 4;
      const uint32_t* km = reinterpret_cast<const uint32_t*>(stage + w * D / 2);
      const uint32_t* vm = km + w * D / 16;
      const int grp = R::group_of(lane);
      for (int t0 = 0; t0 < w; t0 += 8) {
        float part[G][8];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const uint32_t bits = R::load_codes(kc + (t0 + t) * (D / 4), lane);
          const uint32_t mt = km[(t0 + t) * (D / 16) + grp];
          const float sk = meta_scale(mt), zk = meta_zero(mt);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            float dc = 0.f;
#pragma unroll
            for (int e = 0; e < DPL; ++e) dc = fmaf(q[h][e], (float)((bits >> (2 * e)) & 3u), dc);
            part[h][t] = fmaf(sk, dc, zk * qsum[h]);
          }
        }
        const int tl = t0 + ((lane >> 2) & 7);
        float sc[G], p[G];
#pragma unroll
        for (int h = 0; h < G; ++h) sc[h] = reduce8(part[h], lane);
        online(sc, p);
        if ((lane & 3) == 0) {
#pragma unroll
          for (int h = 0; h < G; ++h) {
            lsum[h] += p[h];
            lw[h] += p[h];
            nw[h] = fmaf(p[h], nrm[tl * G + h], nw[h]);
          }
        }
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const uint32_t bits = R::load_codes(vc + (t0 + t) * (D / 4), lane);
          const uint32_t mt = vm[(t0 + t) * (D / 16) + grp];
          const float sv = meta_scale(mt), zv = meta_zero(mt);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float pt = __shfl_sync(0xffffffffu, p[h], t * 4);
            const float ps = pt * sv;
#pragma unroll
            for (int e = 0; e < DPL; ++e) acc[h][e] = fmaf(ps, (float)((bits >> (2 * e)) & 3u), acc[h][e]);
            zacc[h] = fmaf(pt, zv, zacc[h]);
          }
        }
      }
    }
    __syncwarp();
    // end of a window: record its partial scores
    const bool last_task = pg + 1 >= n_tasks(j);
    if (last_task && kind != 2) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float l2 = warp_sum(lw[h]), n2 = warp_sum(nw[h]);
        if (lane == 0) {
          float* wp = a.win_part + ((ub + j) * G + h) * 4;
          wp[0] = m[h];
          wp[1] = l2;
          wp[2] = n2;
        }
        lw[h] = 0.f;
        nw[h] = 0.f;
      }
    }
    advance(j, pg);
    ++k;
  }
  // drain copies still in flight if a wait gave up
  if (!ok) {
    for (; k < issued; ++k) mbar_wait_bounded(&bars[k % kNST], (k / kNST) & 1, st.status, 2000 + u);
  }

  // ---- merge the warps of this CTA into one split partial ----
  __syncthreads();
  float* mw = reinterpret_cast<float*>(smem);             // [kNW][G]
  float* lwv = mw + kNW * G;                              // [kNW][G]
  float* aw = lwv + kNW * G;                              // [kNW][G][D]
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float l2 = warp_sum(lsum[h]);
    if (lane == 0) {
      mw[warp * G + h] = m[h];
      lwv[warp * G + h] = l2;
    }
#pragma unroll
    for (int e = 0; e < DPL; ++e) aw[((size_t)warp * G + h) * D + lane * DPL + e] = acc[h][e] + zacc[h];
  }
  __syncthreads();
  float* sp = a.split_part + ((size_t)u * a.max_splits + split) * G * (D + 2);
  for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
    const int h = i / D, d = i % D;
    float M = -INFINITY;
    for (int x = 0; x < kNW; ++x) M = fmaxf(M, mw[x * G + h]);
    float L = 0.f, A = 0.f;
    if (M != -INFINITY) {
      for (int x = 0; x < kNW; ++x) {
        const float f = exp2f(mw[x * G + h] - M);
        L += lwv[x * G + h] * f;
        A += aw[((size_t)x * G + h) * D + d] * f;
      }
    }
    sp[h * (D + 2) + 2 + d] = A;
    if (d == 0) {
      sp[h * (D + 2) + 0] = M;
      sp[h * (D + 2) + 1] = L;
    }
  }

  // ---- the last CTA of the unit combines ----
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(&a.tickets[u], 1u) == (unsigned)(a.splits - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  float* lse = reinterpret_cast<float*>(smem);  // [G]
  float* red = lse + QE_MAX_G;                  // [32]
  const float* sp0 = a.split_part + (size_t)u * a.max_splits * G * (D + 2);
  if (threadIdx.x < G) {
    const int h = threadIdx.x;
    float M = -INFINITY;
    for (int x = 0; x < a.splits; ++x) M = fmaxf(M, __ldcg(sp0 + (x * G + h) * (D + 2)));
    float L = 0.f;
    for (int x = 0; x < a.splits; ++x) {
      const float mx = __ldcg(sp0 + (x * G + h) * (D + 2));
      if (mx != -INFINITY) L += __ldcg(sp0 + (x * G + h) * (D + 2) + 1) * exp2f(mx - M);
    }
    lse[h] = M + log2f(L);
    red[h] = M;
    red[8 + h] = L;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
    const int h = i / D, d = i % D;
    const float M = red[h], L = red[8 + h];
    float A = 0.f;
    for (int x = 0; x < a.splits; ++x) {
      const float mx = __ldcg(sp0 + (x * G + h) * (D + 2));
      if (mx != -INFINITY) A += __ldcg(sp0 + (x * G + h) * (D + 2) + 2 + d) * exp2f(mx - M);
    }
    a.out[((size_t)b * st.Hq + (size_t)kvh * G + h) * D + d] = A / L;
  }
  // exact per-window mass and perturbation of this step
  for (int jj = threadIdx.x; jj < nf + nq; jj += blockDim.x) {
    const int win = jj < nf ? st.full_list[ub + jj] : st.int2_list[ub + jj - nf];
    if (win < 0 || win >= st.Wmax) continue;
    float dm = 0.f, dp = 0.f;
    const float* wp = a.win_part + (ub + jj) * G * 4;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float f = exp2f(__ldcg(wp + h * 4 + 0) - lse[h]);
      dm = fmaf(__ldcg(wp + h * 4 + 1), f, dm);
      dp = fmaf(__ldcg(wp + h * 4 + 2), f, dp);
    }
    st.mass[ub + win] += dm;
    st.pert[ub + win] += dp;
  }
  // tail tokens: cumulative per-token attention, window mass
  float tm = 0.f;
  for (int i = threadIdx.x; i < a.tail_len * G; i += blockDim.x) {
    const int h = i % G;
    const float pv = exp2f(__ldcg(a.tail_s + (size_t)u * w * G + i) - lse[h]);
    st.tail_p[(size_t)u * w * G + i] += pv;
    tm += pv;
  }
  tm = warp_sum(tm);
  __syncthreads();
  if (lane == 0) red[16 + warp] = tm;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int x = 0; x < kNW; ++x) s += red[16 + x];
    if (has_tail) st.mass[ub + a.tail_win] += s;
    a.tickets[u] = 0;
  }
}

template <typename T, int D, int G>
int launch_decode_t(qe_ctx* c, const void* q, float* out, cudaStream_t s) {
  constexpr int PAGE_BYTES = 2 * QE_PAGE * D * 2;
  constexpr int STAGE = PAGE_BYTES + 64 * G * 4;
  const size_t smem = (size_t)kNW * kNST * STAGE + kNW * kNST * 8;
  static_assert((size_t)kNW * G * (D + 2) * 4 <= (size_t)kNW * kNST * STAGE, "merge area");
  auto kern = decode_kernel<T, D, G>;
  QE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  int per_sm = 1, sms = 148, dev = 0;
  QE_CUDA_TRY(cudaGetDevice(&dev));
  QE_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  QE_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kNW * 32, smem));
  if (per_sm < 1) per_sm = 1;
  DecodeArgs a{};
  a.st = make_state(c);
  a.q = q;
  a.out = out;
  a.split_part = c->split_part;
  a.win_part = c->win_part;
  a.tail_s = c->tail_s;
  a.tickets = c->tickets;
  a.max_splits = c->cfg.max_splits;
  a.tail_win = c->complete;
  a.tail_len = c->n - c->complete * c->cfg.window;
  a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
  const int U = c->lay.units;
  const int nwin = c->n_full_max + c->n_int2_max + 1;
  int S = (2 * per_sm * sms + U - 1) / U;
  if (S > nwin) S = nwin;
  if (S > c->cfg.max_splits) S = c->cfg.max_splits;
  if (S < 1) S = 1;
  a.splits = S;
  kern<<<U * S, kNW * 32, smem, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? QE_OK : QE_ERR_CUDA;
}

template <typename T, int D>
int launch_decode_g(qe_ctx* c, const void* q, float* out, cudaStream_t s) {
  switch (c->G) {
    case 1: return launch_decode_t<T, D, 1>(c, q, out, s);
    case 2: return launch_decode_t<T, D, 2>(c, q, out, s);
    case 4: return launch_decode_t<T, D, 4>(c, q, out, s);
    case 5: return launch_decode_t<T, D, 5>(c, q, out, s);
    case 8: return launch_decode_t<T, D, 8>(c, q, out, s);
    default: return QE_ERR_UNSUPPORTED_SHAPE;
  }
}

}  // namespace

int launch_decode(qe_ctx* c, const void* q, float* out, cudaStream_t s) {
  const bool bf = c->cfg.dtype == QE_BF16;
  if (c->cfg.D == 128)
    return bf ? launch_decode_g<__nv_bfloat16, 128>(c, q, out, s) : launch_decode_g<__half, 128>(c, q, out, s);
  return bf ? launch_decode_g<__nv_bfloat16, 64>(c, q, out, s) : launch_decode_g<__half, 64>(c, q, out, s);
}
