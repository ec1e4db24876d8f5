// Split-K GQA decode attention over the full-precision and INT2 tiers, fused with the
// cumulative window scores and (optionally) the append of the step's token.
//
// "Resumo Técnico: QEvict" - Mecanismos Principais: window-level routing driven by
// attention accumulated over time (Pontuação Cumulativa); the recoverable INT2 tier stays
// readable by attention (Metodologia 2); GQA decode path (Implementação).
// "Resumo Técnico: CriticalKV" - Etapa 2: the perturbation score A_i * ||V_i W_O||_1.
//
// Work split. Per unit u = (b, g) the live windows are [full windows | INT2 windows | tail].
// The unit's S CTAs form one thread-block cluster; CTA s takes the s-th S-th of the full
// windows and of the INT2 windows (the tail counts as one more INT2 window of the last CTA),
// so every SM streams the same mix of bandwidth-heavy full pages and arithmetic-heavy INT2
// entries. Inside a CTA each warp takes whole windows round-robin and streams them through
// its own ring of shared-memory stages (completion on an mbarrier per stage): a full page
// arrives as 128-byte-swizzled TMA boxes from a tensor map over the page pool, an INT2
// ledger entry or a tail page as one 1-D bulk copy, each with its tokens' projected-value norms.
//
// Full-precision windows run on the warp-level tensor cores (m16n8k16, f32 accumulate):
// S = Q K^T with the G query rows padded to 16, then O^T = V^T P^T with P split into two
// 16-bit parts so the product keeps float32 accuracy. A decode step has G <= 8 query rows per
// KV head; a tcgen05 tile (M >= 64) would be mostly padding and its TMEM round trip buys
// nothing on a path that HBM bounds, so these pages stay on mma.sync.
//
// INT2 and tail windows run on the CUDA cores. A token is handled by LPT = D / DPL lanes; lane
// `sub` owns the DPL contiguous head-dim elements [DPL*sub, DPL*sub + DPL), i.e. one INT2
// group (DPL = 16) or half of one (DPL = 8), so it needs one scale/zero per token. With
// DPL = 16 the two 8-element chunks of a lane are loaded in a lane-dependent order (register
// chunk c holds memory chunk c ^ sw) so that every 16-byte shared-memory load instruction of
// the warp touches each bank once. A warp works on TPS = 32 / LPT tokens at a time; q and the
// accumulators of the G query heads stay in registers as float pairs and all multiply-adds
// are packed (f32x2). A token's G dot products are summed over its lanes with a butterfly, so
// every lane of the group holds the scores and no weight broadcast is needed. Each lane group
// keeps its own online-softmax state (log2 domain); the accumulators are rescaled only when
// the running maximum grows by more than 2^8.
//
// INT2 decoding without float conversions: a pair of 2-bit codes (even element E, odd E+1)
// is shifted once into the mantissas of 4.0 and 1.0, giving x = 4 + c_E/4 and 1 + c_(E+1)/4
// exactly; the affine map k = c*s + z is folded into the per-token scale (4s) and a per-pair
// offset, so a score is 4s (q . x) + z sum(q) - 4s (4 sum(q_even) + sum(q_odd)).
//
// Scoring without a second pass: at the end of each window every lane group records its
// (max, sum_i 2^(s_i-max), sum_i 2^(s_i-max) n_i) per head in its own slot. After the pass the
// cluster merges the CTA partials through distributed shared memory into the unit's log-sum-
// exp; each CTA writes its share of the output and adds the exact attention mass and
// perturbation of the windows it streamed to the cumulative scores. The tail window's norms
// are not known yet; its per-token attention is accumulated instead (tail_p) and folded in
// when the window completes.
#include <math.h>

#include "append.cuh"
#include "int2.cuh"
#include "qe_internal.cuh"
#include "tc_common.cuh"
#include "warp_mma.cuh"

namespace {

#ifndef QE_DECODE_NW
#define QE_DECODE_NW 2
#endif
#ifndef QE_DECODE_NST
#define QE_DECODE_NST 3
#endif
#ifndef QE_DECODE_MINB
#define QE_DECODE_MINB 4
#endif
#ifndef QE_DECODE_FULL_LAST
#define QE_DECODE_FULL_LAST 0  // 1: odd warps stream their full-precision windows last
#endif
#ifndef QE_DECODE_SB
#define QE_DECODE_SB 4
#endif
constexpr int kNW = QE_DECODE_NW;    // warps per CTA
#define QE_MAX_SPLITS_CLUSTER 16          // CTAs per unit (one cluster, non-portable size)
constexpr int kNST = QE_DECODE_NST;  // stages per warp
constexpr float kRescale = 8.f;  // rescale the accumulators when the max grows by > 2^8

// Per-window score partials: one slot per lane group of {max, sum p, sum p n} x G heads,
// weights 2^(s - max) relative to the slot's max; an unused slot holds max -1e30 and zeros.
struct DecodeArgs {
  DevState st;
  const void* q;     // [B][Hq][D]
  float* out;        // [B][Hq][D]
  float* win_part;   // [U][Wmax][win_part_floats(D, G)]
  float* tail_s;     // [U][window][G]
  int splits;        // CTAs per unit = cluster size
  int tail_win, tail_len;
  float scale_log2;  // log2(e) / sqrt(D)
  // optional fused append of the step's token at position append_pos (k_new != nullptr): the
  // CTA that streams the tail window writes it before its first copy
  const uint4* k_new;
  const uint4* v_new;
  uint4* tailV;
  int append_pos;
};

template <int D, int G>
struct Map {
  static constexpr int DPL = decode_dpl(G);    // head-dim elements per lane
  static constexpr int LPT = D / DPL;          // lanes per token
  static constexpr int TPS = 32 / LPT;         // tokens per warp step
  static constexpr int SB = (16 / TPS) < QE_DECODE_SB ? (16 / TPS) : QE_DECODE_SB;  // tokens per group per batch
  static constexpr int SBT = SB * TPS;         // tokens per batch (divides 16)
  static constexpr int NP = DPL / 2;           // float pairs per lane
};

// 2^x with the hardware approximation (relative error about 2^-22; results below 2^-126
// flush to zero, which no sum here can notice).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// thread-block cluster helpers: barrier over the cluster's CTAs, and a load from the shared
// memory of CTA `rank` of the cluster at the address of a local shared variable
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_cluster(const float* local, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(local)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Chunk order of a lane (DPL = 16): register chunk c holds memory chunk c ^ sw. It may
// depend on `sub` only: lanes with the same `sub` in different token groups must hold the
// same elements in the same registers, since the groups are summed register by register.
// At D = 64 a row is one bank cycle and no lane-only order helps; those loads stay 2-way.
template <int D, int DPL>
__device__ __forceinline__ int chunk_swap(int sub, int grp) {
  (void)grp;
  if constexpr (DPL == 16 && D == 128) return (sub >> 2) & 1;
  else return 0;
}

template <typename T>
__device__ __forceinline__ void cvt8(const uint4 w, float2* x) {
  x[0] = make_float2(Elem<T>::lo(w.x), Elem<T>::hi(w.x));
  x[1] = make_float2(Elem<T>::lo(w.y), Elem<T>::hi(w.y));
  x[2] = make_float2(Elem<T>::lo(w.z), Elem<T>::hi(w.z));
  x[3] = make_float2(Elem<T>::lo(w.w), Elem<T>::hi(w.w));
}

// the lane's DPL elements of a row as float pairs
template <typename T, int DPL>
__device__ __forceinline__ void load_row(const T* row, int sub, int sw, float2 (&x)[DPL / 2]) {
  const uint4* p = reinterpret_cast<const uint4*>(row + DPL * sub);
  if constexpr (DPL == 16) {
    cvt8<T>(p[sw], x);
    cvt8<T>(p[sw ^ 1], x + 4);
  } else {
    cvt8<T>(p[0], x);
  }
}

// Codes E (even) and E+1 from one shift: the pair {4 + c_E/4, 1 + c_(E+1)/4}. Code E lands in
// mantissa bits 19-20 of 4.0 (4 * (1 + c/16)) and code E+1 in bits 21-22 of 1.0, so both
// values are exact and the code's contribution is c/4 in either case; only the constant part
// differs (4 for even elements, 1 for odd ones).
template <int E>
__device__ __forceinline__ float2 code_pair(uint32_t bits) {
  constexpr int sh = 19 - 2 * E;
  const uint32_t v = sh >= 0 ? (bits << (sh >= 0 ? sh : 0)) : (bits >> (sh < 0 ? -sh : 0));
  return make_float2(__uint_as_float((v & 0x00180000u) | 0x40800000u),
                     __uint_as_float((v & 0x00600000u) | 0x3f800000u));
}

template <int NP>
__device__ __forceinline__ void decode_codes(uint32_t bits, float2 (&x)[NP]) {
  x[0] = code_pair<0>(bits);
  x[1] = code_pair<2>(bits);
  x[2] = code_pair<4>(bits);
  x[3] = code_pair<6>(bits);
  if constexpr (NP == 8) {
    x[4] = code_pair<8>(bits);
    x[5] = code_pair<10>(bits);
    x[6] = code_pair<12>(bits);
    x[7] = code_pair<14>(bits);
  }
}

// the lane's codes of one row, with register chunk c = memory chunk c ^ sw in bits 16c..
template <int DPL>
__device__ __forceinline__ uint32_t load_codes(const uint8_t* row, int sub, int sw) {
  if constexpr (DPL == 16) {
    const uint32_t b = reinterpret_cast<const uint32_t*>(row)[sub];
    return sw ? __funnelshift_l(b, b, 16) : b;
  } else {
    return reinterpret_cast<const uint16_t*>(row)[sub];
  }
}

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// Shared-memory stage of one task (1024-byte aligned). A full-precision page arrives as TMA
// boxes of 16 rows x 64 elements with the 128-byte swizzle (box (part, x) at
// (part * D/64 + x) * 2048, part 0 = K rows, 1 = V rows), so the 8 rows of every ldmatrix
// tile sit in distinct banks; tail pages and INT2 ledger entries are 1-D bulk copies in their
// contiguous layout. Up to 64 tokens' norms follow at PAGE_BYTES.
template <int D, int G>
struct StageLayout {
  static constexpr int PAGE_BYTES = 2 * QE_PAGE * D * 2;            // K rows then V rows
  static constexpr int RAW = PAGE_BYTES + 64 * G * 4;
  static constexpr int BYTES = (RAW + 1023) / 1024 * 1024;
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(kNW * 32, QE_DECODE_MINB)
    decode_kernel(const __grid_constant__ CUtensorMap tmP, DecodeArgs a) {
  using M = Map<D, G>;
  constexpr int DPL = M::DPL, LPT = M::LPT, TPS = M::TPS, SB = M::SB, SBT = M::SBT, NP = M::NP;
  using SL = StageLayout<D, G>;
  constexpr int PAGE_BYTES = SL::PAGE_BYTES;
  constexpr int STAGE = SL::BYTES;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const DevState& st = a.st;
  const int u = blockIdx.x / a.splits, split = blockIdx.x % a.splits;
  const int b = u / st.Hkv, kvh = u % st.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane / LPT, sub = lane % LPT;
  const int sw = chunk_swap<D, DPL>(sub, grp);
  const int w = st.window, ppw = st.ppw;
  const size_t ub = (size_t)u * st.Wmax;
  const int gi = DPL * sub / 16;  // this lane's INT2 group within a row

  // this split's share of each tier
  const int nf = st.stacks[u * 4 + 2], nq = st.stacks[u * 4 + 3];
  const int f0 = (int)((long long)nf * split / a.splits), f1 = (int)((long long)nf * (split + 1) / a.splits);
  // the last split also streams the tail window (and appends the new token): it counts as one
  // INT2 window of that split's share
  const int nqv = a.tail_len > 0 ? nq + 1 : nq;
  const int q0 = (int)((long long)nqv * split / a.splits);
  const int q1 = min(nq, (int)((long long)nqv * (split + 1) / a.splits));
  const int has_tail = (a.tail_len > 0 && split == a.splits - 1) ? 1 : 0;
  const int nF = f1 - f0, nQ = q1 - q0, nJ = nF + nQ + has_tail;
  // fused append: the warp that streams the tail window writes the new token first (its tail
  // task comes last, after this warp's own fence); the other warp starts at once
  if (a.k_new != nullptr && has_tail && warp == (nJ - 1) % kNW)
    append_token_warp(st, u, a.append_pos, a.k_new, a.v_new, a.tailV);

  uint8_t* ring = smem + warp * kNST * STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kNW * kNST * STAGE) + warp * kNST;
  if (lane == 0) {
    for (int s = 0; s < kNST; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();

  // SIMT state for the INT2 and tail windows (set up after the full-precision phase): the G
  // query heads of this group, this lane's DPL elements, in the log2 domain; per lane-group
  // online-softmax state; lw/nw: sums of the current window
  float2 q[G][NP];
  float qsum[G];   // sum of the lane's q elements
  float qsum2[G];  // 4 * (sum over even elements) + (sum over odd elements): the constant part of q . x
  float2 acc[G][NP];
  float2 zacc[G];  // INT2 value offsets (even, odd element) weighted by p * ...
  float m[G], lsum[G], lw[G], nw[G];

  // virtual index j of this split -> (kind, list index)
  auto kind_of = [&](int j) { return j < nF ? 0 : (j < nF + nQ ? 1 : 2); };  // full, int2, tail
  auto list_idx = [&](int j) { return j < nF ? f0 + j : nf + q0 + (j - nF); };
  auto n_tasks = [&](int j) {
    const int k = kind_of(j);
    return k == 0 ? ppw : (k == 1 ? 1 : (a.tail_len + QE_PAGE - 1) / QE_PAGE);
  };
  // This warp's windows are j = warp + kNW * r, r < n_own; the first n_own_full are
  // full-precision. With QE_DECODE_FULL_LAST, odd warps stream their full-precision windows
  // last (measured: no gain at c2, so off). Tasks are addressed by the ordinal o of the window
  // in this warp's order.
  const int n_own = nJ > warp ? (nJ - warp + kNW - 1) / kNW : 0;
  const int n_own_full = nF > warp ? (nF - warp + kNW - 1) / kNW : 0;
  const bool full_last = QE_DECODE_FULL_LAST && (warp & 1) && n_own_full > 0 && n_own_full < n_own;
  auto jmap = [&](int o) {
    const int r = !full_last ? o : (o < n_own - n_own_full ? n_own_full + o : o - (n_own - n_own_full));
    return warp + kNW * r;
  };
  auto advance = [&](int& o, int& pg) {
    if (++pg >= n_tasks(jmap(o))) {
      pg = 0;
      ++o;
    }
  };
  // Index prefetch: lane l holds the window id and the page ids (full, tail) or the ledger
  // slot (INT2) of this warp's window of ordinal rb + l, so issuing a copy never waits on a
  // dependent global load. Reloaded every 32 windows.
  int e_win = -1, e_id[4] = {-1, -1, -1, -1}, rb = -32;
  auto load_ids = [&](int base) {
    rb = base;
    const int jj = base + lane < n_own ? jmap(base + lane) : nJ;
    e_win = -1;
#pragma unroll
    for (int p = 0; p < 4; ++p) e_id[p] = -1;
    if (jj < nJ) {
      const int kd = kind_of(jj);
      const int win = kd == 0 ? st.full_list[ub + f0 + jj]
                              : (kd == 1 ? st.int2_list[ub + q0 + (jj - nF)] : a.tail_win);
      if (win >= 0 && win < st.Wmax) {
        e_win = win;
        if (kd == 1) {
          e_id[0] = st.win_slot[ub + win];
        } else {
#pragma unroll
          for (int p = 0; p < 4; ++p)
            if (p < ppw) e_id[p] = st.win_pages[(ub + win) * ppw + p];
        }
      }
    }
  };
  // issue the copies of task (window ordinal r, page pg) into stage s (all lanes call)
  auto issue = [&](int r, int pg, int s) {
    const int j = jmap(r);
    if (r - rb >= 32) load_ids(r - r % 32);
    const int src = r - rb;
    const int win = __shfl_sync(0xffffffffu, e_win, src);
    const int sel = pg == 0 ? e_id[0] : (pg == 1 ? e_id[1] : (pg == 2 ? e_id[2] : e_id[3]));
    const int id = __shfl_sync(0xffffffffu, sel, src);
    uint8_t* dst = ring + s * STAGE;
    uint64_t* bar = &bars[s];
    const int k = kind_of(j);
    fence_proxy_async_smem();
    if (lane != 0) return;
    if (k == 0) {
      // full-precision page: 2 * D/64 swizzled TMA boxes, then the page's norms
      if (win < 0 || id < 0 || id >= st.P) {
        qe_record_error(st.status, QE_ERR_DEVICE_FAULT, u);
        mbar_arrive_expect_tx(bar, 0);
        return;
      }
      const uint32_t nb = QE_PAGE * G * 4;
      mbar_arrive_expect_tx(bar, PAGE_BYTES + nb);
      const int row0 = (u * st.P + id) * 2 * QE_PAGE;
#pragma unroll
      for (int part = 0; part < 2; ++part)
#pragma unroll
        for (int xb = 0; xb < D / 64; ++xb)
          tc::tma_load_2d(dst + (part * (D / 64) + xb) * 2048, &tmP, xb * 64, row0 + part * QE_PAGE, bar);
      bulk_g2s(dst + PAGE_BYTES, st.norms + ((size_t)u * st.norm_pitch + (size_t)win * w + pg * QE_PAGE) * G, nb,
               bar);
      return;
    }
    if (k == 1) {
      if (win < 0 || id < 0 || id >= st.S) {
        qe_record_error(st.status, QE_ERR_DEVICE_FAULT, u);
        mbar_arrive_expect_tx(bar, 0);
        return;
      }
      const uint32_t nb = (uint32_t)(w * G * 4);
      mbar_arrive_expect_tx(bar, (uint32_t)st.slot_bytes + nb);
      bulk_g2s(dst, st.slots + ((size_t)u * st.S + id) * st.slot_bytes, (uint32_t)st.slot_bytes, bar);
      bulk_g2s(dst + PAGE_BYTES, st.norms + ((size_t)u * st.norm_pitch + (size_t)win * w) * G, nb, bar);
    } else {
      if (win < 0 || id < 0 || id >= st.P) {
        qe_record_error(st.status, QE_ERR_DEVICE_FAULT, u);
        mbar_arrive_expect_tx(bar, 0);
        return;
      }
      const uint8_t* src_p = st.pages + ((size_t)u * st.P + id) * st.page_bytes;
      {
        mbar_arrive_expect_tx(bar, PAGE_BYTES);
        bulk_g2s(dst, src_p, PAGE_BYTES, bar);
      }
    }
  };

  // softmax bookkeeping for one batch: s[i][h] are the scores of the group's SB tokens
  // (-inf where invalid); on return they hold the weights 2^(s - m). The running max m
  // starts at a finite -1e30 so that 2^(-inf - m) = 0 needs no guard. One rarely taken
  // branch per batch covers every head.
  auto online = [&](float (&s)[SB][G]) {
    float mb[G];
    bool grow = false;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      mb[h] = s[0][h];
#pragma unroll
      for (int i = 1; i < SB; ++i) mb[h] = fmaxf(mb[h], s[i][h]);
      grow |= mb[h] > m[h] + kRescale;
    }
    if (grow) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float mn = mb[h] > m[h] + kRescale ? mb[h] : m[h];
        const float f = ex2(m[h] - mn);
        const float2 f2 = make_float2(f, f);
#pragma unroll
        for (int e = 0; e < NP; ++e) acc[h][e] = __fmul2_rn(acc[h][e], f2);
        zacc[h] = __fmul2_rn(zacc[h], f2);
        lsum[h] *= f;
        lw[h] *= f;
        nw[h] *= f;
        m[h] = mn;
      }
    }
#pragma unroll
    for (int i = 0; i < SB; ++i)
#pragma unroll
      for (int h = 0; h < G; ++h) s[i][h] = ex2(s[i][h] - m[h]);
  };

  // sum every score over the LPT lanes of its token (pairs of heads added as f32x2)
  auto butterfly = [&](float (&s)[SB][G]) {
#pragma unroll
    for (int o = LPT / 2; o; o >>= 1)
#pragma unroll
      for (int i = 0; i < SB; ++i) {
#pragma unroll
        for (int h = 0; h + 1 < G; h += 2) {
          const float2 r = make_float2(__shfl_xor_sync(0xffffffffu, s[i][h], o),
                                       __shfl_xor_sync(0xffffffffu, s[i][h + 1], o));
          const float2 v = __fadd2_rn(make_float2(s[i][h], s[i][h + 1]), r);
          s[i][h] = v.x;
          s[i][h + 1] = v.y;
        }
        if constexpr (G % 2) s[i][G - 1] += __shfl_xor_sync(0xffffffffu, s[i][G - 1], o);
      }
  };

  // window sums of one token: lw += p, nw += p * n (pairs of heads as f32x2)
  auto window_sums = [&](const float (&p)[G], const float* n) {
#pragma unroll
    for (int h = 0; h + 1 < G; h += 2) {
      const float2 pp = make_float2(p[h], p[h + 1]);
      const float2 l2 = __fadd2_rn(make_float2(lw[h], lw[h + 1]), pp);
      // n + h is 8-byte aligned only when G is even (n = norms + t * G)
      const float2 nn = G % 2 == 0 ? *reinterpret_cast<const float2*>(n + h) : make_float2(n[h], n[h + 1]);
      const float2 n2 = ffma2(pp, nn, make_float2(nw[h], nw[h + 1]));
      lw[h] = l2.x;
      lw[h + 1] = l2.y;
      nw[h] = n2.x;
      nw[h + 1] = n2.y;
    }
    if constexpr (G % 2) {
      lw[G - 1] += p[G - 1];
      nw[G - 1] = fmaf(p[G - 1], n[G - 1], nw[G - 1]);
    }
  };

  // QK of one row of K for every head
  auto qk_row = [&](const float2 (&kx)[NP], float (&out)[G]) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float2 d2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int e = 0; e < NP; ++e) d2 = ffma2(q[h][e], kx[e], d2);
      out[h] = d2.x + d2.y;
    }
  };

  // PV of one row of V for every head: acc[h] += p[h] * v
  auto pv_row = [&](const float2 (&vx)[NP], const float (&p)[G]) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float2 p2 = make_float2(p[h], p[h]);
#pragma unroll
      for (int e = 0; e < NP; ++e) acc[h][e] = ffma2(p2, vx[e], acc[h][e]);
    }
  };

  int o = 0, pg = 0;                  // window ordinal and page being computed
  int io = 0, ipg = 0, issued = 0;    // next task to copy
  for (int s = 0; s < kNST - 1 && io < n_own; ++s) {
    issue(io, ipg, s);
    advance(io, ipg);
    ++issued;
  }
  int k = 0;
  bool ok = true;
  const int g8 = lane >> 2, t4 = lane & 3;

  // ---- full-precision pages on the tensor cores ----
  // S = Q K^T with A = the G query rows (padded to 16, raw q), B = 8-token tiles of K
  // (ldmatrix); lane (g8, t4) then holds head g8's scores of tokens 2t4, 2t4+1, 8+2t4, 9+2t4.
  // O^T = V^T P^T with A = V^T (ldmatrix.trans) and B = P^T taken straight from those
  // registers, split into two 16-bit parts so the product keeps float32 accuracy. At the end
  // the partial (per head: max, sum of weights, O as [G][D]) goes to the stage consumed last
  // (the next copy targets it only after the merge below).
  auto mma_phase = [&]() -> const float* {
      uint32_t qa[D / 16][2];
      {
        const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
            reinterpret_cast<const T*>(a.q) + ((size_t)b * st.Hq + (size_t)kvh * G + (g8 < G ? g8 : 0)) * D);
  #pragma unroll
        for (int kc = 0; kc < D / 16; ++kc) {
          qa[kc][0] = g8 < G ? qrow[kc * 8 + t4] : 0u;
          qa[kc][1] = g8 < G ? qrow[kc * 8 + 4 + t4] : 0u;
        }
      }
      float oacc[D / 16][4];
  #pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) oacc[mt][0] = oacc[mt][1] = oacc[mt][2] = oacc[mt][3] = 0.f;
      float mh = -1e30f, lh = 0.f, lwh = 0.f, nwh = 0.f;  // head g8: running max, sums
      const float hmask = g8 < G ? 1.f : 0.f;
      while (o < n_own && kind_of(jmap(o)) == 0) {
        if (io < n_own) {
          issue(io, ipg, issued % kNST);
          advance(io, ipg);
          ++issued;
        }
        const int s = k % kNST;
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[s], (k / kNST) & 1, st.status, 1000 + u));
        if (!ok) break;
        const uint8_t* stage = ring + s * STAGE;
        const float* nrm = reinterpret_cast<const float*>(stage + PAGE_BYTES);
        float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
  #pragma unroll
        for (int kc2 = 0; kc2 < D / 32; ++kc2) {
          uint32_t kb[4];
          ldsm_x4(kb, stage + swz<D>(0, lane & 7, kc2 * 32 + (lane >> 3) * 8));
          MmaOp<T>::run(c0, qa[2 * kc2][0], 0u, qa[2 * kc2][1], 0u, kb[0], kb[1]);
          MmaOp<T>::run(c0, qa[2 * kc2 + 1][0], 0u, qa[2 * kc2 + 1][1], 0u, kb[2], kb[3]);
          ldsm_x4(kb, stage + swz<D>(0, 8 + (lane & 7), kc2 * 32 + (lane >> 3) * 8));
          MmaOp<T>::run(c1, qa[2 * kc2][0], 0u, qa[2 * kc2][1], 0u, kb[0], kb[1]);
          MmaOp<T>::run(c1, qa[2 * kc2 + 1][0], 0u, qa[2 * kc2 + 1][1], 0u, kb[2], kb[3]);
        }
        float mx = fmaxf(fmaxf(c0[0], c0[1]), fmaxf(c1[0], c1[1]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float ms = mx * a.scale_log2;
        const bool grow = ms > mh + kRescale;
        if (__any_sync(0xffffffffu, grow)) {
          const float mn = grow ? ms : mh;
          const float f = ex2(mh - mn);
          lh *= f;
          lwh *= f;
          nwh *= f;
          mh = mn;
          // O^T column pair (2 t4, 2 t4 + 1) belongs to heads held by lanes 8 t4 and 8 t4 + 4
          const float fa = __shfl_sync(0xffffffffu, f, 8 * t4);
          const float fb = __shfl_sync(0xffffffffu, f, 8 * t4 + 4);
  #pragma unroll
          for (int mt = 0; mt < D / 16; ++mt) {
            oacc[mt][0] *= fa;
            oacc[mt][1] *= fb;
            oacc[mt][2] *= fa;
            oacc[mt][3] *= fb;
          }
        }
        const float p0 = hmask * ex2(fmaf(c0[0], a.scale_log2, -mh));
        const float p1 = hmask * ex2(fmaf(c0[1], a.scale_log2, -mh));
        const float p2 = hmask * ex2(fmaf(c1[0], a.scale_log2, -mh));
        const float p3 = hmask * ex2(fmaf(c1[1], a.scale_log2, -mh));
        const float psum = (p0 + p1) + (p2 + p3);
        lh += psum;
        lwh += psum;
        if (g8 < G) {
          nwh = fmaf(p0, nrm[(2 * t4) * G + g8], nwh);
          nwh = fmaf(p1, nrm[(2 * t4 + 1) * G + g8], nwh);
          nwh = fmaf(p2, nrm[(8 + 2 * t4) * G + g8], nwh);
          nwh = fmaf(p3, nrm[(9 + 2 * t4) * G + g8], nwh);
        }
        uint32_t ph0, pl0, ph1, pl1;
        MmaOp<T>::split(p0, p1, ph0, pl0);
        MmaOp<T>::split(p2, p3, ph1, pl1);
  #pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          uint32_t va[4];
          ldsm_x4_t(va, stage + swz<D>(1, ((lane >> 4) << 3) + (lane & 7), mt * 16 + ((lane >> 3) & 1) * 8));
          MmaOp<T>::run(oacc[mt], va[0], va[1], va[2], va[3], ph0, ph1);
          MmaOp<T>::run(oacc[mt], va[0], va[1], va[2], va[3], pl0, pl1);
        }
        __syncwarp();
        if (pg + 1 >= ppw) {
          // end of a window: its partial (m, sum p, sum p n) per head
          float l2 = lwh + __shfl_xor_sync(0xffffffffu, lwh, 1);
          l2 += __shfl_xor_sync(0xffffffffu, l2, 2);
          float n2 = nwh + __shfl_xor_sync(0xffffffffu, nwh, 1);
          n2 += __shfl_xor_sync(0xffffffffu, n2, 2);
          if (g8 < G) {
            // slot 0 holds the window's partial, the other lanes mark the remaining slots unused
            float* wp = a.win_part + (ub + list_idx(jmap(o))) * win_part_floats(D, G) + g8;
#pragma unroll
            for (int slot = t4; slot < TPS; slot += 4) {
              wp[slot * 3 * G] = slot == 0 ? mh : -1e30f;
              wp[slot * 3 * G + G] = slot == 0 ? l2 : 0.f;
              wp[slot * 3 * G + 2 * G] = slot == 0 ? n2 : 0.f;
            }
          }
          lwh = 0.f;
          nwh = 0.f;
        }
        advance(o, pg);
        ++k;
      }
    lh += __shfl_xor_sync(0xffffffffu, lh, 1);
    lh += __shfl_xor_sync(0xffffffffu, lh, 2);
    float* fo = reinterpret_cast<float*>(ring + ((k + kNST - 1) % kNST) * STAGE);
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      if (2 * t4 < G) {
        fo[(2 * t4) * D + mt * 16 + g8] = oacc[mt][0];
        fo[(2 * t4) * D + mt * 16 + g8 + 8] = oacc[mt][2];
      }
      if (2 * t4 + 1 < G) {
        fo[(2 * t4 + 1) * D + mt * 16 + g8] = oacc[mt][1];
        fo[(2 * t4 + 1) * D + mt * 16 + g8 + 8] = oacc[mt][3];
      }
    }
    if (t4 == 0 && g8 < G) {
      fo[G * D + g8] = mh;
      fo[G * D + G + g8] = lh;
    }
    __syncwarp();
    return fo;
  };

  // ---- SIMT state for the INT2 and tail windows ----
  auto load_q = [&]() {
    const T* qb = reinterpret_cast<const T*>(a.q) + ((size_t)b * st.Hq + (size_t)kvh * G) * D;
    const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      load_row<T, DPL>(qb + (size_t)h * D, sub, sw, q[h]);
      float2 s2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int e = 0; e < NP; ++e) {
        q[h][e] = __fmul2_rn(q[h][e], sc2);
        s2 = __fadd2_rn(s2, q[h][e]);
      }
      qsum[h] = s2.x + s2.y;
      qsum2[h] = fmaf(4.f, s2.x, s2.y);
    }
  };
  auto simt_empty = [&]() {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      zacc[h] = make_float2(0.f, 0.f);
      m[h] = -1e30f;
      lsum[h] = 0.f;
      lw[h] = 0.f;
      nw[h] = 0.f;
#pragma unroll
      for (int e = 0; e < NP; ++e) acc[h][e] = make_float2(0.f, 0.f);
    }
  };
  // merge a tensor-core partial (at a window boundary) into the SIMT state; lane group 0
  // takes its values, every lane group rescales to the common maximum
  auto merge = [&](const float* fo) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float mf = fo[G * D + h], lf = fo[G * D + G + h];
      const float M = fmaxf(m[h], mf);
      const float fs = ex2(m[h] - M), ff = grp == 0 ? ex2(mf - M) : 0.f;
      const float2 fs2 = make_float2(fs, fs), ff2 = make_float2(ff, ff);
      lsum[h] = fmaf(lsum[h], fs, lf * ff);
      zacc[h] = __fmul2_rn(zacc[h], fs2);
#pragma unroll
      for (int e = 0; e < NP; ++e) {
        // register pair e of chunk c = e / 4 sits in memory chunk c ^ sw
        const int d = DPL * sub + 8 * ((e / 4) ^ sw) + 2 * (e % 4);
        acc[h][e] = ffma2(make_float2(fo[h * D + d], fo[h * D + d + 1]), ff2, __fmul2_rn(acc[h][e], fs2));
      }
      m[h] = M;
    }
    __syncwarp();
  };

  // ---- INT2 ledger entries and the tail window on the CUDA cores ----
  auto simt_phase = [&]() {
    while (ok && o < n_own && kind_of(jmap(o)) != 0) {
      if (io < n_own) {
        issue(io, ipg, issued % kNST);
        advance(io, ipg);
        ++issued;
      }
      const int s = k % kNST;
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[s], (k / kNST) & 1, st.status, 1000 + u));
      if (!ok) break;
      const uint8_t* stage = ring + s * STAGE;
      const int j = jmap(o);
      const int kind = kind_of(j);
      const float* nrm = reinterpret_cast<const float*>(stage + PAGE_BYTES);
      if (kind == 2) {
        // ---- a page of the tail window: mask tokens past its length, keep raw scores ----
        const T* Ks = reinterpret_cast<const T*>(stage);
        const T* Vs = Ks + QE_PAGE * D;
        const int valid = min(QE_PAGE, a.tail_len - pg * QE_PAGE);
        for (int t0 = 0; t0 < valid; t0 += SBT) {
          float sc[SB][G];
  #pragma unroll
          for (int i = 0; i < SB; ++i) {
            float2 kx[NP];
            load_row<T, DPL>(Ks + (size_t)(t0 + i * TPS + grp) * D, sub, sw, kx);
            qk_row(kx, sc[i]);
          }
          butterfly(sc);
  #pragma unroll
          for (int i = 0; i < SB; ++i) {
            const int t = t0 + i * TPS + grp;
            if (t >= valid) {
  #pragma unroll
              for (int h = 0; h < G; ++h) sc[i][h] = -INFINITY;
            } else if (sub == 0) {
  #pragma unroll
              for (int h = 0; h < G; ++h) a.tail_s[((size_t)u * w + pg * QE_PAGE + t) * G + h] = sc[i][h];
            }
          }
          online(sc);
  #pragma unroll
          for (int i = 0; i < SB; ++i) {
            const int t = t0 + i * TPS + grp;
  #pragma unroll
            for (int h = 0; h < G; ++h) lw[h] += sc[i][h];
            if (t < valid) {
              float2 vx[NP];
              load_row<T, DPL>(Vs + (size_t)t * D, sub, sw, vx);
              pv_row(vx, sc[i]);
            }
          }
        }
      } else {
        // ---- INT2 ledger entry: codes K [w][D/4] | codes V | meta K [w][D/16] | meta V ----
        const uint8_t* kc = stage;
        const uint8_t* vc = stage + w * D / 4;
        const uint32_t* km = reinterpret_cast<const uint32_t*>(stage + w * D / 2);
        const uint32_t* vm = km + w * D / 16;
        for (int t0 = 0; t0 < w; t0 += SBT) {
          float sc[SB][G];
  #pragma unroll
          for (int i = 0; i < SB; ++i) {
            const int t = t0 + i * TPS + grp;
            float2 x[NP];
            decode_codes<NP>(load_codes<DPL>(kc + t * (D / 4), sub, sw), x);
            const uint32_t mt = km[t * (D / 16) + gi];
            const float s4 = 4.f * meta_scale(mt), z = meta_zero(mt);
            float d[G];
            qk_row(x, d);
            // q . x = qsum2 + (q . c) / 4, so q . k = s (q . c) + z qsum = 4s (q . x) + z qsum - 4s qsum2
  #pragma unroll
            for (int h = 0; h + 1 < G; h += 2) {
              const float2 c0 = ffma2(make_float2(z, z), make_float2(qsum[h], qsum[h + 1]),
                                      __fmul2_rn(make_float2(-s4, -s4), make_float2(qsum2[h], qsum2[h + 1])));
              const float2 r = ffma2(make_float2(s4, s4), make_float2(d[h], d[h + 1]), c0);
              sc[i][h] = r.x;
              sc[i][h + 1] = r.y;
            }
            if constexpr (G % 2)
              sc[i][G - 1] = fmaf(s4, d[G - 1], fmaf(z, qsum[G - 1], -s4 * qsum2[G - 1]));
          }
          butterfly(sc);
          online(sc);
  #pragma unroll
          for (int i = 0; i < SB; ++i) {
            const int t = t0 + i * TPS + grp;
            window_sums(sc[i], nrm + t * G);
            float2 x[NP];
            decode_codes<NP>(load_codes<DPL>(vc + t * (D / 4), sub, sw), x);
            const uint32_t mt = vm[t * (D / 16) + gi];
            const float s4 = 4.f * meta_scale(mt), z = meta_zero(mt);
            // v = 4s * x + (z - 16s) for even elements (x = 4 + c/4), 4s * x + (z - 4s) for odd
            // ones (x = 1 + c/4): acc += (p * 4s) * x, zacc += p * (z - 16s, z - 4s)
            const float2 zz = make_float2(fmaf(-4.f, s4, z), z - s4);
            float ps[G];
  #pragma unroll
            for (int h = 0; h < G; ++h) {
              ps[h] = sc[i][h] * s4;
              zacc[h] = ffma2(make_float2(sc[i][h], sc[i][h]), zz, zacc[h]);
            }
            pv_row(x, ps);
          }
        }
      }
      __syncwarp();
      if (pg + 1 >= n_tasks(j)) {
        // end of a window: each lane group's leader records its (max, sum p, sum p n) per head
        // in its own slot (no cross-group reduction here: the score update folds the slots)
        if (kind != 2 && sub == 0) {
          float* ws = a.win_part + (ub + list_idx(j)) * win_part_floats(D, G) + grp * 3 * G;
          if constexpr (G == 4) {
            reinterpret_cast<float4*>(ws)[0] = make_float4(m[0], m[1], m[2], m[3]);
            reinterpret_cast<float4*>(ws + G)[0] = make_float4(lw[0], lw[1], lw[2], lw[3]);
            reinterpret_cast<float4*>(ws + 2 * G)[0] = make_float4(nw[0], nw[1], nw[2], nw[3]);
          } else {
#pragma unroll
            for (int h = 0; h < G; ++h) {
              ws[h] = m[h];
              ws[G + h] = lw[h];
              ws[2 * G + h] = nw[h];
            }
          }
        }
  #pragma unroll
        for (int h = 0; h < G; ++h) {
          lsum[h] += lw[h];
          lw[h] = 0.f;
          nw[h] = 0.f;
        }
      }
      advance(o, pg);
      ++k;
    }
  };

  // at most two segments (full then the rest, or the rest then full); each phase has one call
  // site so that it is inlined and its state stays in registers
  simt_empty();
  for (int seg = 0; seg < 2 && ok && o < n_own; ++seg) {
    if (kind_of(jmap(o)) == 0) {
      merge(mma_phase());
    } else {
      load_q();
      simt_phase();
    }
  }
  if (!ok) {  // drain copies still in flight if a wait gave up
    for (; k < issued; ++k) mbar_wait_bounded(&bars[k % kNST], (k / kNST) & 1, st.status, 2000 + u);
  }

  // ---- merge lane groups, then warps, into the CTA's partial ----
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float mx = m[h];
#pragma unroll
    for (int o = LPT; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float f = ex2(m[h] - mx);
    lsum[h] *= f;
    const float2 f2 = make_float2(f, f);
#pragma unroll
    for (int e = 0; e < NP; ++e) acc[h][e] = __fmul2_rn(__fadd2_rn(acc[h][e], zacc[h]), f2);
#pragma unroll
    for (int o = LPT; o < 32; o <<= 1) {
      lsum[h] += __shfl_xor_sync(0xffffffffu, lsum[h], o);
#pragma unroll
      for (int e = 0; e < NP; ++e) {
        acc[h][e].x += __shfl_xor_sync(0xffffffffu, acc[h][e].x, o);
        acc[h][e].y += __shfl_xor_sync(0xffffffffu, acc[h][e].y, o);
      }
    }
    m[h] = mx;
  }
  __syncthreads();
  float* mw = reinterpret_cast<float*>(smem);  // [kNW][G]
  float* lwv = mw + kNW * G;                   // [kNW][G]
  float* aw = lwv + kNW * G;                   // [kNW][G][D]
  float* cm = aw + kNW * G * D;                // [G]     CTA partial: max,
  float* cl = cm + QE_MAX_G;                   // [G]     sum of weights,
  float* ca = cl + QE_MAX_G;                   // [G][D]  weighted values (read by the cluster)
  float* pm = ca + G * D;                      // [S][G]  every CTA's max,
  float* pl = pm + QE_MAX_SPLITS_CLUSTER * QE_MAX_G;  // [S][G] sum of weights,
  float* pf = pl + QE_MAX_SPLITS_CLUSTER * QE_MAX_G;  // [S][G] and rescale factor
  float* gl = pf + QE_MAX_SPLITS_CLUSTER * QE_MAX_G;  // [G] unit sum of weights
  float* lse = gl + QE_MAX_G;                         // [G] unit log2-sum-exp
  float* red = lse + QE_MAX_G;                        // [kNW]
  if (lane < LPT) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      if (lane == 0) {
        mw[warp * G + h] = m[h];
        lwv[warp * G + h] = lsum[h];
      }
#pragma unroll
      for (int e = 0; e < NP; ++e) {
        // register pair e of chunk c = e / 4 sits in memory chunk c ^ sw
        const int d = DPL * sub + 8 * ((e / 4) ^ sw) + 2 * (e % 4);
        aw[((size_t)warp * G + h) * D + d] = acc[h][e].x;
        aw[((size_t)warp * G + h) * D + d + 1] = acc[h][e].y;
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
    const int h = i / D;
    float Mx = mw[h];
#pragma unroll
    for (int x = 1; x < kNW; ++x) Mx = fmaxf(Mx, mw[x * G + h]);
    float L = 0.f, A = 0.f;
#pragma unroll
    for (int x = 0; x < kNW; ++x) {
      const float f = ex2(mw[x * G + h] - Mx);
      L = fmaf(lwv[x * G + h], f, L);
      A = fmaf(aw[((size_t)x * G + h) * D + i % D], f, A);
    }
    ca[i] = A;
    if (i % D == 0) {
      cm[h] = Mx;
      cl[h] = L;
    }
  }

  // ---- the unit's S CTAs form one cluster: merge the partials through distributed
  // shared memory; each CTA writes its share of the output and the scores of its windows ----
  const int S = a.splits;
  cluster_sync();
  for (int i = threadIdx.x; i < S * G; i += blockDim.x) {
    pm[i] = ld_cluster(cm + i % G, (uint32_t)(i / G));
    pl[i] = ld_cluster(cl + i % G, (uint32_t)(i / G));
  }
  __syncthreads();
  if (threadIdx.x < G) {
    const int h = threadIdx.x;
    float M = pm[h];
    for (int r = 1; r < S; ++r) M = fmaxf(M, pm[r * G + h]);
    float L = 0.f;
    for (int r = 0; r < S; ++r) {
      const float f = ex2(pm[r * G + h] - M);
      pf[r * G + h] = f;
      L = fmaf(pl[r * G + h], f, L);
    }
    gl[h] = L;
    lse[h] = M + log2f(L);
  }
  __syncthreads();
  {
    const int per = (G * D + S - 1) / S;
    const int i1 = min((split + 1) * per, G * D);
    for (int i = split * per + threadIdx.x; i < i1; i += blockDim.x) {
      const int h = i / D;
      float A = 0.f;
      for (int r = 0; r < S; ++r) A = fmaf(ld_cluster(ca + i, (uint32_t)r), pf[r * G + h], A);
      a.out[((size_t)b * st.Hq + (size_t)kvh * G + h) * D + i % D] = A / gl[h];
    }
  }
  // exact attention mass and perturbation of this step for the windows this CTA streamed
  for (int jj = threadIdx.x; jj < nF + nQ; jj += blockDim.x) {
    const int li = list_idx(jj);
    const int win = jj < nF ? st.full_list[ub + li] : st.int2_list[ub + li - nf];
    if (win < 0 || win >= st.Wmax) continue;
    float dm = 0.f, dp = 0.f;
    const float* wp = a.win_part + (ub + li) * win_part_floats(D, G);
#pragma unroll
    for (int slot = 0; slot < TPS; ++slot) {
      const float* ws = wp + slot * 3 * G;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float f = ex2(ws[h] - lse[h]);
        dm = fmaf(ws[G + h], f, dm);
        dp = fmaf(ws[2 * G + h], f, dp);
      }
    }
    st.mass[ub + win] += dm;
    st.pert[ub + win] += dp;
  }
  // tail tokens (last CTA of the cluster): cumulative per-token attention and window mass
  if (has_tail) {
    float tm = 0.f;
    for (int i = threadIdx.x; i < a.tail_len * G; i += blockDim.x) {
      const int h = i % G;
      const float pv = ex2(a.tail_s[(size_t)u * w * G + i] - lse[h]);
      st.tail_p[(size_t)u * w * G + i] += pv;
      tm += pv;
    }
    tm = warp_sum(tm);
    if (lane == 0) red[warp] = tm;
    __syncthreads();
    if (threadIdx.x == 0) {
      float s2 = 0.f;
      for (int x = 0; x < kNW; ++x) s2 += red[x];
      st.mass[ub + a.tail_win] += s2;
    }
  }
  cluster_sync();  // keep this CTA's partial alive until every CTA of the cluster has read it
}

template <typename T, int D, int G>
int launch_decode_t(qe_ctx* c, const void* q, float* out, cudaStream_t s, const void* k_new,
                    const void* v_new) {
  constexpr int STAGE = StageLayout<D, G>::BYTES;
  const size_t smem = 1024 + (size_t)kNW * kNST * STAGE + kNW * kNST * 8;  // + alignment slack
  static_assert((size_t)(kNW * G * (D + 2) + 2 * QE_MAX_G + G * D + 3 * QE_MAX_SPLITS_CLUSTER * QE_MAX_G +
                         2 * QE_MAX_G + kNW) * 4 <= (size_t)kNW * kNST * STAGE,
                "merge area");
  auto kern = decode_kernel<T, D, G>;
  // One-time set-up per instantiation and device (kept out of the per-step path and of graph
  // capture): clusters[S] = how many clusters of S CTAs can be resident at once.
  static QeOnce once;
  static int clusters_of[QE_MAX_DEVICES][QE_MAX_SPLITS_CLUSTER + 1];
  int dev = 0;
  const int se = qe_once_per_device(once, &dev, [&](int d) {
    QE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    QE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
    for (int S = 1; S <= QE_MAX_SPLITS_CLUSTER; ++S) {
      cudaLaunchConfig_t qc = {};
      cudaLaunchAttribute qa[1];
      qa[0].id = cudaLaunchAttributeClusterDimension;
      qa[0].val.clusterDim.x = S;
      qa[0].val.clusterDim.y = 1;
      qa[0].val.clusterDim.z = 1;
      qc.gridDim = dim3(S);
      qc.blockDim = dim3(kNW * 32);
      qc.dynamicSmemBytes = smem;
      qc.attrs = qa;
      qc.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &qc) != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
      }
      clusters_of[d][S] = n;
    }
    return QE_OK;
  });
  if (se) return se;
  const int* clusters = clusters_of[dev];
  DecodeArgs a{};
  a.st = make_state(c);
  // the page pool as a 2-D tensor [units * P * 32 rows][D] for the swizzled TMA page loads
  CUtensorMap tmP;
  {
    const unsigned long long rows = (unsigned long long)a.st.U * a.st.P * 2 * QE_PAGE;
    if (rows >= (1ull << 31)) return QE_ERR_UNSUPPORTED_SHAPE;
    const int e = tc::make_map(&tmP, a.st.pages, c->cfg.dtype == QE_BF16, D, rows, 64, QE_PAGE);
    if (e) return e;
  }
  a.q = q;
  a.out = out;
  a.win_part = c->win_part;
  a.tail_s = c->tail_s;
  a.tail_win = c->complete;
  a.tail_len = c->n - c->complete * c->cfg.window;
  a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
  a.k_new = static_cast<const uint4*>(k_new);
  a.v_new = static_cast<const uint4*>(v_new);
  a.tailV = reinterpret_cast<uint4*>(c->tailV);
  a.append_pos = c->n - 1;
  const int U = c->lay.units;
  // The largest split count whose U clusters are all resident in one wave, never more splits
  // than windows per tier nor than the configured maximum.
  const int nwin = c->n_full_max > c->n_int2_max ? c->n_full_max : c->n_int2_max;
  int S = 1;
  for (int t = QE_MAX_SPLITS_CLUSTER; t >= 1; --t)
    if (clusters[t] >= U && t <= nwin && t <= c->cfg.max_splits) {
      S = t;
      break;
    }
  a.splits = S;
  cudaLaunchConfig_t lc = {};
  cudaLaunchAttribute la[1];
  la[0].id = cudaLaunchAttributeClusterDimension;
  la[0].val.clusterDim.x = S;
  la[0].val.clusterDim.y = 1;
  la[0].val.clusterDim.z = 1;
  lc.gridDim = dim3(U * S);
  lc.blockDim = dim3(kNW * 32);
  lc.dynamicSmemBytes = smem;
  lc.stream = s;
  lc.attrs = la;
  lc.numAttrs = 1;
  QE_CUDA_TRY(cudaLaunchKernelEx(&lc, kern, tmP, a));
  return QE_OK;
}

template <typename T, int D>
int launch_decode_g(qe_ctx* c, const void* q, float* out, cudaStream_t s, const void* k, const void* v) {
  switch (c->G) {
    case 1: return launch_decode_t<T, D, 1>(c, q, out, s, k, v);
    case 2: return launch_decode_t<T, D, 2>(c, q, out, s, k, v);
    case 4: return launch_decode_t<T, D, 4>(c, q, out, s, k, v);
    case 5: return launch_decode_t<T, D, 5>(c, q, out, s, k, v);
    case 8: return launch_decode_t<T, D, 8>(c, q, out, s, k, v);
    default: return QE_ERR_UNSUPPORTED_SHAPE;
  }
}

}  // namespace

int launch_decode(qe_ctx* c, const void* q, float* out, cudaStream_t s, const void* k_new,
                  const void* v_new) {
  const bool bf = c->cfg.dtype == QE_BF16;
  if (c->cfg.D == 128)
    return bf ? launch_decode_g<__nv_bfloat16, 128>(c, q, out, s, k_new, v_new)
              : launch_decode_g<__half, 128>(c, q, out, s, k_new, v_new);
  return bf ? launch_decode_g<__nv_bfloat16, 64>(c, q, out, s, k_new, v_new)
            : launch_decode_g<__half, 64>(c, q, out, s, k_new, v_new);
}
