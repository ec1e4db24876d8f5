// Split-K GQA decode attention over the full-precision and INT2 tiers, fused with the
// cumulative window scores and (optionally) the append of the step's token.
//
// "Resumo Técnico: QEvict" - Mecanismos Principais: window-level routing driven by
// attention accumulated over time (Pontuação Cumulativa); the recoverable INT2 tier stays
// readable by attention (Metodologia 2); GQA decode path (Implementação).
// "Resumo Técnico: CriticalKV" - Etapa 2: the perturbation score A_i * ||V_i W_O||_1.
//
// Work split. Per unit u = (b, g) the live windows are [full windows | tail | INT2 windows].
// The unit's S CTAs form one thread-block cluster; CTA s takes the s-th S-th of the full
// windows and of the INT2 windows (the tail counts as one more INT2 window of the last CTA),
// so every SM streams the same mix of bandwidth-heavy full pages and compact INT2 entries.
// Inside a CTA each warp takes whole windows round-robin and streams them through its own
// ring of shared-memory stages (completion on an mbarrier per stage): a full or tail page
// arrives as 128-byte-swizzled TMA boxes from a tensor map over the page pool, an INT2 ledger
// entry as one 1-D bulk copy, each with its tokens' projected-value norms.
//
// Every tier runs on the warp-level tensor cores (mma.sync, f32 accumulate) in one register
// layout: the G query heads of the group are the rows of S = Q K^T (padded to 16), 16 tokens
// are its columns, so lane (r, t) holds head r's scores of tokens 2t, 2t+1, 8+2t, 9+2t - which
// is exactly the B fragment of O^T = V^T P^T. A decode step has G <= 8 query rows per KV head;
// a tcgen05 tile (M >= 64) would be mostly padding and its TMEM round trip buys nothing on a
// path that HBM bounds, so the decode stays on mma.sync.
//
// Full-precision pages: S from ldmatrix K tiles, P split into two 16-bit parts of the cache
// dtype (hi + residual) so O keeps float32 accuracy, V^T by ldmatrix.trans.
//
// INT2 blocks (16 tokens, layout in int2_block.cuh): a K or V value is c*s + z with a 2-bit code
// c and an fp16 scale s and zero z per 16-element group. The codes enter the MMA exactly as
// fp16 subnormals c * 4^i * 2^-24 (one mask per register); per group g
//   S += s_g * (Q_g . C_g)  (one MMA per 8 tokens, then an f32x2 FMA by the token scales),
//   S += Z (sum of q over each group)  (one m16n8k8 MMA per 8 tokens, q sums split hi + lo),
//   O_g^T += C_g^T (P * s_g)  (one MMA per group; P * s rounded once to fp16),
//   O^T += Z^T P  (one MMA per 16 tokens, P split hi + lo).
// The powers 4^i and 2^-24 are folded into q, the staged scales and the accumulator. The
// block's scales are converted to float32 once per warp into a small staging area.
//
// Scoring without a second pass: at the end of each window the warp records its
// (max, sum_i 2^(s_i-max), sum_i 2^(s_i-max) n_i) per head. After the pass the cluster merges
// the CTA partials through distributed shared memory into the unit's log-sum-exp; each CTA
// writes its share of the output and adds the exact attention mass and perturbation of the
// windows it streamed to the cumulative scores. The tail window's norms are not known yet;
// its per-token attention is accumulated instead (tail_p) and folded in when it completes.
#include <math.h>

#include "append.cuh"
#include "int2_block.cuh"
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
constexpr int kNW = QE_DECODE_NW;    // warps per CTA
#define QE_MAX_SPLITS_CLUSTER 16          // CTAs per unit (one cluster, non-portable size)
constexpr int kNST = QE_DECODE_NST;  // stages per warp
constexpr float kRescale = 8.f;  // rescale the accumulators when the max grows by > 2^8

struct DecodeArgs {
  DevState st;
  const void* q;     // [B][Hq][D]
  float* out;        // [B][Hq][D]
  float* win_part;   // [U][Wmax][3 G]: {max, sum p, sum p n} per head
  float* tail_s;     // [U][window][G]
  int splits;        // CTAs per unit = cluster size
  int tail_win, tail_len;
  float scale_log2;  // log2(e) / sqrt(D)
  // optional fused append of the step's token at position append_pos (k_new != nullptr): the
  // warp that streams the tail window writes it before issuing the tail's copies
  const uint4* k_new;
  const uint4* v_new;
  uint4* tailV;
  int append_pos;
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

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// {lo, hi} rounded to an fp16 pair (lo in the low half)
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float h_lo(uint32_t x) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(x & 0xffffu)));
}
__device__ __forceinline__ float h_hi(uint32_t x) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(x >> 16)));
}

// fp16 MMAs with f32 accumulate: m16n8k16 (A 4 regs, B 2 regs) and m16n8k8 (A 2 regs, B 1 reg)
__device__ __forceinline__ void mma_h16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  MmaOp<__half>::run(c, a0, a1, a2, a3, b0, b1);
}
__device__ __forceinline__ void mma_h8(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

// Register i (0..3) of a packed code word: the codes at bits [2i, 2i+1] of each 16-bit half as
// the fp16 subnormals c * 4^i * 2^-24.
template <int I>
__device__ __forceinline__ uint32_t code_reg(uint32_t x) {
  return x & (0x00030003u << (2 * I));
}

// Shared memory of a warp: a ring of kNST page stages (1024-byte aligned) and, elsewhere, a ring
// of kNST norm stages and the INT2 scale staging. A full-precision or tail page arrives as TMA
// boxes of 16 rows x 64 elements with the 128-byte swizzle (box (part, x) at (part * D/64 + x) *
// 2048, part 0 = K rows, 1 = V rows), so the 8 rows of every ldmatrix tile sit in distinct
// banks; an INT2 ledger entry is a 1-D bulk copy (w/16 blocks of 16*D bytes, at most a page).
// A norm stage holds the task's tokens' norms (window * G floats, runtime size).
template <int D>
struct StageLayout {
  static constexpr int PAGE_BYTES = 2 * QE_PAGE * D * 2;            // K rows then V rows
  static constexpr int BYTES = (PAGE_BYTES + 1023) / 1024 * 1024;
};
// Per-warp staging of one INT2 block's scales in float32: [K, V][t (0..3)][group][4 tokens
// 2t, 2t+1, 8+2t, 9+2t], rows padded by 4 floats so the four t rows sit in distinct banks.
template <int D>
struct ScaleStage {
  static constexpr int ROW = (D / 16) * 4 + 4;  // floats per t row
  static constexpr int FLOATS = 2 * 4 * ROW;
  static constexpr int BYTES = FLOATS * 4;
};
// bytes of one norm stage for a window of w tokens (16-byte multiple)
__host__ __device__ constexpr int norm_stage_bytes(int w, int G) { return (w * G * 4 + 15) / 16 * 16; }
// per-warp auxiliary area (norm ring, then scale staging) and the whole dynamic shared memory
template <int D>
__host__ __device__ constexpr int aux_bytes(int w, int G) { return 3 * norm_stage_bytes(w, G) + ScaleStage<D>::BYTES; }

template <typename T, int D, int G>
__global__ void __launch_bounds__(kNW * 32, QE_DECODE_MINB)
    decode_kernel(const __grid_constant__ CUtensorMap tmP, DecodeArgs a) {
  using BL = Int2Block<D>;
  constexpr int G8 = BL::G8, WPL = BL::WPL;
  using SL = StageLayout<D>;
  constexpr int PAGE_BYTES = SL::PAGE_BYTES;
  constexpr int STAGE = SL::BYTES;
  constexpr int SROW = ScaleStage<D>::ROW;
  static_assert(kNST == 3, "aux_bytes assumes three stages");
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const DevState& st = a.st;
  const int u = blockIdx.x / a.splits, split = blockIdx.x % a.splits;
  const int b = u / st.Hkv, kvh = u % st.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int w = st.window, ppw = st.ppw;
  const size_t ub = (size_t)u * st.Wmax;
  const float sl = a.scale_log2;

  // this split's share of each tier
  const int nf = st.stacks[u * 4 + 2], nq = st.stacks[u * 4 + 3];
  const int f0 = (int)((long long)nf * split / a.splits), f1 = (int)((long long)nf * (split + 1) / a.splits);
  // the last split also streams the tail window (and appends the new token): it counts as one
  // INT2 window of that split's share
  const int nqv = a.tail_len > 0 ? nq + 1 : nq;
  const int q0 = (int)((long long)nqv * split / a.splits);
  const int q1 = min(nq, (int)((long long)nqv * (split + 1) / a.splits));
  const int has_tail = (a.tail_len > 0 && split == a.splits - 1) ? 1 : 0;
  const int nF = f1 - f0, nQ = q1 - q0, nJ = nF + has_tail + nQ;

  const int NSB = norm_stage_bytes(w, G);
  uint8_t* ring = smem + warp * kNST * STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kNW * kNST * STAGE) + warp * kNST;
  uint8_t* aux = smem + kNW * kNST * STAGE + kNW * kNST * 8 + warp * aux_bytes<D>(w, G);
  uint8_t* nring = aux;                                           // [kNST][NSB]
  float* sst = reinterpret_cast<float*>(aux + kNST * NSB);        // scale staging
  if (lane == 0) {
    for (int s = 0; s < kNST; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();

  // virtual index j of this split: [0, nF) full, nF the tail (when present), then INT2
  auto kind_of = [&](int j) { return j < nF ? 0 : (j < nF + has_tail ? 2 : 1); };  // full, int2, tail
  auto list_idx = [&](int j) { return j < nF ? f0 + j : nf + q0 + (j - nF - has_tail); };
  auto n_tasks = [&](int j) {
    const int k = kind_of(j);
    return k == 0 ? ppw : (k == 1 ? 1 : (a.tail_len + QE_PAGE - 1) / QE_PAGE);
  };
  // This warp's windows are j = warp + kNW * o, o < n_own (kinds in the order above).
  const int n_own = nJ > warp ? (nJ - warp + kNW - 1) / kNW : 0;
  auto jmap = [&](int o) { return warp + kNW * o; };
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
                              : (kd == 1 ? st.int2_list[ub + q0 + (jj - nF - has_tail)] : a.tail_win);
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
  // fused append: page of the step's token (written by this warp just before the tail's copies)
  int app_pg = -1, app_page = -1;
  // issue the copies of task (window ordinal r, page pg) into stage s (all lanes call)
  auto issue = [&](int r, int pg, int s) {
    const int j = jmap(r);
    if (r - rb >= 32) load_ids(r - r % 32);
    const int src = r - rb;
    const int win = __shfl_sync(0xffffffffu, e_win, src);
    const int sel = pg == 0 ? e_id[0] : (pg == 1 ? e_id[1] : (pg == 2 ? e_id[2] : e_id[3]));
    int id = __shfl_sync(0xffffffffu, sel, src);
    uint8_t* dst = ring + s * STAGE;
    uint8_t* ndst = nring + s * NSB;
    uint64_t* bar = &bars[s];
    const int k = kind_of(j);
    if (k == 2 && pg == 0 && a.k_new != nullptr) {
      // the step's token goes into the tail window before its pages are copied
      app_page = append_token_warp(st, u, a.append_pos, a.k_new, a.v_new, a.tailV);
      app_pg = (a.append_pos % w) / QE_PAGE;
    }
    if (k == 2 && pg == app_pg) id = app_page;
    fence_proxy_async_smem();
    if (lane != 0) return;
    if (k != 1) {
      // full-precision or tail page: 2 * D/64 swizzled TMA boxes (+ the page's norms)
      if (win < 0 || id < 0 || id >= st.P) {
        qe_record_error(st.status, QE_ERR_DEVICE_FAULT, u);
        mbar_arrive_expect_tx(bar, 0);
        return;
      }
      const uint32_t nb = k == 0 ? QE_PAGE * G * 4 : 0;
      mbar_arrive_expect_tx(bar, PAGE_BYTES + nb);
      const int row0 = (u * st.P + id) * 2 * QE_PAGE;
#pragma unroll
      for (int part = 0; part < 2; ++part)
#pragma unroll
        for (int xb = 0; xb < D / 64; ++xb)
          tc::tma_load_2d(dst + (part * (D / 64) + xb) * 2048, &tmP, xb * 64, row0 + part * QE_PAGE, bar);
      if (k == 0)
        bulk_g2s(ndst, st.norms + ((size_t)u * st.norm_pitch + (size_t)win * w + pg * QE_PAGE) * G, nb, bar);
      return;
    }
    if (win < 0 || id < 0 || id >= st.S) {
      qe_record_error(st.status, QE_ERR_DEVICE_FAULT, u);
      mbar_arrive_expect_tx(bar, 0);
      return;
    }
    const uint32_t nb = (uint32_t)(w * G * 4);
    mbar_arrive_expect_tx(bar, (uint32_t)st.slot_bytes + nb);
    bulk_g2s(dst, st.slots + ((size_t)u * st.S + id) * st.slot_bytes, (uint32_t)st.slot_bytes, bar);
    bulk_g2s(ndst, st.norms + ((size_t)u * st.norm_pitch + (size_t)win * w) * G, nb, bar);
  };

  // online softmax state of head g8 (lanes g8 >= G carry padding rows): running max (log2
  // domain), sum of weights, and the current window's sums of weights and weighted norms
  float mh = -1e30f, lh = 0.f, lwh = 0.f, nwh = 0.f;
  const float hmask = g8 < G ? 1.f : 0.f;
  // O^T accumulators: oacc[m] holds rows (head-dim elements) 16m + g8 (c0, c1) and 16m + 8 + g8
  // (c2, c3), columns (heads) 2 t4 and 2 t4 + 1. zacc: the INT2 zero-point part, rows = groups.
  float oacc[G8][4];
#pragma unroll
  for (int m = 0; m < G8; ++m) oacc[m][0] = oacc[m][1] = oacc[m][2] = oacc[m][3] = 0.f;
  float zacc[4] = {0.f, 0.f, 0.f, 0.f};

  // Softmax bookkeeping of one 16-token task: s holds head g8's log2-domain scores of tokens
  // 2t4, 2t4+1, 8+2t4, 9+2t4 (-inf where absent); p receives their weights 2^(s - max). The
  // running max starts at a finite -1e30 so that 2^(-inf - m) = 0 needs no guard; one rarely
  // taken branch rescales the accumulators when the max grows by more than 2^kRescale.
  auto softmax = [&](const float (&s)[4], float (&p)[4], const float* nrm) {
    float mx = fmaxf(fmaxf(s[0], s[1]), fmaxf(s[2], s[3]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const bool grow = mx > mh + kRescale;
    if (__any_sync(0xffffffffu, grow)) {
      const float mn = grow ? mx : mh;
      const float f = ex2(mh - mn);
      lh *= f;
      lwh *= f;
      nwh *= f;
      mh = mn;
      // O^T columns 2 t4, 2 t4 + 1 belong to the heads of lanes 8 t4 and 8 t4 + 4
      const float fa = __shfl_sync(0xffffffffu, f, 8 * t4);
      const float fb = __shfl_sync(0xffffffffu, f, 8 * t4 + 4);
#pragma unroll
      for (int m = 0; m < G8; ++m) {
        oacc[m][0] *= fa;
        oacc[m][1] *= fb;
        oacc[m][2] *= fa;
        oacc[m][3] *= fb;
      }
      zacc[0] *= fa;
      zacc[1] *= fb;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) p[i] = hmask * ex2(s[i] - mh);
    const float psum = (p[0] + p[1]) + (p[2] + p[3]);
    lh += psum;
    lwh += psum;
    if (nrm != nullptr && g8 < G) {
      nwh = fmaf(p[0], nrm[(2 * t4) * G + g8], nwh);
      nwh = fmaf(p[1], nrm[(2 * t4 + 1) * G + g8], nwh);
      nwh = fmaf(p[2], nrm[(8 + 2 * t4) * G + g8], nwh);
      nwh = fmaf(p[3], nrm[(9 + 2 * t4) * G + g8], nwh);
    }
  };
  // end of a window: its partial (max, sum p, sum p n) per head into the window's slot
  auto window_end = [&](int li) {
    float l2 = lwh + __shfl_xor_sync(0xffffffffu, lwh, 1);
    l2 += __shfl_xor_sync(0xffffffffu, l2, 2);
    float n2 = nwh + __shfl_xor_sync(0xffffffffu, nwh, 1);
    n2 += __shfl_xor_sync(0xffffffffu, n2, 2);
    if (t4 == 0 && g8 < G) {
      float* wp = a.win_part + (ub + li) * win_part_floats(D, G) + g8;
      wp[0] = mh;
      wp[G] = l2;
      wp[2 * G] = n2;
    }
    lwh = 0.f;
    nwh = 0.f;
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

  // q fragments (A operand, cache dtype): head g8's elements 16m + 2t4, +1 and 16m + 8 + 2t4, +1
  uint32_t qa[G8][2];
  {
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
        reinterpret_cast<const T*>(a.q) + ((size_t)b * st.Hq + (size_t)kvh * G + (g8 < G ? g8 : 0)) * D);
#pragma unroll
    for (int m = 0; m < G8; ++m) {
      qa[m][0] = g8 < G ? qrow[m * 8 + t4] : 0u;
      qa[m][1] = g8 < G ? qrow[m * 8 + 4 + t4] : 0u;
    }
  }

  // ---- phase 1: full-precision windows, then the tail, from swizzled TMA pages ----
  while (o < n_own && kind_of(jmap(o)) != 1) {
    if (io < n_own) {
      issue(io, ipg, issued % kNST);
      advance(io, ipg);
      ++issued;
    }
    const int s = k % kNST;
    ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[s], (k / kNST) & 1, st.status, 1000 + u));
    if (!ok) break;
    uint8_t* stage = ring + s * STAGE;
    const int j = jmap(o);
    const bool tail = kind_of(j) == 2;
    const int valid = tail ? min(QE_PAGE, a.tail_len - pg * QE_PAGE) : QE_PAGE;
    if (valid < QE_PAGE) {
      // rows past the tail's last token hold stale data: zero their V rows (weight 0 must not
      // meet a NaN) and mask their scores below
      for (int i = lane; i < (QE_PAGE - valid) * (D / 64) * 8; i += 32) {
        const int row = valid + i / ((D / 64) * 8), rest = i % ((D / 64) * 8);
        *reinterpret_cast<uint4*>(stage + ((D / 64) + rest / 8) * 2048 + row * 128 + (rest % 8) * 16) =
            make_uint4(0u, 0u, 0u, 0u);
      }
      __syncwarp();
    }
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
    float sc[4] = {c0[0] * sl, c0[1] * sl, c1[0] * sl, c1[1] * sl};
    if (tail) {
      const int tk[4] = {2 * t4, 2 * t4 + 1, 8 + 2 * t4, 9 + 2 * t4};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (tk[i] >= valid) sc[i] = -INFINITY;
        else if (g8 < G) a.tail_s[((size_t)u * w + pg * QE_PAGE + tk[i]) * G + g8] = sc[i];
      }
    }
    float p[4];
    softmax(sc, p, tail ? nullptr : reinterpret_cast<const float*>(nring + s * NSB));
    uint32_t ph0, pl0, ph1, pl1;
    MmaOp<T>::split(p[0], p[1], ph0, pl0);
    MmaOp<T>::split(p[2], p[3], ph1, pl1);
#pragma unroll
    for (int m = 0; m < G8; ++m) {
      uint32_t va[4];
      ldsm_x4_t(va, stage + swz<D>(1, ((lane >> 4) << 3) + (lane & 7), m * 16 + ((lane >> 3) & 1) * 8));
      MmaOp<T>::run(oacc[m], va[0], va[1], va[2], va[3], ph0, ph1);
      MmaOp<T>::run(oacc[m], va[0], va[1], va[2], va[3], pl0, pl1);
    }
    __syncwarp();
    if (tail) {
      // the tail's mass is formed at the end from its token scores; its sums belong to no slot
      lwh = 0.f;
      nwh = 0.f;
    } else if (pg + 1 >= ppw) {
      window_end(list_idx(j));
    }
    advance(o, pg);
    ++k;
  }

  // ---- phase 2: INT2 ledger entries ----
  // From here on the accumulators hold O^T * 2^-24 in rows g8 and O^T * 2^-20 in rows 8 + g8
  // (the scale of the subnormal code operands); the zero-point part stays unscaled in zacc.
#pragma unroll
  for (int m = 0; m < G8; ++m) {
    oacc[m][0] *= 0x1p-24f;
    oacc[m][1] *= 0x1p-24f;
    oacc[m][2] *= 0x1p-20f;
    oacc[m][3] *= 0x1p-20f;
  }
  if (ok && o < n_own) {
    // q as fp16 with the elements 8 + 2t4, 9 + 2t4 of each group quartered (their codes carry
    // 4x), and head g8's sum of q over groups 2t4, 2t4 + 1 in the log2 domain, split hi + lo
    uint32_t qh[G8][2];
    float qs[G8];
#pragma unroll
    for (int m = 0; m < G8; ++m) {
      const float x0 = Elem<T>::lo(qa[m][0]), x1 = Elem<T>::hi(qa[m][0]);
      const float x2 = Elem<T>::lo(qa[m][1]), x3 = Elem<T>::hi(qa[m][1]);
      qh[m][0] = pack_h2(x0, x1);
      qh[m][1] = pack_h2(0.25f * x2, 0.25f * x3);
      float t = (x0 + x1) + (x2 + x3);
      t += __shfl_xor_sync(0xffffffffu, t, 1);
      t += __shfl_xor_sync(0xffffffffu, t, 2);
      qs[m] = t * sl;
    }
    float qg0 = 0.f, qg1 = 0.f;
#pragma unroll
    for (int m = 0; m < G8; ++m) {
      if (m == 2 * t4) qg0 = qs[m];
      if (m == 2 * t4 + 1) qg1 = qs[m];
    }
    const uint32_t qgh = pack_h2(qg0, qg1);
    const uint32_t qgl = pack_h2(qg0 - h_lo(qgh), qg1 - h_hi(qgh));
    // staged scale factors: K scores of tokens 0..7 carry 2^-24, of tokens 8..15 16 * 2^-24;
    // V rows 8..15 of the block carry 4x in their codes, so their P * s is quartered
    const int stk = lane & 15, kvsel = lane >> 4;
    const float sfac = kvsel == 0 ? (stk < 8 ? 0x1p24f * sl : 0x1p20f * sl) : (stk < 8 ? 1.f : 0.25f);
    float* sdst = sst + kvsel * 4 * SROW + ((stk & 7) >> 1) * SROW + ((stk & 1) + 2 * (stk >> 3));
    const float* sk = sst + t4 * SROW;
    const float* sv = sst + 4 * SROW + t4 * SROW;

    while (o < n_own) {
      if (io < n_own) {
        issue(io, ipg, issued % kNST);
        advance(io, ipg);
        ++issued;
      }
      const int s = k % kNST;
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[s], (k / kNST) & 1, st.status, 1000 + u));
      if (!ok) break;
      const uint8_t* stage = ring + s * STAGE;
      const float* nrm = reinterpret_cast<const float*>(nring + s * NSB);
      for (int bk = 0; bk < w / 16; ++bk) {
        const uint8_t* blk = stage + bk * BL::BYTES;
        {  // stage this block's scales: lanes 0-15 the K scales of token lane, 16-31 the V scales
          const __half* srow = reinterpret_cast<const __half*>(blk + (kvsel ? BL::VS : BL::KS)) + stk * G8;
#pragma unroll
          for (int m = 0; m < G8; ++m) sdst[m * 4] = __half2float(srow[m]) * sfac;
        }
        __syncwarp();
        // ---- K side: scores of tokens 2t4, 2t4+1 (tile A) and 8+2t4, 9+2t4 (tile B) ----
        float sc[4];
        {
          const uint32_t zA = 2 * t4 < G8 ? *reinterpret_cast<const uint32_t*>(blk + BL::KZ + (g8 * G8 + 2 * t4) * 2) : 0u;
          const uint32_t zB =
              2 * t4 < G8 ? *reinterpret_cast<const uint32_t*>(blk + BL::KZ + ((8 + g8) * G8 + 2 * t4) * 2) : 0u;
          float za[4] = {0.f, 0.f, 0.f, 0.f}, zb[4] = {0.f, 0.f, 0.f, 0.f};
          mma_h8(za, qgh, 0u, zA);
          mma_h8(za, qgl, 0u, zA);
          mma_h8(zb, qgh, 0u, zB);
          mma_h8(zb, qgl, 0u, zB);
          sc[0] = za[0];
          sc[1] = za[1];
          sc[2] = zb[0];
          sc[3] = zb[1];
        }
        uint32_t kw[WPL];
        if constexpr (WPL == 4) {
          const uint4 v4 = *reinterpret_cast<const uint4*>(blk + BL::KC + lane * 16);
          kw[0] = v4.x; kw[1] = v4.y; kw[2] = v4.z; kw[3] = v4.w;
        } else {
          const uint2 v2 = *reinterpret_cast<const uint2*>(blk + BL::KC + lane * 8);
          kw[0] = v2.x; kw[1] = v2.y;
        }
#pragma unroll
        for (int jj = 0; jj < WPL; ++jj) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int m = 2 * jj + e;
            const uint32_t x = e ? (kw[jj] >> 8) : kw[jj];
            float cA[4] = {0.f, 0.f, 0.f, 0.f}, cB[4] = {0.f, 0.f, 0.f, 0.f};
            mma_h16(cA, qh[m][0], 0u, qh[m][1], 0u, code_reg<0>(x), code_reg<1>(x));
            mma_h16(cB, qh[m][0], 0u, qh[m][1], 0u, code_reg<2>(x), code_reg<3>(x));
            const float4 s4 = *reinterpret_cast<const float4*>(sk + m * 4);
            const float2 ra = ffma2(make_float2(s4.x, s4.y), make_float2(cA[0], cA[1]), make_float2(sc[0], sc[1]));
            const float2 rb = ffma2(make_float2(s4.z, s4.w), make_float2(cB[0], cB[1]), make_float2(sc[2], sc[3]));
            sc[0] = ra.x;
            sc[1] = ra.y;
            sc[2] = rb.x;
            sc[3] = rb.y;
          }
        }
        float p[4];
        softmax(sc, p, nrm + bk * 16 * G);
        // ---- V side ----
        {
          uint32_t ph0, pl0, ph1, pl1;
          MmaOp<__half>::split(p[0], p[1], ph0, pl0);
          MmaOp<__half>::split(p[2], p[3], ph1, pl1);
          const uint32_t za0 = g8 < G8 ? *reinterpret_cast<const uint32_t*>(blk + BL::VZ + (g8 * 16 + 2 * t4) * 2) : 0u;
          const uint32_t za2 =
              g8 < G8 ? *reinterpret_cast<const uint32_t*>(blk + BL::VZ + (g8 * 16 + 8 + 2 * t4) * 2) : 0u;
          mma_h16(zacc, za0, 0u, za2, 0u, ph0, ph1);
          mma_h16(zacc, za0, 0u, za2, 0u, pl0, pl1);
        }
        uint32_t vw[WPL];
        if constexpr (WPL == 4) {
          const uint4 v4 = *reinterpret_cast<const uint4*>(blk + BL::VC + lane * 16);
          vw[0] = v4.x; vw[1] = v4.y; vw[2] = v4.z; vw[3] = v4.w;
        } else {
          const uint2 v2 = *reinterpret_cast<const uint2*>(blk + BL::VC + lane * 8);
          vw[0] = v2.x; vw[1] = v2.y;
        }
#pragma unroll
        for (int jj = 0; jj < WPL; ++jj) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int m = 2 * jj + e;
            const uint32_t x = e ? (vw[jj] >> 8) : vw[jj];
            const float4 s4 = *reinterpret_cast<const float4*>(sv + m * 4);
            const uint32_t b0 = pack_h2(p[0] * s4.x, p[1] * s4.y);
            const uint32_t b1 = pack_h2(p[2] * s4.z, p[3] * s4.w);
            mma_h16(oacc[m], code_reg<0>(x), code_reg<2>(x), code_reg<1>(x), code_reg<3>(x), b0, b1);
          }
        }
        __syncwarp();  // the next block restages the scales
      }
      window_end(list_idx(jmap(o)));
      advance(o, pg);
      ++k;
    }
  }
  if (!ok) {  // drain copies still in flight if a wait gave up
    for (; k < issued; ++k) mbar_wait_bounded(&bars[k % kNST], (k / kNST) & 1, st.status, 2000 + u);
  }
  // back to O^T: undo the code scales and add the zero-point part of each element's group
#pragma unroll
  for (int m = 0; m < G8; ++m) {
    const float z0 = __shfl_sync(0xffffffffu, zacc[0], 4 * m + t4);
    const float z1 = __shfl_sync(0xffffffffu, zacc[1], 4 * m + t4);
    oacc[m][0] = fmaf(oacc[m][0], 0x1p24f, z0);
    oacc[m][1] = fmaf(oacc[m][1], 0x1p24f, z1);
    oacc[m][2] = fmaf(oacc[m][2], 0x1p20f, z0);
    oacc[m][3] = fmaf(oacc[m][3], 0x1p20f, z1);
  }
  lh += __shfl_xor_sync(0xffffffffu, lh, 1);
  lh += __shfl_xor_sync(0xffffffffu, lh, 2);

  // ---- merge the warps into the CTA's partial ----
  const bool cta_ok = __syncthreads_and(ok ? 1 : 0) != 0;  // also: every warp is done with its ring
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
  float* okv = red + kNW;                             // [1] this CTA finished every wait
  if (t4 == 0 && g8 < G) {
    mw[warp * G + g8] = mh;
    lwv[warp * G + g8] = lh;
  }
#pragma unroll
  for (int m = 0; m < G8; ++m) {
    float* a0 = aw + (size_t)warp * G * D;
    if (2 * t4 < G) {
      a0[(2 * t4) * D + m * 16 + g8] = oacc[m][0];
      a0[(2 * t4) * D + m * 16 + 8 + g8] = oacc[m][2];
    }
    if (2 * t4 + 1 < G) {
      a0[(2 * t4 + 1) * D + m * 16 + g8] = oacc[m][1];
      a0[(2 * t4 + 1) * D + m * 16 + 8 + g8] = oacc[m][3];
    }
  }
  if (threadIdx.x == 0) okv[0] = cta_ok ? 1.f : 0.f;
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
  // every CTA of the unit must have finished its waits: a CTA that gave up holds partials of
  // a part of its windows, and window partials it never wrote may be stale
  float all_ok = 1.f;
  for (int r = 0; r < S; ++r) all_ok = fminf(all_ok, ld_cluster(okv, (uint32_t)r));
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
  if (all_ok > 0.f) {
    // exact attention mass and perturbation of this step for the windows this CTA streamed
    for (int jj = threadIdx.x; jj < nF + nQ; jj += blockDim.x) {
      const int vj = jj < nF ? jj : jj + has_tail;
      const int li = list_idx(vj);
      const int win = jj < nF ? st.full_list[ub + li] : st.int2_list[ub + li - nf];
      if (win < 0 || win >= st.Wmax) continue;
      const float* wp = a.win_part + (ub + li) * win_part_floats(D, G);
      float dm = 0.f, dp = 0.f;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float f = ex2(wp[h] - lse[h]);
        dm = fmaf(wp[G + h], f, dm);
        dp = fmaf(wp[2 * G + h], f, dp);
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
  }
  cluster_sync();  // keep this CTA's partial alive until every CTA of the cluster has read it
}

template <typename T, int D, int G>
int launch_decode_t(qe_ctx* c, const void* q, float* out, cudaStream_t s, const void* k_new,
                    const void* v_new) {
  constexpr int STAGE = StageLayout<D>::BYTES;
  auto smem_for = [](int w) {
    return (size_t)1024 + (size_t)kNW * kNST * STAGE + kNW * kNST * 8 + (size_t)kNW * aux_bytes<D>(w, G);
  };
  static_assert((size_t)(kNW * G * (D + 2) + 2 * QE_MAX_G + G * D + 3 * QE_MAX_SPLITS_CLUSTER * QE_MAX_G +
                         2 * QE_MAX_G + kNW + 1) * 4 <= (size_t)kNW * kNST * STAGE,
                "merge area");
  auto kern = decode_kernel<T, D, G>;
  // One-time set-up per instantiation and device (kept out of the per-step path and of graph
  // capture): clusters[wi][S] = how many clusters of S CTAs can be resident at once with the
  // shared memory of window size 16 << wi.
  static QeOnce once;
  static int clusters_of[QE_MAX_DEVICES][3][QE_MAX_SPLITS_CLUSTER + 1];
  int dev = 0;
  const int se = qe_once_per_device(once, &dev, [&](int d) {
    QE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_for(64)));
    QE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
    for (int wi = 0; wi < 3; ++wi)
      for (int S = 1; S <= QE_MAX_SPLITS_CLUSTER; ++S) {
        cudaLaunchConfig_t qc = {};
        cudaLaunchAttribute qa[1];
        qa[0].id = cudaLaunchAttributeClusterDimension;
        qa[0].val.clusterDim.x = S;
        qa[0].val.clusterDim.y = 1;
        qa[0].val.clusterDim.z = 1;
        qc.gridDim = dim3(S);
        qc.blockDim = dim3(kNW * 32);
        qc.dynamicSmemBytes = smem_for(16 << wi);
        qc.attrs = qa;
        qc.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &qc) != cudaSuccess) {
          (void)cudaGetLastError();
          n = 0;
        }
        clusters_of[d][wi][S] = n;
      }
    return QE_OK;
  });
  if (se) return se;
  const int wi = c->cfg.window == 16 ? 0 : (c->cfg.window == 32 ? 1 : 2);
  const size_t smem = smem_for(c->cfg.window);
  const int* clusters = clusters_of[dev][wi];
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
