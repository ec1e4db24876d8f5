// Split-K GQA decode attention over the full-precision and INT2 tiers, fused with the
// cumulative window scores and (optionally) the append of the step's token.
//
// "Resumo Técnico: QEvict" - Mecanismos Principais: window-level routing driven by
// attention accumulated over time (Pontuação Cumulativa); the recoverable INT2 tier stays
// readable by attention (Metodologia 2); GQA decode path (Implementação).
// "Resumo Técnico: CriticalKV" - Etapa 2: the perturbation score A_i * ||V_i W_O||_1.
//
// Work split. Per unit u = (b, g) the live windows are [tail | full windows | INT2 windows].
// The unit's S CTAs form one thread-block cluster; CTA s takes the s-th S-th of the full
// windows and of the INT2 windows (the tail counts as one more INT2 window of the last CTA),
// so every SM streams the same mix of bandwidth-heavy full pages and compact INT2 entries.
// Inside a CTA warp w takes windows w, w + kNW, ...; even warps walk them in list order, odd
// warps start with their INT2 windows, so some warps of an SM stream full pages while others
// do the INT2 arithmetic. A warp streams its windows as tasks of 16*D*2 bytes through its own
// ring of shared-memory stages (completion on an mbarrier per stage): the K rows of a full or
// tail page, its V rows (128-byte-swizzled TMA boxes from a tensor map over the page pool), or
// a chunk of up to 32 tokens of an INT2 ledger entry (one 1-D bulk copy), each with its
// tokens' projected-value norms.
//
// Every tier runs on the warp-level tensor cores (mma.sync, f32 accumulate) with the tokens
// as MMA rows: S^T = K Q^T takes 16 tokens as the A operand and the G <= 8 query heads of the
// group as the B columns (no padding rows), so lane (r, t) holds the scores of tokens r and
// 8 + r for heads 2t and 2t + 1; P^T goes through movmatrix into the B fragment of
// O^T = V^T P^T. A decode step has G <= 8 query heads per KV head; a tcgen05 tile (M >= 64)
// would be mostly padding and its TMEM round trip buys nothing on a path that HBM bounds, so
// the decode stays on mma.sync.
//
// Full-precision pages: S^T from ldmatrix K tiles (two independent accumulator chains), P split
// into two 16-bit parts of the cache dtype (hi + residual) so O keeps float32 accuracy, V^T by
// ldmatrix.trans.
//
// INT2 blocks (16 tokens, layout in int2_block.cuh): a K or V value is c*s + z with a 2-bit code
// c and an fp16 scale s and zero z per 16-element group. The codes enter the MMA exactly as
// fp16 subnormals c * 4^i * 2^-24 (one mask per register); per group g
//   S^T += s_g * (C_g Q_g^T)  (one MMA per 16 tokens, then an f32x2 FMA by the token scales),
//   S^T += Z (sum of q over each group)  (m16n8k8 MMAs, q sums split hi + lo),
//   O_g^T += C_g^T (P^T s_g)  (two MMAs per group: the weight-times-scale operand carried as
//                              an exact fp16 sum hi + lo),
//   O^T += Z^T P^T  (one MMA per 16 tokens and 16-bit part of P).
// The token scales reach the lanes that need them as float32 through one more MMA per group
// (the group's scales times a 0/1 selection matrix), so no conversion or staging is needed.
// The powers 4^i and 2^-24 are folded into q, the selection matrix and the accumulator, which
// holds O^T scaled by 2^-24 (rows 0-7) and 2^-20 (rows 8-15) while INT2 chunks stream.
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
#define QE_DECODE_NW 3
#endif
#ifndef QE_DECODE_MINB
#define QE_DECODE_MINB 4
#endif
constexpr int kNW = QE_DECODE_NW;    // warps per CTA
#define QE_MAX_SPLITS_CLUSTER 16     // CTAs per unit (one cluster, non-portable size)
constexpr float kRescale = 8.f;      // rescale the accumulators when the max grows by > 2^8

// stages per warp (fewer for wide groups, whose norm slots are larger)
__host__ __device__ constexpr int nst_of(int G) { return G <= 4 ? 4 : 3; }
// bytes of one stage: the K (or V) rows of a page, or an INT2 chunk of up to 32 tokens
template <int D>
__host__ __device__ constexpr int stage_bytes() { return (QE_PAGE * D * 2 + 1023) / 1024 * 1024; }
// bytes of one norm slot: the norms of up to 32 tokens
__host__ __device__ constexpr int norm_slot_bytes(int G) { return 32 * G * 4; }
template <int D, int G>
__host__ __device__ constexpr size_t decode_smem_bytes() {
  return 1024 + (size_t)kNW * nst_of(G) * (stage_bytes<D>() + norm_slot_bytes(G) + 8);
}

struct DecodeArgs {
  DevState st;
  const void* q;     // [B][Hq][D]
  float* out;        // [B][Hq][D]
  float* win_part;   // [U][Wmax][3 G]: {max, sum p, sum p n} per head
  float* tail_s;     // [U][window][G]
  int splits;        // CTAs per unit = cluster size
  int nf, nq;        // full / INT2 windows of every unit, or -1: read them from the device state
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
// memory of CTA `rank` of the cluster at the address of a local shared variable (issued after
// a cluster barrier; the barrier orders it)
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_cluster(const float* local, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(local)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a));
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
  asm(
      "mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

// fp16 pair product, round to nearest
__device__ __forceinline__ uint32_t __hmul2_u32(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
// fp16 pair a * b + c, one rounding
__device__ __forceinline__ uint32_t __hfma2_u32(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}
// The weight-times-scale product w s of a pair, where w = wh + wl (fp16 high and low parts), as
// an unevaluated fp16 sum hi + lo: hi = fl(wh s); lo = fl(fl(wh s - hi) + wl s), where wh s - hi
// (the rounding error of a product) is exact in fp16 barring underflow, so hi + lo carries
// w s to about 2^-20 relative, where the single product wh s (dropping wl) is off by up to 2^-10.
// The error term is one fused multiply-add with a negated addend (the negation folds into it).
__device__ __forceinline__ void ws_split(uint32_t wh, uint32_t wl, uint32_t sc, uint32_t& hi, uint32_t& lo) {
  hi = __hmul2_u32(wh, sc);
  uint32_t e;
  asm("{\n\t.reg .b32 n;\n\tneg.f16x2 n, %2;\n\tfma.rn.f16x2 %0, %1, %3, n;\n\t}"
      : "=r"(e)
      : "r"(wh), "r"(hi), "r"(sc));
  lo = __hfma2_u32(wl, sc, e);
}

// Register i (0..3) of a packed code word: the codes at bits [2i, 2i+1] of each 16-bit half as
// the fp16 subnormals c * 4^i * 2^-24.
template <int I>
__device__ __forceinline__ uint32_t code_reg(uint32_t x) {
  return x & (0x00030003u << (2 * I));
}

template <typename T, int D, int G, int W>
__global__ void __launch_bounds__(kNW * 32, QE_DECODE_MINB)
    decode_kernel(const __grid_constant__ CUtensorMap tmP, DecodeArgs a) {
  using BL = Int2Block<D>;
  constexpr int G8 = BL::G8, WPL = BL::WPL;
  constexpr int NST = nst_of(G);
  constexpr int PPW = W / QE_PAGE;               // pages per window
  constexpr int BPC = W >= 32 ? 2 : 1;           // INT2 blocks per chunk task
  constexpr int CPW = W / (QE_PAGE * BPC);       // INT2 chunk tasks per window
  constexpr int HALF = QE_PAGE * D * 2;          // bytes of a page's K (or V) rows
  constexpr int STAGE = stage_bytes<D>();
  constexpr int NSB = norm_slot_bytes(G);
  constexpr int NB = D / 64;                     // TMA boxes per K or V half
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const DevState& st = a.st;
  if (threadIdx.x == 0) asm volatile("prefetch.tensormap [%0];" ::"l"(&tmP) : "memory");
  const int u = blockIdx.x / a.splits, split = blockIdx.x % a.splits;
  const int b = u / st.Hkv, kvh = u % st.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  const size_t ub = (size_t)u * st.Wmax;
  const float sl = a.scale_log2;

  // this split's share of each tier
  const int nf = a.nf >= 0 ? a.nf : st.stacks[u * 4 + 2];
  const int nq = a.nq >= 0 ? a.nq : st.stacks[u * 4 + 3];
  const int f0 = (int)((long long)nf * split / a.splits), f1 = (int)((long long)nf * (split + 1) / a.splits);
  // the last split also streams the tail window (and appends the new token): it counts as one
  // INT2 window of that split's share
  const int nqv = a.tail_len > 0 ? nq + 1 : nq;
  const int q0 = (int)((long long)nqv * split / a.splits);
  const int q1 = min(nq, (int)((long long)nqv * (split + 1) / a.splits));
  const int has_tail = (a.tail_len > 0 && split == a.splits - 1) ? 1 : 0;
  const int nF = f1 - f0, nQ = q1 - q0, nJ = nF + has_tail + nQ;
  const int tail_pages = (a.tail_len + QE_PAGE - 1) / QE_PAGE;

  uint8_t* ring = smem + warp * NST * STAGE;
  uint8_t* nring = smem + kNW * NST * STAGE + warp * NST * NSB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kNW * NST * (STAGE + NSB)) + warp * NST;
  if (lane == 0) {
    for (int s = 0; s < NST; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();

  // Windows of this split in the order [tail (when present) | full | INT2]; warp w takes
  // windows j = w + kNW * o' (each window a run of tasks: full and tail windows K, V of every
  // page; INT2 windows their chunks). Even warps walk their windows in that order, odd warps
  // start with their INT2 windows (o' = o + their number of tail and full windows, mod n_own),
  // so that at any time some warps of the SM stream full-precision pages while others do the
  // INT2 tier's dequantising arithmetic, and warp 0 starts with the tail and its append.
  auto kind_of = [&](int j) { return j < has_tail ? 2 : (j < has_tail + nF ? 0 : 1); };  // full 0, INT2 1, tail 2
  // position in the full list, or nf + position in the INT2 list (the window-partial slot)
  auto list_idx = [&](int j) {
    const int v = j - has_tail;
    return v < nF ? f0 + v : nf + q0 + (v - nF);
  };
  auto n_sub = [&](int kind) { return kind == 0 ? 2 * PPW : (kind == 1 ? CPW : 2 * tail_pages); };
  const int n_own = nJ > warp ? (nJ - warp + kNW - 1) / kNW : 0;
  const int n_ft = has_tail + nF;
  const int rot = (warp & 1) && n_ft > warp ? (n_ft - warp + kNW - 1) / kNW : 0;
  auto j_of = [&](int o) {
    int oo = o + rot;
    if (oo >= n_own) oo -= n_own;
    return warp + kNW * oo;
  };
  struct Cursor {
    int o, i;  // window ordinal of this warp, task within the window
  };
  auto cur_kind = [&](const Cursor& c) { return kind_of(j_of(c.o)); };
  auto cur_set = [&](Cursor& c, int o) {
    c.o = o;
    c.i = 0;
  };
  // next task; a new window when the current one is done
  auto cur_next = [&](Cursor& c) {
    if (++c.i >= n_sub(cur_kind(c))) {
      c.i = 0;
      ++c.o;
    }
  };
  auto cur_list_idx = [&](const Cursor& c) { return list_idx(j_of(c.o)); };
  // Index prefetch: lane l holds the window id and the page ids (full, tail) or the ledger
  // slot (INT2) of this warp's window of ordinal rb + l, so issuing a copy never waits on a
  // dependent global load. Reloaded every 32 windows.
  int e_win = -1, e_id[PPW], rb = -32;
  auto load_ids = [&](int base) {
    rb = base;
    const int jj = base + lane < n_own ? j_of(base + lane) : nJ;
    e_win = -1;
#pragma unroll
    for (int p = 0; p < PPW; ++p) e_id[p] = -1;
    if (jj < nJ) {
      const int kd = kind_of(jj);
      const int li = kd == 2 ? 0 : list_idx(jj);
      const int win = kd == 0 ? st.full_list[ub + li] : (kd == 1 ? st.int2_list[ub + li - nf] : a.tail_win);
      if (win >= 0 && win < st.Wmax) {
        e_win = win;
        if (kd == 1) {
          e_id[0] = st.win_slot[ub + win];
        } else {
#pragma unroll
          for (int p = 0; p < PPW; ++p) e_id[p] = st.win_pages[(ub + win) * PPW + p];
        }
      }
    }
  };
  // fused append: page of the step's token (written by this warp just before the tail's copies)
  int app_pg = -1, app_page = -1;
  // issue the copies of task (window ordinal r, task i) into stage s (all lanes call)
  auto issue = [&](const Cursor& c, int s) {
    const int r = c.o, i = c.i, k = cur_kind(c);
    if (r - rb >= 32) load_ids(r - r % 32);
    const int src = r - rb;
    const int pg = k == 1 ? 0 : (i >> 1);
    int sel = e_id[0];
#pragma unroll
    for (int p = 1; p < PPW; ++p)
      if (pg == p) sel = e_id[p];
    const int win = __shfl_sync(0xffffffffu, e_win, src);
    int id = __shfl_sync(0xffffffffu, sel, src);
    if (k == 2 && i == 0 && a.k_new != nullptr) {
      // the step's token goes into the tail window before its pages are copied
      app_page = append_token_warp(st, u, a.append_pos, a.k_new, a.v_new, a.tailV);
      app_pg = (a.append_pos % W) / QE_PAGE;
    }
    if (k == 2 && pg == app_pg) id = app_page;
    fence_proxy_async_smem();
    if (lane != 0) return;
    uint8_t* dst = ring + s * STAGE;
    uint64_t* bar = &bars[s];
    if (k != 1) {
      // the K (i even) or V (i odd) rows of a full-precision or tail page: D/64 swizzled TMA
      // boxes; a full page's K task also brings the page's norms
      if (win < 0 || id < 0 || id >= st.P) {
        qe_record_error(st.status, QE_ERR_DEVICE_FAULT, u);
        mbar_arrive_expect_tx(bar, 0);
        return;
      }
      const bool nrm = k == 0 && (i & 1) == 0;
      const uint32_t nb = nrm ? QE_PAGE * G * 4 : 0;
      mbar_arrive_expect_tx(bar, HALF + nb);
      const int row0 = (u * st.P + id) * 2 * QE_PAGE + (i & 1) * QE_PAGE;
#pragma unroll
      for (int xb = 0; xb < NB; ++xb) tc::tma_load_2d(dst + xb * 2048, &tmP, xb * 64, row0, bar);
      if (nrm)
        bulk_g2s(nring + s * NSB, st.norms + ((size_t)u * st.norm_pitch + (size_t)win * W + pg * QE_PAGE) * G, nb,
                 bar);
      return;
    }
    if (win < 0 || id < 0 || id >= st.S) {
      qe_record_error(st.status, QE_ERR_DEVICE_FAULT, u);
      mbar_arrive_expect_tx(bar, 0);
      return;
    }
    constexpr uint32_t cb = BPC * BL::BYTES, nb = BPC * QE_PAGE * G * 4;
    mbar_arrive_expect_tx(bar, cb + nb);
    bulk_g2s(dst, st.slots + ((size_t)u * st.S + id) * st.slot_bytes + (size_t)i * cb, cb, bar);
    bulk_g2s(nring + s * NSB, st.norms + ((size_t)u * st.norm_pitch + (size_t)win * W + i * BPC * QE_PAGE) * G, nb,
             bar);
  };

  // Scores come out of S^T = K Q^T with tokens as MMA rows and heads as columns: lane (g8, t4)
  // holds the scores of tokens g8 and 8 + g8 for heads 2 t4 and 2 t4 + 1 (slots 0, 1 and 2, 3
  // of every 16-token block). Each lane keeps the online-softmax state of its two heads: running
  // max (log2 domain), sum of weights, and the current window's sums of weights and weighted
  // norms (per-lane partial sums over its tokens, reduced over the eight token rows when used).
  const int h0 = 2 * t4, h1 = 2 * t4 + 1;
  const float hm0 = h0 < G ? 1.f : 0.f, hm1 = h1 < G ? 1.f : 0.f;
  float m0 = -1e30f, m1 = -1e30f, l0 = 0.f, l1 = 0.f, lw0 = 0.f, lw1 = 0.f, nw0 = 0.f, nw1 = 0.f;
  // O^T accumulators: oacc[m] holds rows (head-dim elements) 16m + g8 (c0, c1) and 16m + 8 + g8
  // (c2, c3), columns (heads) h0 and h1. zacc: the INT2 zero-point part, rows = groups.
  float oacc[G8][4];
#pragma unroll
  for (int m = 0; m < G8; ++m) oacc[m][0] = oacc[m][1] = oacc[m][2] = oacc[m][3] = 0.f;
  float zacc[4] = {0.f, 0.f, 0.f, 0.f};

  // Softmax bookkeeping of N/4 16-token blocks: s holds this lane's log2-domain scores (slots
  // 4b + {0: token g8 head h0, 1: token g8 head h1, 2: token 8+g8 head h0, 3: token 8+g8 head h1},
  // -inf where absent); p receives the weights 2^(s - max). The running max starts at a finite
  // -1e30 so that 2^(-inf - m) = 0 needs no guard; one rarely taken branch rescales the
  // accumulators when a head's max grows by more than 2^kRescale. nrm (may be null): the blocks'
  // norms, [16 N/4 tokens][G].
  auto softmax = [&](auto& s, auto& p, const float* nrm) {
    constexpr int N = sizeof(s) / sizeof(float);
    float x0 = s[0], x1 = s[1];
#pragma unroll
    for (int i = 2; i < N; i += 2) {
      x0 = fmaxf(x0, s[i]);
      x1 = fmaxf(x1, s[i + 1]);
    }
    // a head's max grows past m + kRescale exactly when one of its lanes sees such a score; only
    // then is the max reduced over the eight token rows
    const bool grow = x0 > m0 + kRescale || x1 > m1 + kRescale;
    if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, o));
        x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, o));
      }
      const float n0 = x0 > m0 + kRescale ? x0 : m0, n1 = x1 > m1 + kRescale ? x1 : m1;
      const float f0 = ex2(m0 - n0), f1 = ex2(m1 - n1);
      l0 *= f0;
      lw0 *= f0;
      nw0 *= f0;
      l1 *= f1;
      lw1 *= f1;
      nw1 *= f1;
      m0 = n0;
      m1 = n1;
#pragma unroll
      for (int m = 0; m < G8; ++m) {
        oacc[m][0] *= f0;
        oacc[m][1] *= f1;
        oacc[m][2] *= f0;
        oacc[m][3] *= f1;
      }
      zacc[0] *= f0;
      zacc[1] *= f1;
    }
    float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
    for (int i = 0; i < N; i += 2) {
      p[i] = hm0 * ex2(s[i] - m0);
      p[i + 1] = hm1 * ex2(s[i + 1] - m1);
      ps0 += p[i];
      ps1 += p[i + 1];
    }
    l0 += ps0;
    l1 += ps1;
    lw0 += ps0;
    lw1 += ps1;
    if (nrm != nullptr) {
#pragma unroll
      for (int i = 0; i < N; i += 2) {
        const int tok = 16 * (i >> 2) + g8 + 8 * ((i >> 1) & 1);
        const float* nr = nrm + tok * G;
        float a0, a1;
        if constexpr (G % 2 == 0) {
          const float2 v = *reinterpret_cast<const float2*>(nr + (h0 < G ? h0 : 0));
          a0 = v.x;
          a1 = v.y;
        } else {
          a0 = nr[h0 < G ? h0 : 0];
          a1 = nr[h1 < G ? h1 : 0];
        }
        nw0 = fmaf(p[i], a0, nw0);
        nw1 = fmaf(p[i + 1], a1, nw1);
      }
    }
  };
  // end of a window: its partial (max, sum p, sum p n) per head into the window's slot
  auto window_end = [&](int li) {
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      lw0 += __shfl_xor_sync(0xffffffffu, lw0, o);
      lw1 += __shfl_xor_sync(0xffffffffu, lw1, o);
      nw0 += __shfl_xor_sync(0xffffffffu, nw0, o);
      nw1 += __shfl_xor_sync(0xffffffffu, nw1, o);
    }
    if (g8 == 0) {
      float* wp = a.win_part + (ub + li) * win_part_floats(D, G);
      if (h0 < G) {
        wp[h0] = m0;
        wp[G + h0] = lw0;
        wp[2 * G + h0] = nw0;
      }
      if (h1 < G) {
        wp[h1] = m1;
        wp[G + h1] = lw1;
        wp[2 * G + h1] = nw1;
      }
    }
    lw0 = lw1 = nw0 = nw1 = 0.f;
  };
  // P of one 16-token block as the B fragment of O^T = V^T P^T (tokens 2t4, 2t4+1 | 8+2t4,
  // 9+2t4 of head g8): the 16-bit pairs of the score layout, transposed 8x8 by movmatrix
  auto transpose_pair = [&](uint32_t x) {
    uint32_t y;
    asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
  };

  Cursor cc, ci;  // the task being computed, the next task to copy
  cur_set(cc, 0);
  cur_set(ci, 0);
  // The first task's copies go out at once; the rest of the prologue's copies only after the
  // query operands are set up, so that at launch, when every warp of the grid asks for its
  // stages together, the first stages are not queued behind the later ones.
  int issued = 0;
  for (int s = 0; s < 1 && ci.o < n_own; ++s) {
    issue(ci, s);
    cur_next(ci);
    ++issued;
  }
  int k = 0;
  bool ok = true;
  // wait for the task computed next, after issuing the one NST - 1 ahead
  auto next_stage = [&]() -> int {
    if (ci.o < n_own) {
      issue(ci, issued % NST);
      cur_next(ci);
      ++issued;
    }
    const int s = k % NST;
    ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[s], (k / NST) & 1, st.status, 1000 + u));
    return s;
  };

  // q as the B operand of S^T = K Q^T (cache dtype): head g8's elements 16m + 2t4, +1 (qb[m][0])
  // and 16m + 8 + 2t4, +1 (qb[m][1]); zero for padding heads
  uint32_t qb[G8][2];
  {
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
        reinterpret_cast<const T*>(a.q) + ((size_t)b * st.Hq + (size_t)kvh * G + (g8 < G ? g8 : 0)) * D);
#pragma unroll
    for (int m = 0; m < G8; ++m) {
      qb[m][0] = g8 < G ? qrow[m * 8 + t4] : 0u;
      qb[m][1] = g8 < G ? qrow[m * 8 + 4 + t4] : 0u;
    }
  }

  // INT2 operands, computed once:
  // q as fp16 with the elements 8 + 2t4, 9 + 2t4 of each group quartered (their codes carry
  // 4x), and head g8's sum of q over groups 2t4, 2t4 + 1 in the log2 domain, split hi + lo
  // (the B operand of the zero-point product Z Q_g)
  uint32_t qh[G8][2];
  float qg0 = 0.f, qg1 = 0.f;
#pragma unroll
  for (int m = 0; m < G8; ++m) {
    const float x0 = Elem<T>::lo(qb[m][0]), x1 = Elem<T>::hi(qb[m][0]);
    const float x2 = Elem<T>::lo(qb[m][1]), x3 = Elem<T>::hi(qb[m][1]);
    qh[m][0] = pack_h2(x0, x1);
    qh[m][1] = pack_h2(0.25f * x2, 0.25f * x3);
    float t = (x0 + x1) + (x2 + x3);
    t += __shfl_xor_sync(0xffffffffu, t, 1);
    t += __shfl_xor_sync(0xffffffffu, t, 2);
    if (m == 2 * t4) qg0 = t * sl;
    if (m == 2 * t4 + 1) qg1 = t * sl;
  }
  const uint32_t qgh = pack_h2(qg0, qg1);
  const uint32_t qgl = pack_h2(qg0 - h_lo(qgh), qg1 - h_hi(qgh));
  // selection matrix that deals a token's K scale to both head columns: row 0 picks all
  const uint32_t sel0 = t4 == 0 ? 0x3c00u : 0u;
  const float2 fa = make_float2(0x1p24f * sl, 0x1p24f * sl), fb = make_float2(0x1p20f * sl, 0x1p20f * sl);
  constexpr uint32_t kQuarter2 = 0x34003400u;  // fp16 pair {0.25, 0.25}

  // The accumulators hold O^T while full-precision and tail pages are streamed, and O^T * 2^-24
  // in rows g8 / O^T * 2^-20 in rows 8 + g8 (the scale of the subnormal code operands) while INT2
  // chunks are; they are rescaled at every switch (the zero-point part stays unscaled in zacc).
  auto to_units = [&](bool int2) {
    const float lo = int2 ? 0x1p-24f : 0x1p24f, hi = int2 ? 0x1p-20f : 0x1p20f;
#pragma unroll
    for (int m = 0; m < G8; ++m) {
      oacc[m][0] *= lo;
      oacc[m][1] *= lo;
      oacc[m][2] *= hi;
      oacc[m][3] *= hi;
    }
  };
  for (int s = issued; s < NST - 1 && ci.o < n_own; ++s) {
    issue(ci, s);
    cur_next(ci);
    ++issued;
  }
  bool int2_units = false;
  uint32_t ph0 = 0, pl0 = 0, ph1 = 0, pl1 = 0;  // P^T of the last K task, for its V task
  int valid = QE_PAGE;
  while (cc.o < n_own) {
    const int s = next_stage();
    if (!ok) break;
    const int kd = cur_kind(cc), ti = cc.i;
    if ((kd == 1) != int2_units) {
      int2_units = kd == 1;
      to_units(int2_units);
    }
    if (kd != 1) {
      uint8_t* stage = ring + s * STAGE;
      const bool tail = kd == 2;
      if ((ti & 1) == 0) {
        // K rows: S^T = K Q^T over 16 tokens, two independent chains
        valid = tail ? min(QE_PAGE, a.tail_len - (ti >> 1) * QE_PAGE) : QE_PAGE;
        float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int m = 0; m < G8; ++m) {
          uint32_t ka[4];
          ldsm_x4(ka, stage + swz<D>(0, ((lane >> 3) & 1) * 8 + (lane & 7), m * 16 + (lane >> 4) * 8));
          if (m & 1) MmaOp<T>::run(c1, ka[0], ka[1], ka[2], ka[3], qb[m][0], qb[m][1]);
          else MmaOp<T>::run(c0, ka[0], ka[1], ka[2], ka[3], qb[m][0], qb[m][1]);
        }
        float sc[4] = {(c0[0] + c1[0]) * sl, (c0[1] + c1[1]) * sl, (c0[2] + c1[2]) * sl, (c0[3] + c1[3]) * sl};
        if (tail) {
          const int pg = ti >> 1;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int tk = g8 + 8 * (i >> 1), hh = 2 * t4 + (i & 1);
            if (tk >= valid) sc[i] = -INFINITY;
            else if (hh < G) a.tail_s[((size_t)u * W + pg * QE_PAGE + tk) * G + hh] = sc[i];
          }
        }
        float p[4];
        softmax(sc, p, tail ? nullptr : reinterpret_cast<const float*>(nring + s * NSB));
        uint32_t x0, y0, x1, y1;
        MmaOp<T>::split(p[0], p[1], x0, y0);
        MmaOp<T>::split(p[2], p[3], x1, y1);
        ph0 = transpose_pair(x0);
        pl0 = transpose_pair(y0);
        ph1 = transpose_pair(x1);
        pl1 = transpose_pair(y1);
        if (tail) {
          // the tail's mass is formed at the end from its token scores; its sums belong to no slot
          lw0 = lw1 = nw0 = nw1 = 0.f;
        }
      } else {
        // V rows: O^T += V^T P^T
        if (valid < QE_PAGE) {
          // rows past the tail's last token hold stale data: zero them (weight 0 must not meet
          // a NaN)
          for (int i = lane; i < (QE_PAGE - valid) * NB * 8; i += 32) {
            const int row = valid + i / (NB * 8), rest = i % (NB * 8);
            *reinterpret_cast<uint4*>(stage + (rest / 8) * 2048 + row * 128 + (rest % 8) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
          __syncwarp();
        }
#pragma unroll
        for (int m = 0; m < G8; ++m) {
          uint32_t va[4];
          ldsm_x4_t(va, stage + swz<D>(0, ((lane >> 4) << 3) + (lane & 7), m * 16 + ((lane >> 3) & 1) * 8));
          MmaOp<T>::run(oacc[m], va[0], va[1], va[2], va[3], ph0, ph1);
          MmaOp<T>::run(oacc[m], va[0], va[1], va[2], va[3], pl0, pl1);
        }
        if (!tail && ti == 2 * PPW - 1) window_end(cur_list_idx(cc));
      }
    } else {
      const uint8_t* stage = ring + s * STAGE;
      float sc[4 * BPC], p[4 * BPC];
#pragma unroll
      for (int bk = 0; bk < BPC; ++bk) {
        // ---- K side: S^T = (C s + Z) Q^T for tokens g8, 8 + g8 and heads h0, h1 ----
        const uint8_t* blk = stage + bk * BL::BYTES;
        float zs[4] = {0.f, 0.f, 0.f, 0.f};
        {
          const uint32_t zA =
              2 * t4 < G8 ? *reinterpret_cast<const uint32_t*>(blk + BL::KZ + (g8 * G8 + 2 * t4) * 2) : 0u;
          const uint32_t zB =
              2 * t4 < G8 ? *reinterpret_cast<const uint32_t*>(blk + BL::KZ + ((8 + g8) * G8 + 2 * t4) * 2) : 0u;
          mma_h8(zs, zA, zB, qgh);
          mma_h8(zs, zA, zB, qgl);
        }
        uint32_t kw[WPL];
        if constexpr (WPL == 4) {
          const uint4 v4 = *reinterpret_cast<const uint4*>(blk + BL::KC + lane * 16);
          kw[0] = v4.x; kw[1] = v4.y; kw[2] = v4.z; kw[3] = v4.w;
        } else {
          const uint2 v2 = *reinterpret_cast<const uint2*>(blk + BL::KC + lane * 8);
          kw[0] = v2.x; kw[1] = v2.y;
        }
        float2 sA = make_float2(0.f, 0.f), sB = make_float2(0.f, 0.f);
#pragma unroll
        for (int jj = 0; jj < WPL; ++jj) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int m = 2 * jj + e;
            const uint32_t x = e ? (kw[jj] >> 8) : kw[jj];
            // this lane's token scales s(g8), s(8 + g8) as float32 in both head columns
            const uint32_t sp = *reinterpret_cast<const uint32_t*>(blk + BL::KS + (m * QE_PAGE + 2 * g8) * 2);
            float cs[4] = {0.f, 0.f, 0.f, 0.f}, cc[4] = {0.f, 0.f, 0.f, 0.f};
            mma_h8(cs, sp, __byte_perm(sp, 0u, 0x1032), sel0);
            mma_h16(cc, code_reg<0>(x), code_reg<2>(x), code_reg<1>(x), code_reg<3>(x), qh[m][0], qh[m][1]);
            sA = ffma2(make_float2(cs[0], cs[1]), make_float2(cc[0], cc[1]), sA);
            sB = ffma2(make_float2(cs[2], cs[3]), make_float2(cc[2], cc[3]), sB);
          }
        }
        sA = ffma2(sA, fa, make_float2(zs[0], zs[1]));
        sB = ffma2(sB, fb, make_float2(zs[2], zs[3]));
        sc[4 * bk + 0] = sA.x;
        sc[4 * bk + 1] = sA.y;
        sc[4 * bk + 2] = sB.x;
        sc[4 * bk + 3] = sB.y;
      }
      softmax(sc, p, reinterpret_cast<const float*>(nring + s * NSB));
#pragma unroll
      for (int bk = 0; bk < BPC; ++bk) {
        // ---- V side: O^T += V^T (P^T s) per group, zero points Z^T P^T ----
        const uint8_t* blk = stage + bk * BL::BYTES;
        const float* pb = p + 4 * bk;
        uint32_t x0, y0, x1, y1;
        MmaOp<__half>::split(pb[0], pb[1], x0, y0);
        MmaOp<__half>::split(pb[2], pb[3], x1, y1);
        const uint32_t ph0 = transpose_pair(x0), pl0 = transpose_pair(y0);
        const uint32_t ph1 = transpose_pair(x1), pl1 = transpose_pair(y1);
        {
          uint2 zg = make_uint2(0u, 0u);
          if (g8 < G8) zg = *reinterpret_cast<const uint2*>(blk + BL::VZ + (g8 * QE_PAGE + 4 * t4) * 2);
          mma_h16(zacc, zg.x, 0u, zg.y, 0u, ph0, ph1);
          mma_h16(zacc, zg.x, 0u, zg.y, 0u, pl0, pl1);
        }
        // the codes of tokens 8..15 carry 4x: their weights are quartered (exact)
        const uint32_t pq1 = __hmul2_u32(ph1, kQuarter2), pql1 = __hmul2_u32(pl1, kQuarter2);
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
            const uint2 sg = *reinterpret_cast<const uint2*>(blk + BL::VS + (m * QE_PAGE + 4 * t4) * 2);
            uint32_t h0, l0, h1, l1;
            ws_split(ph0, pl0, sg.x, h0, l0);
            ws_split(pq1, pql1, sg.y, h1, l1);
            const uint32_t c0 = code_reg<0>(x), c1 = code_reg<1>(x), c2 = code_reg<2>(x), c3 = code_reg<3>(x);
            mma_h16(oacc[m], c0, c2, c1, c3, h0, h1);
            mma_h16(oacc[m], c0, c2, c1, c3, l0, l1);
          }
        }
      }
      if (ti == CPW - 1) window_end(cur_list_idx(cc));
    }
    __syncwarp();
    cur_next(cc);
    ++k;
  }
  if (int2_units) to_units(false);
  if (!ok) {  // drain copies still in flight if a wait gave up
    for (; k < issued; ++k) mbar_wait_bounded(&bars[k % NST], (k / NST) & 1, st.status, 2000 + u);
  }
  // add the zero-point part of each element's group
#pragma unroll
  for (int m = 0; m < G8; ++m) {
    const float z0 = __shfl_sync(0xffffffffu, zacc[0], 4 * m + t4);
    const float z1 = __shfl_sync(0xffffffffu, zacc[1], 4 * m + t4);
    oacc[m][0] += z0;
    oacc[m][1] += z1;
    oacc[m][2] += z0;
    oacc[m][3] += z1;
  }
#pragma unroll
  for (int o2 = 4; o2 < 32; o2 <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o2);
  }

  // the window scores this CTA updates (one window per thread and pass): their ids and
  // cumulative values are fetched before the CTA barrier, so that the loads overlap the wait for
  // the slowest warp; their step partials (written by any warp of the CTA) after it
  constexpr int kPre = 1;
  int pw_win[kPre], pw_li[kPre];
  float pw_m[kPre], pw_p[kPre], pw_part[kPre][3 * G];
#pragma unroll
  for (int x = 0; x < kPre; ++x) {
    const int jj = threadIdx.x + x * kNW * 32;
    pw_win[x] = -1;
    pw_li[x] = 0;
    if (jj < nF + nQ) {
      const int li = jj < nF ? f0 + jj : nf + q0 + (jj - nF);
      const int win = jj < nF ? st.full_list[ub + li] : st.int2_list[ub + li - nf];
      if (win >= 0 && win < st.Wmax) {
        pw_win[x] = win;
        pw_li[x] = li;
        pw_m[x] = st.mass[ub + win];
        pw_p[x] = st.pert[ub + win];
      }
    }
  }
  float tail_m0 = 0.f;  // the tail window's cumulative mass
  if (has_tail && threadIdx.x == 0) tail_m0 = st.mass[ub + a.tail_win];
  // ---- merge the warps into the CTA's partial ----
  const bool cta_ok = __syncthreads_and(ok ? 1 : 0) != 0;  // also: every warp is done with its ring
  // the tail tokens' scores (written by a warp of this CTA during the pass) and cumulative
  // attention, fetched now so that the loads overlap the merges
  constexpr int kTailPer = (W * G + kNW * 32 - 1) / (kNW * 32);
  float t_s[kTailPer], t_p[kTailPer];
  if (has_tail) {
#pragma unroll
    for (int x = 0; x < kTailPer; ++x) {
      const int i = threadIdx.x + x * kNW * 32;
      t_s[x] = t_p[x] = 0.f;
      if (i < a.tail_len * G) {
        t_s[x] = a.tail_s[(size_t)u * W * G + i];
        t_p[x] = st.tail_p[(size_t)u * W * G + i];
      }
    }
  }
#pragma unroll
  for (int x = 0; x < kPre; ++x)
    if (pw_win[x] >= 0) {
      const float* wp = a.win_part + (ub + pw_li[x]) * win_part_floats(D, G);
#pragma unroll
      for (int h = 0; h < 3 * G; ++h) pw_part[x][h] = wp[h];
    }
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
  float* oks = okv + 1;                               // [S] every CTA's flag
  if (g8 == 0) {
    if (h0 < G) {
      mw[warp * G + h0] = m0;
      lwv[warp * G + h0] = l0;
    }
    if (h1 < G) {
      mw[warp * G + h1] = m1;
      lwv[warp * G + h1] = l1;
    }
  }
  {
    float* a0 = aw + (size_t)warp * G * D;
#pragma unroll
    for (int m = 0; m < G8; ++m) {
      if (2 * t4 < G) {
        a0[(2 * t4) * D + m * 16 + g8] = oacc[m][0];
        a0[(2 * t4) * D + m * 16 + 8 + g8] = oacc[m][2];
      }
      if (2 * t4 + 1 < G) {
        a0[(2 * t4 + 1) * D + m * 16 + g8] = oacc[m][1];
        a0[(2 * t4 + 1) * D + m * 16 + 8 + g8] = oacc[m][3];
      }
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
  const int per = (G * D + S - 1) / S;
  const int o1 = min((split + 1) * per, G * D);
  const int i_first = split * per + threadIdx.x;
  cluster_sync();
  // this thread's first output element: its S partials are fetched in the same round as the
  // CTA maxima and sums
  float vfirst[QE_MAX_SPLITS_CLUSTER];
  if (i_first < o1) {
#pragma unroll
    for (int r = 0; r < QE_MAX_SPLITS_CLUSTER; ++r)
      if (r < S) vfirst[r] = ld_cluster(ca + i_first, (uint32_t)r);
  }
  for (int i = threadIdx.x; i < S * G; i += blockDim.x) {
    const float vm = ld_cluster(cm + i % G, (uint32_t)(i / G));
    const float vl = ld_cluster(cl + i % G, (uint32_t)(i / G));
    pm[i] = vm;
    pl[i] = vl;
  }
  // every CTA of the unit must have finished its waits: a CTA that gave up holds partials of
  // a part of its windows, and window partials it never wrote may be stale
  if (threadIdx.x < S) oks[threadIdx.x] = ld_cluster(okv, (uint32_t)threadIdx.x);
  __syncthreads();
  float all_ok = 1.f;
  for (int r = 0; r < S; ++r) all_ok = fminf(all_ok, oks[r]);
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
  if (i_first < o1) {
    const int h = i_first / D;
    float A = 0.f;
#pragma unroll
    for (int r = 0; r < QE_MAX_SPLITS_CLUSTER; ++r)
      if (r < S) A = fmaf(vfirst[r], pf[r * G + h], A);
    a.out[((size_t)b * st.Hq + (size_t)kvh * G + h) * D + i_first % D] = A / gl[h];
  }
  {
    for (int i = i_first + blockDim.x; i < o1; i += blockDim.x) {
      const int h = i / D;
      float v[QE_MAX_SPLITS_CLUSTER];
#pragma unroll
      for (int r = 0; r < QE_MAX_SPLITS_CLUSTER; ++r)
        if (r < S) v[r] = ld_cluster(ca + i, (uint32_t)r);
      float A = 0.f;
#pragma unroll
      for (int r = 0; r < QE_MAX_SPLITS_CLUSTER; ++r)
        if (r < S) A = fmaf(v[r], pf[r * G + h], A);
      a.out[((size_t)b * st.Hq + (size_t)kvh * G + h) * D + i % D] = A / gl[h];
    }
  }
  // this CTA has read every partial it needs from the cluster (the values are in registers,
  // there is nothing to order): signal it now, and wait for the other CTAs, which may still read
  // this CTA's partial, only before exiting
  cluster_arrive_relaxed();
  if (all_ok > 0.f) {
    // exact attention mass and perturbation of this step for the windows this CTA streamed
    auto update = [&](int win, float m0, float p0, const float* wp) {
      float dm = 0.f, dp = 0.f;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float f = ex2(wp[h] - lse[h]);
        dm = fmaf(wp[G + h], f, dm);
        dp = fmaf(wp[2 * G + h], f, dp);
      }
      st.mass[ub + win] = m0 + dm;
      st.pert[ub + win] = p0 + dp;
    };
#pragma unroll
    for (int x = 0; x < kPre; ++x)
      if (pw_win[x] >= 0) update(pw_win[x], pw_m[x], pw_p[x], pw_part[x]);
    for (int jj = threadIdx.x + kPre * kNW * 32; jj < nF + nQ; jj += blockDim.x) {
      const int li = jj < nF ? f0 + jj : nf + q0 + (jj - nF);
      const int win = jj < nF ? st.full_list[ub + li] : st.int2_list[ub + li - nf];
      if (win >= 0 && win < st.Wmax)
        update(win, st.mass[ub + win], st.pert[ub + win], a.win_part + (ub + li) * win_part_floats(D, G));
    }
    // tail tokens (last CTA of the cluster): cumulative per-token attention and window mass
    if (has_tail) {
      float tm = 0.f;
#pragma unroll
      for (int x = 0; x < kTailPer; ++x) {
        const int i = threadIdx.x + x * kNW * 32;
        if (i < a.tail_len * G) {
          const float pv = ex2(t_s[x] - lse[i % G]);
          st.tail_p[(size_t)u * W * G + i] = t_p[x] + pv;
          tm += pv;
        }
      }
      tm = warp_sum(tm);
      if (lane == 0) red[warp] = tm;
      __syncthreads();
      if (threadIdx.x == 0) {
        float s2 = 0.f;
        for (int x = 0; x < kNW; ++x) s2 += red[x];
        st.mass[ub + a.tail_win] = tail_m0 + s2;
      }
    }
  }
  cluster_wait();  // keep this CTA's partial alive until every CTA of the cluster has read it
}

template <typename T, int D, int G, int W>
int launch_decode_w(qe_ctx* c, const void* q, float* out, cudaStream_t s, const void* k_new,
                    const void* v_new) {
  constexpr size_t smem = decode_smem_bytes<D, G>();
  static_assert((size_t)(kNW * G * (D + 2) + 2 * QE_MAX_G + G * D + 3 * QE_MAX_SPLITS_CLUSTER * QE_MAX_G +
                         2 * QE_MAX_G + kNW + 1 + QE_MAX_SPLITS_CLUSTER) * 4 <=
                    (size_t)kNW * nst_of(G) * stage_bytes<D>(),
                "merge area");
  auto kern = decode_kernel<T, D, G, W>;
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
  a.nf = c->counts_exact ? c->n_full_max : -1;
  a.nq = c->counts_exact ? c->n_int2_max : -1;
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

template <typename T, int D, int G>
int launch_decode_t(qe_ctx* c, const void* q, float* out, cudaStream_t s, const void* k, const void* v) {
  switch (c->cfg.window) {
    case 16: return launch_decode_w<T, D, G, 16>(c, q, out, s, k, v);
    case 32: return launch_decode_w<T, D, G, 32>(c, q, out, s, k, v);
    case 64: return launch_decode_w<T, D, G, 64>(c, q, out, s, k, v);
    default: return QE_ERR_UNSUPPORTED_SHAPE;
  }
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
