// SEKV-style mixed-resolution attention over entropy-guided spans.
//
// "Resumo Técnico: SEKV" - Metodologia 1 (Segmentação de Intervalos Guiada por Entropia:
// tokens of high surprisal are anchors kept at full resolution; the tokens between anchors form
// spans), 2 (each span has a GPU-resident summary: the surprisal-weighted, normalised mean of
// its keys) and 3 (Atenção de Resolução Mista: anchors contribute their K/V, spans that are not
// expanded contribute their summary with a size correction, expanded spans their tokens). The
// trained routing projections and thresholds and the CPU low-rank reconstruction are not part
// of this path: a span is expanded when the largest scaled score of its summary over the
// group's query heads reaches a given threshold, and an expanded span contributes the tokens
// the caller keeps.
//
// Build (once per cache): one CTA per sequence scans the surprisal and writes the anchor
// positions and the span bounds (block-wide prefix sums); one warp per (kv head, span) forms
// the summary key and value in fp32. Attend (every step): one warp per (kv head, span) decides
// the expansion; then the unit's items (anchors, then spans) are split over S CTAs, a warp
// takes whole items and keeps an online softmax per head (the score of a summary gets
// log2|S| added in the log2 domain), and a last kernel merges the S partials.
#include <math.h>

#include "qe_internal.cuh"
#include "warp_mma.cuh"

namespace {

constexpr int kSekvWarps = 4;      // warps per CTA (gate, summarize, attend)
constexpr int kSekvMaxSplits = 32;
constexpr int kSekvSpanBlocks = 64;    // CTAs per unit for the per-span kernels (grid-stride over spans)

struct SekvLayout {
  size_t counts, anchor_pos, span_start, span_end, kbar, vbar, expanded, part_ml, part_o, tok, sums, lcount, total;
  int cap;  // spans per sequence at most: (n + 1) / 2 (two spans are separated by an anchor)
};

SekvLayout sekv_layout(int B, int Hkv, int n, int D, int G) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t U = (size_t)B * Hkv;
  SekvLayout L{};
  L.cap = (n + 1) / 2;
  L.counts = 0;
  L.anchor_pos = up(L.counts + (size_t)B * 2 * 4);
  L.span_start = up(L.anchor_pos + (size_t)B * n * 4);
  L.span_end = up(L.span_start + (size_t)B * L.cap * 4);
  L.kbar = up(L.span_end + (size_t)B * L.cap * 4);
  L.vbar = up(L.kbar + U * L.cap * D * 4);
  L.expanded = up(L.vbar + U * L.cap * D * 4);
  L.part_ml = up(L.expanded + U * L.cap);
  L.part_o = up(L.part_ml + U * kSekvMaxSplits * G * 2 * 4);
  L.tok = up(L.part_o + U * kSekvMaxSplits * G * (size_t)D * 4);  // [U][n] tokens attended one by one
  L.sums = up(L.tok + U * (size_t)n * 4);                          // [U][cap] spans attended by summary
  L.lcount = up(L.sums + U * (size_t)L.cap * 4);                   // [U][2] their counts
  L.total = up(L.lcount + U * 2 * 4);
  return L;
}


__device__ __forceinline__ float ex2s(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// NP (a power of two, 4..32) values per lane summed over the warp: a reduce-scatter (at partner
// distance o the lane keeps the lower or upper half of its block, by bit o of its index, and adds
// the partner's copy of that half) and then an all-gather (the same levels in reverse), so every
// lane ends with all NP sums; NP - 1 shuffles each way instead of five per value.
template <int NP>
__device__ __forceinline__ void warp_sum_all(float (&d)[NP], int lane) {
#pragma unroll
  for (int lvl = 0; lvl < 5; ++lvl) {
    const int o = 16 >> lvl, width = NP >> lvl;
    if (width > 1) {
      const int half = width >> 1;
      const bool up = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < half; ++i) {
        const float send = up ? d[i] : d[i + half];
        const float keep = up ? d[i + half] : d[i];
        d[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    } else {
      d[0] += __shfl_xor_sync(0xffffffffu, d[0], o);
    }
  }
#pragma unroll
  for (int lvl = 4; lvl >= 0; --lvl) {
    const int o = 16 >> lvl, width = NP >> lvl;
    if (width > 1) {
      const int half = width >> 1;
      const bool up = (lane & o) != 0;
      float r[NP / 2];
#pragma unroll
      for (int i = 0; i < half; ++i) r[i] = __shfl_xor_sync(0xffffffffu, d[i], o);
#pragma unroll
      for (int i = 0; i < half; ++i) {
        const float mine = d[i];
        d[i] = up ? r[i] : mine;
        d[i + half] = up ? mine : r[i];
      }
    }
  }
}

// exclusive prefix sum of a 0/1 flag over the block (blockDim.x = 1024); *total gets the sum
__device__ int block_scan01(int v, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned m = __ballot_sync(0xffffffffu, v);
  const int in_warp = __popc(m & ((1u << lane) - 1u));
  if (lane == 0) wsum[warp] = __popc(m);
  __syncthreads();
  if (warp == 0) {
    int x = lane < (int)(blockDim.x >> 5) ? wsum[lane] : 0;
    int inc = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    wsum[lane] = inc - x;  // exclusive
    if (lane == 31) wsum[32] = inc;
  }
  __syncthreads();
  const int r = wsum[warp] + in_warp;
  *total = wsum[32];
  __syncthreads();
  return r;
}

// exclusive prefix sum of a non-negative int over the block (blockDim.x = 1024); *total gets the sum
__device__ int block_scan_int(int v, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const int x = lane < (int)(blockDim.x >> 5) ? wsum[lane] : 0;
    int xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += y;
    }
    wsum[lane] = xi - x;
    if (lane == 31) wsum[32] = xi;
  }
  __syncthreads();
  const int r = wsum[warp] + inc - v;
  *total = wsum[32];
  __syncthreads();
  return r;
}

// anchors: H_t >= tau; spans: maximal runs of non-anchors (start, end exclusive)
__global__ void __launch_bounds__(1024) sekv_segment_kernel(const float* __restrict__ H, int n, float tau, int cap,
                                                            int32_t* counts, int32_t* anchor_pos,
                                                            int32_t* span_start, int32_t* span_end) {
  const int b = blockIdx.x;
  const float* h = H + (size_t)b * n;
  __shared__ int wsum[33];
  int carry_a = 0, carry_s = 0;
  for (int base = 0; base < n; base += blockDim.x) {
    const int t = base + threadIdx.x;
    const bool in = t < n;
    const bool anc = in && h[t] >= tau;
    const bool start = in && !anc && (t == 0 || h[t - 1] >= tau);
    const bool end = in && !anc && (t == n - 1 || h[t + 1] >= tau);
    int ta, ts;
    const int ia = block_scan01(anc ? 1 : 0, wsum, &ta);
    const int is = block_scan01(start ? 1 : 0, wsum, &ts);
    if (anc) anchor_pos[(size_t)b * n + carry_a + ia] = t;
    if (start) span_start[(size_t)b * cap + carry_s + is] = t;
    // the span that token t ends began at the last start at or before t
    if (end) span_end[(size_t)b * cap + carry_s + is + (start ? 1 : 0) - 1] = t + 1;
    carry_a += ta;
    carry_s += ts;
  }
  if (threadIdx.x == 0) {
    counts[b * 2 + 0] = carry_a;
    counts[b * 2 + 1] = carry_s;
  }
}

template <typename T, int DPL>
__device__ __forceinline__ void load_dims(const T* row, int lane, float (&x)[DPL]) {
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

// one warp per (kv head, span): kbar = sum H_t K_t / sum H_t (plain mean if the sum is 0)
template <typename T, int DPL>
__global__ void __launch_bounds__(kSekvWarps * 32)
    sekv_summarize_kernel(const T* __restrict__ K, const T* __restrict__ V, const float* __restrict__ H, int n,
                          int Hkv, int cap, const int32_t* counts, const int32_t* span_start,
                          const int32_t* span_end, float* kbar, float* vbar) {
  constexpr int D = 32 * DPL;
  const int u = blockIdx.x, b = u / Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nspans = counts[b * 2 + 1];
  for (int i = blockIdx.y * kSekvWarps + warp; i < nspans; i += gridDim.y * kSekvWarps) {
    const int s = span_start[(size_t)b * cap + i], e = span_end[(size_t)b * cap + i];
    float ak[DPL] = {}, av[DPL] = {}, pk[DPL] = {}, pv[DPL] = {};
    float ws = 0.f;
    for (int t = s; t < e; ++t) {
      const float w = H[(size_t)b * n + t];
      float kx[DPL], vx[DPL];
      load_dims<T, DPL>(K + ((size_t)u * n + t) * D, lane, kx);
      load_dims<T, DPL>(V + ((size_t)u * n + t) * D, lane, vx);
  #pragma unroll
      for (int j = 0; j < DPL; ++j) {
        ak[j] = fmaf(w, kx[j], ak[j]);
        av[j] = fmaf(w, vx[j], av[j]);
        pk[j] += kx[j];
        pv[j] += vx[j];
      }
      ws += w;
    }
    const float inv = ws > 0.f ? 1.f / ws : 1.f / (float)(e - s);
    float* kr = kbar + ((size_t)u * cap + i) * D + lane * DPL;
    float* vr = vbar + ((size_t)u * cap + i) * D + lane * DPL;
  #pragma unroll
    for (int j = 0; j < DPL; ++j) {
      kr[j] = (ws > 0.f ? ak[j] : pk[j]) * inv;
      vr[j] = (ws > 0.f ? av[j] : pv[j]) * inv;
    }
  }
}

// one warp per four (kv head, span) pairs at a time: expanded = max_h q_h . kbar / sqrt(D) >= theta
template <typename T, int DPL, int G>
__global__ void __launch_bounds__(kSekvWarps * 32)
    sekv_gate_kernel(const T* __restrict__ q, int Hq, int Hkv, int cap, const int32_t* counts,
                     const float* __restrict__ kbar, float scale, float theta, uint8_t* expanded) {
  constexpr int D = 32 * DPL, KB = 4, NPAIR = G * KB;
  constexpr int NP = NPAIR <= 4 ? 4 : (NPAIR <= 8 ? 8 : (NPAIR <= 16 ? 16 : 32));
  const int u = blockIdx.x, b = u / Hkv, kvh = u % Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nspans = counts[b * 2 + 1];
  float qx[G][DPL];
#pragma unroll
  for (int h = 0; h < G; ++h) load_dims<T, DPL>(q + ((size_t)b * Hq + (size_t)kvh * G + h) * D, lane, qx[h]);
  const int stride = gridDim.y * kSekvWarps;
  for (int base = blockIdx.y * kSekvWarps + warp; base < nspans; base += KB * stride) {
    float kx[KB][DPL];
#pragma unroll
    for (int k = 0; k < KB; ++k) {
      const int i = base + k * stride;
      const float* kr = kbar + ((size_t)u * cap + (i < nspans ? i : 0)) * D + lane * DPL;
#pragma unroll
      for (int j = 0; j < DPL; ++j) kx[k][j] = i < nspans ? kr[j] : 0.f;
    }
    float d[NP];
#pragma unroll
    for (int v = 0; v < NP; ++v) {
      float t = 0.f;
      if (v < NPAIR) {
#pragma unroll
        for (int j = 0; j < DPL; ++j) t = fmaf(qx[v / KB][j], kx[v % KB][j], t);
      }
      d[v] = t;
    }
    warp_sum_all<NP>(d, lane);
#pragma unroll
    for (int k = 0; k < KB; ++k) {
      const int i = base + k * stride;
      float g = -INFINITY;
#pragma unroll
      for (int h = 0; h < G; ++h) g = fmaxf(g, d[h * KB + k] * scale);
      if (lane == k && i < nspans) expanded[(size_t)u * cap + i] = g >= theta ? 1 : 0;
    }
  }
}

// Per step, one CTA per unit: the tokens attended one by one (the anchors, then every token of
// each expanded span, in position order within a span) and the spans attended by their summary.
__global__ void __launch_bounds__(1024) sekv_lists_kernel(const int32_t* __restrict__ counts,
                                                          const int32_t* __restrict__ anchor_pos,
                                                          const int32_t* __restrict__ span_start,
                                                          const int32_t* __restrict__ span_end,
                                                          const uint8_t* __restrict__ expanded, int n, int cap,
                                                          int Hkv, int32_t* tok, int32_t* sums, int32_t* lcount) {
  const int u = blockIdx.x, b = u / Hkv;
  const int A = counts[b * 2 + 0], NS = counts[b * 2 + 1];
  int32_t* tl = tok + (size_t)u * n;
  int32_t* sl = sums + (size_t)u * cap;
  for (int i = threadIdx.x; i < A; i += blockDim.x) tl[i] = anchor_pos[(size_t)b * n + i];
  __shared__ int wsum[33];
  int carry_t = A, carry_s = 0;
  for (int base = 0; base < NS; base += blockDim.x) {
    const int i = base + threadIdx.x;
    const bool in = i < NS;
    const bool ex = in && expanded[(size_t)u * cap + i];
    const int s0 = ex ? span_start[(size_t)b * cap + i] : 0, e0 = ex ? span_end[(size_t)b * cap + i] : 0;
    int tt, ts;
    const int it = block_scan_int(e0 - s0, wsum, &tt);
    const int is = block_scan01(in && !ex ? 1 : 0, wsum, &ts);
    for (int t = s0; t < e0; ++t) tl[carry_t + it + (t - s0)] = t;
    if (in && !ex) sl[carry_s + is] = i;
    carry_t += tt;
    carry_s += ts;
  }
  if (threadIdx.x == 0) {
    lcount[u * 2 + 0] = carry_t;
    lcount[u * 2 + 1] = carry_s;
  }
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src, int bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

struct SekvAttendArgs {
  const void* q;
  const void* K;
  const void* V;
  const int32_t* counts;
  const int32_t* anchor_pos;
  const int32_t* span_start;
  const int32_t* span_end;
  const float* kbar;
  const float* vbar;
  const uint8_t* expanded;
  float* part_ml;  // [U][S][G][2]
  float* part_o;   // [U][S][G][D]
  const int32_t* tok;     // [U][n] tokens attended one by one
  const int32_t* sums;    // [U][cap] spans attended by summary
  const int32_t* lcount;  // [U][2]
  int n, cap, Hq, Hkv, S;
  float scale_log2;
};

// One split of a unit: its share of the unit's tokens attended one by one, 16 per tile on the
// warp-level tensor cores, and its share of the unit's span summaries on the CUDA cores.
// Tokens: a warp gathers the K and V rows of 16 tokens with cp.async into a 128-byte-swizzled
// tile (two stages, the next tile's gather overlapping the current one), S^T = K Q^T with the
// tokens as MMA rows and the query heads as columns, an online softmax per lane for its two
// heads, P split into a 16-bit high part and its residual and turned by movmatrix into the B
// fragment of O^T = V^T P^T. Summaries: four per warp step, the G x 4 (head, summary) dot
// products summed over the warp by a reduce-scatter and an all-gather, the score raised by
// log2|S|. The two partial states of a warp are merged, then the warps, then (next kernel) the
// splits.
template <typename T, int DPL, int G>
__global__ void __launch_bounds__(kSekvWarps * 32) sekv_attend_kernel(SekvAttendArgs a) {
  constexpr int D = 32 * DPL, G8 = D / 16;
  constexpr int TILE = 2 * QE_PAGE * D * 2;  // K rows, then V rows, of 16 tokens
  constexpr int CPR = D / 8;                 // 16-byte chunks per row
  static_assert(G <= 8, "a warp's MMA columns hold at most 8 query heads");
  extern __shared__ __align__(128) uint8_t sekv_smem[];
  const int u = blockIdx.x / a.S, split = blockIdx.x % a.S;
  const int b = u / a.Hkv, kvh = u % a.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g8 = lane >> 2, t4 = lane & 3;
  const int ntok = a.lcount[u * 2 + 0], nsum = a.lcount[u * 2 + 1];
  const int NT = (ntok + 15) / 16;
  const int ta = (int)((long long)NT * split / a.S), tbn = (int)((long long)NT * (split + 1) / a.S);
  const int sa = (int)((long long)nsum * split / a.S), sbn = (int)((long long)nsum * (split + 1) / a.S);
  const T* Kb = reinterpret_cast<const T*>(a.K) + (size_t)u * a.n * D;
  const T* Vb = reinterpret_cast<const T*>(a.V) + (size_t)u * a.n * D;
  const int32_t* tl = a.tok + (size_t)u * a.n;
  const T* qbase = reinterpret_cast<const T*>(a.q) + ((size_t)b * a.Hq + (size_t)kvh * G) * D;
  // q for the summaries: lane l holds elements l*DPL .. of every head
  float qv[G][DPL];
#pragma unroll
  for (int h = 0; h < G; ++h) load_dims<T, DPL>(qbase + (size_t)h * D, lane, qv[h]);
  // q as the B operand of S^T = K Q^T: head g8's elements 16m + 2t4, +1 and 16m + 8 + 2t4, +1
  uint32_t qb[G8][2];
  {
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(qbase + (size_t)(g8 < G ? g8 : 0) * D);
#pragma unroll
    for (int m = 0; m < G8; ++m) {
      qb[m][0] = g8 < G ? qrow[m * 8 + t4] : 0u;
      qb[m][1] = g8 < G ? qrow[m * 8 + 4 + t4] : 0u;
    }
  }

  // ---- tokens on the tensor cores ----
  const int h0 = 2 * t4, h1 = 2 * t4 + 1;
  const float hm0 = h0 < G ? 1.f : 0.f, hm1 = h1 < G ? 1.f : 0.f;
  float m0 = -1e30f, m1 = -1e30f, l0 = 0.f, l1 = 0.f;
  float oacc[G8][4];
#pragma unroll
  for (int m = 0; m < G8; ++m) oacc[m][0] = oacc[m][1] = oacc[m][2] = oacc[m][3] = 0.f;
  uint8_t* ring = sekv_smem + warp * 2 * TILE;
  // gather tile t into stage st: row r is token tl[16 t + r]; rows past the list are zero-filled
  auto gather = [&](int t, int st) {
    const int row = t * 16 + (lane & 15);
    const int pos = (lane < 16 && row < ntok) ? tl[row] : -1;
    uint8_t* dst = ring + st * TILE;
#pragma unroll
    for (int k = 0; k < 16 * CPR / 32; ++k) {
      const int c = lane + 32 * k, r = c / CPR, cc = c % CPR;
      const int p = __shfl_sync(0xffffffffu, pos, r);
      const size_t off = (size_t)(p >= 0 ? p : 0) * D + cc * 8;
      const int bytes = p >= 0 ? 16 : 0;
      cp_async16(dst + swz<D>(0, r, cc * 8), Kb + off, bytes);
      cp_async16(dst + swz<D>(1, r, cc * 8), Vb + off, bytes);
    }
    cp_async_commit();
  };
  auto transpose_pair = [](uint32_t x) {
    uint32_t y;
    asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
  };
  const float sl2 = a.scale_log2;
  int stg = 0;
  if (ta + warp < tbn) gather(ta + warp, 0);
  for (int t = ta + warp; t < tbn; t += kSekvWarps, stg ^= 1) {
    if (t + kSekvWarps < tbn) {
      gather(t + kSekvWarps, stg ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncwarp();
    const uint8_t* tile = ring + stg * TILE;
    const int valid = min(16, ntok - t * 16);
    float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int m = 0; m < G8; ++m) {
      uint32_t ka[4];
      ldsm_x4(ka, tile + swz<D>(0, ((lane >> 3) & 1) * 8 + (lane & 7), m * 16 + (lane >> 4) * 8));
      if (m & 1) MmaOp<T>::run(c1, ka[0], ka[1], ka[2], ka[3], qb[m][0], qb[m][1]);
      else MmaOp<T>::run(c0, ka[0], ka[1], ka[2], ka[3], qb[m][0], qb[m][1]);
    }
    // lane (g8, t4): tokens g8 (slots 0, 1) and 8 + g8 (slots 2, 3), heads h0 (0, 2) and h1 (1, 3)
    float sc[4] = {(c0[0] + c1[0]) * sl2, (c0[1] + c1[1]) * sl2, (c0[2] + c1[2]) * sl2, (c0[3] + c1[3]) * sl2};
    if (g8 >= valid) sc[0] = sc[1] = -INFINITY;
    if (g8 + 8 >= valid) sc[2] = sc[3] = -INFINITY;
    float x0 = fmaxf(sc[0], sc[2]), x1 = fmaxf(sc[1], sc[3]);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, o));
      x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, o));
    }
    const float n0 = fmaxf(m0, x0), n1 = fmaxf(m1, x1);
    const float f0 = ex2s(m0 - n0), f1 = ex2s(m1 - n1);
    l0 *= f0;
    l1 *= f1;
#pragma unroll
    for (int m = 0; m < G8; ++m) {
      oacc[m][0] *= f0;
      oacc[m][1] *= f1;
      oacc[m][2] *= f0;
      oacc[m][3] *= f1;
    }
    m0 = n0;
    m1 = n1;
    const float p0 = hm0 * ex2s(sc[0] - m0), p1 = hm1 * ex2s(sc[1] - m1);
    const float p2 = hm0 * ex2s(sc[2] - m0), p3 = hm1 * ex2s(sc[3] - m1);
    l0 += p0 + p2;
    l1 += p1 + p3;
    uint32_t xh0, xl0, xh1, xl1;
    MmaOp<T>::split(p0, p1, xh0, xl0);
    MmaOp<T>::split(p2, p3, xh1, xl1);
    const uint32_t ph0 = transpose_pair(xh0), pl0 = transpose_pair(xl0);
    const uint32_t ph1 = transpose_pair(xh1), pl1 = transpose_pair(xl1);
#pragma unroll
    for (int m = 0; m < G8; ++m) {
      uint32_t va[4];
      ldsm_x4_t(va, tile + swz<D>(1, ((lane >> 4) << 3) + (lane & 7), m * 16 + ((lane >> 3) & 1) * 8));
      MmaOp<T>::run(oacc[m], va[0], va[1], va[2], va[3], ph0, ph1);
      MmaOp<T>::run(oacc[m], va[0], va[1], va[2], va[3], pl0, pl1);
    }
    __syncwarp();
  }
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }

  // ---- span summaries on the CUDA cores ----
  float m[G], l[G], acc[G][DPL];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -1e30f;
    l[h] = 0.f;
#pragma unroll
    for (int j = 0; j < DPL; ++j) acc[h][j] = 0.f;
  }
  // KB keys at a time: the lane's partial dot products of the G x KB (head, key) pairs are
  // summed over the warp by a reduce-scatter (a lane ends with one full sum) followed by an
  // all-gather (every lane then holds every score), NP - 1 shuffles each instead of five per
  // pair; then every lane updates the same online-softmax state of each head once per batch.
  // bias: the log2-domain score offset of each key (-inf for an unused slot).
  constexpr int KB = 4, NPAIR = G * KB;
  constexpr int NP = NPAIR <= 4 ? 4 : (NPAIR <= 8 ? 8 : (NPAIR <= 16 ? 16 : 32));
  static_assert(NPAIR <= 32, "at most 32 (head, key) pairs per batch");
  auto take_batch = [&](const float (&kx)[KB][DPL], const float (&vx)[KB][DPL], const float (&bias)[KB]) {
    float d[NP];
#pragma unroll
    for (int v = 0; v < NP; ++v) {
      float t = 0.f;
      if (v < NPAIR) {
#pragma unroll
        for (int j = 0; j < DPL; ++j) t = fmaf(qv[v / KB][j], kx[v % KB][j], t);
      }
      d[v] = t;
    }
    warp_sum_all<NP>(d, lane);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float sc[KB], mx = m[h];
#pragma unroll
      for (int k = 0; k < KB; ++k) {
        sc[k] = fmaf(d[h * KB + k], a.scale_log2, bias[k]);
        mx = fmaxf(mx, sc[k]);
      }
      const float f = ex2s(m[h] - mx);
      float p[KB], ps = 0.f;
#pragma unroll
      for (int k = 0; k < KB; ++k) {
        p[k] = ex2s(sc[k] - mx);
        ps += p[k];
      }
      l[h] = fmaf(l[h], f, ps);
#pragma unroll
      for (int j = 0; j < DPL; ++j) {
        float t = acc[h][j] * f;
#pragma unroll
        for (int k = 0; k < KB; ++k) t = fmaf(p[k], vx[k][j], t);
        acc[h][j] = t;
      }
      m[h] = mx;
    }
  };
  // The warp's batches of KB summaries flow through its gather ring (now idle), split into four
  // slots of KB key rows and KB value rows, three batches in flight ahead of the one computed.
  // Batch c holds the warp's summaries base_c + k * kSekvWarps (k < KB), base_c = sa + warp +
  // c * KB * kSekvWarps; a slot's rows are float32, lane l reading its DPL elements.
  constexpr int SROW = D * 4;                 // one float32 row
  constexpr int SLOT = 2 * KB * SROW;         // KB key rows, then KB value rows
  static_assert(4 * SLOT <= 2 * TILE, "four summary slots fit in a warp's gather ring");
  __shared__ float sbias[kSekvWarps][4][KB];
  const int nbatch = sbn > sa + warp ? (sbn - sa - warp + KB * kSekvWarps - 1) / (KB * kSekvWarps) : 0;
  auto sgather = [&](int c) {
    if (c < nbatch) {
      const int base = sa + warp + c * KB * kSekvWarps;
      uint8_t* slot = ring + (c & 3) * SLOT;
      // lane k < KB: the k-th summary's span index and its log2-size bias (-inf when absent)
      int i = -1;
      if (lane < KB) {
        const int it = base + lane * kSekvWarps;
        if (it < sbn) {
          i = a.sums[(size_t)u * a.cap + it];
          const int s0 = a.span_start[(size_t)b * a.cap + i], e0 = a.span_end[(size_t)b * a.cap + i];
          sbias[warp][c & 3][lane] = log2f((float)(e0 - s0));  // the summary stands for e0 - s0 tokens
        } else {
          sbias[warp][c & 3][lane] = -INFINITY;
        }
      }
#pragma unroll
      for (int x = 0; x < 2 * KB * SROW / 16 / 32; ++x) {
        const int ch = lane + 32 * x;           // 16-byte chunk of the slot
        const int row = ch / (SROW / 16);       // 0..KB-1 keys, KB..2KB-1 values
        const int k = row % KB, w16 = ch % (SROW / 16);
        const int ik = __shfl_sync(0xffffffffu, i, k);
        const float* src = (row < KB ? a.kbar : a.vbar) + ((size_t)u * a.cap + (ik >= 0 ? ik : 0)) * D + w16 * 4;
        cp_async16(slot + row * SROW + w16 * 16, src, ik >= 0 ? 16 : 0);
      }
    }
    cp_async_commit();  // one group per batch index, empty past the end, so the waits below line up
  };
  sgather(0);
  sgather(1);
  sgather(2);
  for (int c = 0; c < nbatch; ++c) {
    cp_async_wait<2>();
    __syncwarp();
    const uint8_t* slot = ring + (c & 3) * SLOT;
    float kx[KB][DPL], vx[KB][DPL], bias[KB];
#pragma unroll
    for (int k = 0; k < KB; ++k) {
      const float* kr = reinterpret_cast<const float*>(slot + k * SROW) + lane * DPL;
      const float* vr = reinterpret_cast<const float*>(slot + (KB + k) * SROW) + lane * DPL;
#pragma unroll
      for (int j = 0; j < DPL; ++j) {
        kx[k][j] = kr[j];
        vx[k][j] = vr[j];
      }
      bias[k] = sbias[warp][c & 3][k];
    }
    take_batch(kx, vx, bias);
    __syncwarp();  // the slot is read before the next gather into it
    sgather(c + 3);
  }
  cp_async_wait<0>();

  // ---- merge the warp's two partial states, then the warps, into the CTA partial ----
  __syncthreads();  // every warp is done with its gather ring, which now holds the merge
  float* wm = reinterpret_cast<float*>(sekv_smem);  // [kSekvWarps][G]
  float* wl = wm + kSekvWarps * G;                   // [kSekvWarps][G]
  float* wo = wl + kSekvWarps * G;                   // [kSekvWarps][G][D]
  float* my = wo + (size_t)warp * G * D;
  float fa0 = 0.f, fa1 = 0.f;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float mA = __shfl_sync(0xffffffffu, (h & 1) ? m1 : m0, h >> 1);
    const float lA = __shfl_sync(0xffffffffu, (h & 1) ? l1 : l0, h >> 1);
    const float M = fmaxf(mA, m[h]);
    const float fA = ex2s(mA - M), fB = ex2s(m[h] - M);
    if (lane == 0) {
      wm[warp * G + h] = M;
      wl[warp * G + h] = lA * fA + l[h] * fB;
    }
#pragma unroll
    for (int j = 0; j < DPL; ++j) my[h * D + lane * DPL + j] = acc[h][j] * fB;
    if (h == h0) fa0 = fA;
    if (h == h1) fa1 = fA;
  }
  __syncwarp();
#pragma unroll
  for (int mm = 0; mm < G8; ++mm) {
    if (h0 < G) {
      my[h0 * D + mm * 16 + g8] += oacc[mm][0] * fa0;
      my[h0 * D + mm * 16 + 8 + g8] += oacc[mm][2] * fa0;
    }
    if (h1 < G) {
      my[h1 * D + mm * 16 + g8] += oacc[mm][1] * fa1;
      my[h1 * D + mm * 16 + 8 + g8] += oacc[mm][3] * fa1;
    }
  }
  __syncthreads();
  for (int x = threadIdx.x; x < G * D; x += blockDim.x) {
    const int h = x / D, d = x % D;
    float M = wm[h];
#pragma unroll
    for (int w = 1; w < kSekvWarps; ++w) M = fmaxf(M, wm[w * G + h]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < kSekvWarps; ++w) {
      const float f = ex2s(wm[w * G + h] - M);
      L = fmaf(wl[w * G + h], f, L);
      O = fmaf(wo[((size_t)w * G + h) * D + d], f, O);
    }
    const size_t pi = ((size_t)u * a.S + split) * G + h;
    a.part_o[pi * D + d] = O;
    if (d == 0) {
      a.part_ml[pi * 2 + 0] = M;
      a.part_ml[pi * 2 + 1] = L;
    }
  }
}

// out[b][kvh*G + h][d] = sum_s O_s 2^(M_s - M) / sum_s L_s 2^(M_s - M); one CTA per (unit, head)
__global__ void sekv_combine_kernel(const float* __restrict__ part_ml, const float* __restrict__ part_o, int S, int G,
                                    int D, int Hq, int Hkv, float* out) {
  const int u = blockIdx.x, h = blockIdx.y, b = u / Hkv, kvh = u % Hkv;
  const size_t p0 = (size_t)u * S * G;
  float M = -1e30f;
  for (int s = 0; s < S; ++s) M = fmaxf(M, part_ml[(p0 + (size_t)s * G + h) * 2]);
  float L = 0.f;
  for (int s = 0; s < S; ++s) {
    const size_t pi = p0 + (size_t)s * G + h;
    L = fmaf(part_ml[pi * 2 + 1], ex2s(part_ml[pi * 2] - M), L);
  }
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float O = 0.f;
    for (int s = 0; s < S; ++s) {
      const size_t pi = p0 + (size_t)s * G + h;
      O = fmaf(part_o[pi * D + d], ex2s(part_ml[pi * 2] - M), O);
    }
    out[((size_t)b * Hq + (size_t)kvh * G + h) * D + d] = L > 0.f ? O / L : 0.f;
  }
}

template <typename T, int DPL>
int launch_build(const void* K, const void* V, const float* H, int B, int Hkv, int n, float tau, uint8_t* st,
                 const SekvLayout& L, cudaStream_t s) {
  int32_t* counts = reinterpret_cast<int32_t*>(st + L.counts);
  int32_t* sst = reinterpret_cast<int32_t*>(st + L.span_start);
  int32_t* sen = reinterpret_cast<int32_t*>(st + L.span_end);
  sekv_segment_kernel<<<B, 1024, 0, s>>>(H, n, tau, L.cap, counts, reinterpret_cast<int32_t*>(st + L.anchor_pos),
                                         sst, sen);
  QE_CUDA_TRY(cudaGetLastError());
  const int ny = (L.cap + kSekvWarps - 1) / kSekvWarps;
  const dim3 grid(B * Hkv, ny < kSekvSpanBlocks ? ny : kSekvSpanBlocks);
  sekv_summarize_kernel<T, DPL><<<grid, kSekvWarps * 32, 0, s>>>(
      static_cast<const T*>(K), static_cast<const T*>(V), H, n, Hkv, L.cap, counts, sst, sen,
      reinterpret_cast<float*>(st + L.kbar), reinterpret_cast<float*>(st + L.vbar));
  QE_CUDA_TRY(cudaGetLastError());
  return QE_OK;
}

template <typename T, int DPL, int G>
int launch_attend(const void* q, const void* K, const void* V, int B, int Hq, int Hkv, int n, float theta,
                  uint8_t* st, const SekvLayout& L, float* out, cudaStream_t s) {
  constexpr int D = 32 * DPL;
  constexpr size_t SMEM = (size_t)kSekvWarps * 2 * (2 * QE_PAGE * D * 2);  // two gather stages per warp
  static_assert((2 + D) * kSekvWarps * G * 4 <= SMEM, "the warp merge fits in the gather rings");
  const int U = B * Hkv;
  // one wave of resident CTAs over the units (found once per instantiation and device)
  static QeOnce once;
  static int resident_of[QE_MAX_DEVICES];
  int dev = 0;
  if (int e = qe_once_per_device(once, &dev, [](int d) {
        QE_CUDA_TRY(cudaFuncSetAttribute(sekv_attend_kernel<T, DPL, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM));
        int sms = 0, per_sm = 0;
        QE_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, d));
        QE_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, sekv_attend_kernel<T, DPL, G>,
                                                                  kSekvWarps * 32, SMEM));
        resident_of[d] = sms * (per_sm > 0 ? per_sm : 1);
        return QE_OK;
      }))
    return e;
  int S = resident_of[dev] / U;
  S = S < 1 ? 1 : (S > kSekvMaxSplits ? kSekvMaxSplits : S);
  const int32_t* counts = reinterpret_cast<const int32_t*>(st + L.counts);
  const float* kbar = reinterpret_cast<const float*>(st + L.kbar);
  uint8_t* expanded = st + L.expanded;
  const int ny = (L.cap + kSekvWarps - 1) / kSekvWarps;
  const dim3 ggrid(U, ny < kSekvSpanBlocks ? ny : kSekvSpanBlocks);
  sekv_gate_kernel<T, DPL, G><<<ggrid, kSekvWarps * 32, 0, s>>>(static_cast<const T*>(q), Hq, Hkv, L.cap, counts,
                                                                kbar, (float)(1.0 / sqrt((double)D)), theta,
                                                                expanded);
  QE_CUDA_TRY(cudaGetLastError());
  int32_t* tok = reinterpret_cast<int32_t*>(st + L.tok);
  int32_t* sums = reinterpret_cast<int32_t*>(st + L.sums);
  int32_t* lcount = reinterpret_cast<int32_t*>(st + L.lcount);
  sekv_lists_kernel<<<U, 1024, 0, s>>>(counts, reinterpret_cast<const int32_t*>(st + L.anchor_pos),
                                       reinterpret_cast<const int32_t*>(st + L.span_start),
                                       reinterpret_cast<const int32_t*>(st + L.span_end), expanded, n, L.cap, Hkv,
                                       tok, sums, lcount);
  QE_CUDA_TRY(cudaGetLastError());
  SekvAttendArgs a{};
  a.tok = tok;
  a.sums = sums;
  a.lcount = lcount;
  a.q = q;
  a.K = K;
  a.V = V;
  a.counts = counts;
  a.anchor_pos = reinterpret_cast<const int32_t*>(st + L.anchor_pos);
  a.span_start = reinterpret_cast<const int32_t*>(st + L.span_start);
  a.span_end = reinterpret_cast<const int32_t*>(st + L.span_end);
  a.kbar = kbar;
  a.vbar = reinterpret_cast<const float*>(st + L.vbar);
  a.expanded = expanded;
  a.part_ml = reinterpret_cast<float*>(st + L.part_ml);
  a.part_o = reinterpret_cast<float*>(st + L.part_o);
  a.n = n;
  a.cap = L.cap;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.S = S;
  a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
  sekv_attend_kernel<T, DPL, G><<<U * S, kSekvWarps * 32, SMEM, s>>>(a);
  QE_CUDA_TRY(cudaGetLastError());
  sekv_combine_kernel<<<dim3(U, G), 128, 0, s>>>(a.part_ml, a.part_o, S, G, D, Hq, Hkv, out);
  QE_CUDA_TRY(cudaGetLastError());
  return QE_OK;
}

template <typename T, int DPL>
int attend_g(int G, const void* q, const void* K, const void* V, int B, int Hq, int Hkv, int n, float theta,
             uint8_t* st, const SekvLayout& L, float* out, cudaStream_t s) {
  switch (G) {
    case 1: return launch_attend<T, DPL, 1>(q, K, V, B, Hq, Hkv, n, theta, st, L, out, s);
    case 2: return launch_attend<T, DPL, 2>(q, K, V, B, Hq, Hkv, n, theta, st, L, out, s);
    case 4: return launch_attend<T, DPL, 4>(q, K, V, B, Hq, Hkv, n, theta, st, L, out, s);
    case 5: return launch_attend<T, DPL, 5>(q, K, V, B, Hq, Hkv, n, theta, st, L, out, s);
    case 8: return launch_attend<T, DPL, 8>(q, K, V, B, Hq, Hkv, n, theta, st, L, out, s);
    default: return QE_ERR_UNSUPPORTED_SHAPE;
  }
}

int check_shape(int B, int Hq, int Hkv, int n, int D, int dtype) {
  if (B < 1 || Hkv < 1 || Hq < 1 || Hq % Hkv || n < 1) return QE_ERR_INVALID_ARG;
  if (dtype != QE_FP16 && dtype != QE_BF16) return QE_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return QE_ERR_UNSUPPORTED_SHAPE;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 5 && G != 8) return QE_ERR_UNSUPPORTED_SHAPE;
  // spans per sequence are at most (n + 1) / 2 and index the second grid dimension (<= 65535 CTAs
  // of kSekvWarps spans)
  if (n > 500000 || (long long)B * n >= (1ll << 31)) return QE_ERR_UNSUPPORTED_SHAPE;
  return QE_OK;
}

}  // namespace

extern "C" QE_API size_t qe_sekv_state_bytes(int B, int Hq, int Hkv, int n, int D) {
  if (check_shape(B, Hq, Hkv, n, D, QE_BF16) != QE_OK) return 0;
  return sekv_layout(B, Hkv, n, D, Hq / Hkv).total;
}

extern "C" QE_API int qe_sekv_state_offsets(int B, int Hq, int Hkv, int n, int D, size_t* offsets) {
  if (!offsets) return QE_ERR_INVALID_ARG;
  if (int e = check_shape(B, Hq, Hkv, n, D, QE_BF16)) return e;
  const SekvLayout L = sekv_layout(B, Hkv, n, D, Hq / Hkv);
  const size_t o[8] = {L.counts, L.anchor_pos, L.span_start, L.span_end, L.kbar, L.vbar, L.expanded,
                       (size_t)L.cap};
  for (int i = 0; i < 8; ++i) offsets[i] = o[i];
  return QE_OK;
}

extern "C" QE_API int qe_sekv_build(const void* K, const void* V, const float* H, int B, int Hq, int Hkv, int n,
                                    int D, int dtype, float tau, void* state, size_t state_bytes,
                                    qe_stream_t stream) {
  if (!K || !V || !H || !state) return QE_ERR_INVALID_ARG;
  if (int e = check_shape(B, Hq, Hkv, n, D, dtype)) return e;
  if (!qe_aligned(K, 16) || !qe_aligned(V, 16) || !qe_aligned(H, 4) || !qe_aligned(state, 256))
    return QE_ERR_INVALID_ARG;
  const SekvLayout L = sekv_layout(B, Hkv, n, D, Hq / Hkv);
  if (state_bytes < L.total) return QE_ERR_WORKSPACE;
  uint8_t* st = static_cast<uint8_t*>(state);
  cudaStream_t s = (cudaStream_t)stream;
  const bool bf = dtype == QE_BF16;
  if (D == 128)
    return bf ? launch_build<__nv_bfloat16, 4>(K, V, H, B, Hkv, n, tau, st, L, s)
              : launch_build<__half, 4>(K, V, H, B, Hkv, n, tau, st, L, s);
  return bf ? launch_build<__nv_bfloat16, 2>(K, V, H, B, Hkv, n, tau, st, L, s)
            : launch_build<__half, 2>(K, V, H, B, Hkv, n, tau, st, L, s);
}

extern "C" QE_API int qe_sekv_attend(const void* q, const void* K, const void* V, int B, int Hq, int Hkv, int n,
                                     int D, int dtype, float theta, void* state, size_t state_bytes, float* out,
                                     qe_stream_t stream) {
  if (!q || !K || !V || !state || !out) return QE_ERR_INVALID_ARG;
  if (int e = check_shape(B, Hq, Hkv, n, D, dtype)) return e;
  if (!qe_aligned(q, 16) || !qe_aligned(K, 16) || !qe_aligned(V, 16) || !qe_aligned(state, 256) ||
      !qe_aligned(out, 4))
    return QE_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  const SekvLayout L = sekv_layout(B, Hkv, n, D, G);
  if (state_bytes < L.total) return QE_ERR_WORKSPACE;
  uint8_t* st = static_cast<uint8_t*>(state);
  cudaStream_t s = (cudaStream_t)stream;
  const bool bf = dtype == QE_BF16;
  if (D == 128)
    return bf ? attend_g<__nv_bfloat16, 4>(G, q, K, V, B, Hq, Hkv, n, theta, st, L, out, s)
              : attend_g<__half, 4>(G, q, K, V, B, Hq, Hkv, n, theta, st, L, out, s);
  return bf ? attend_g<__nv_bfloat16, 2>(G, q, K, V, B, Hq, Hkv, n, theta, st, L, out, s)
            : attend_g<__half, 2>(G, q, K, V, B, Hq, Hkv, n, theta, st, L, out, s);
}
