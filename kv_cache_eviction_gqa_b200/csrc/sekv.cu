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

namespace {

constexpr int kSekvWarps = 4;      // warps per CTA (gate, summarize, attend)
constexpr int kSekvMaxSplits = 32;
constexpr int kSekvTargetCtas = 1184;  // 148 SMs x 8
constexpr int kSekvSpanBlocks = 64;    // CTAs per unit for the per-span kernels (grid-stride over spans)

struct SekvLayout {
  size_t counts, anchor_pos, span_start, span_end, kbar, vbar, expanded, part_ml, part_o, total;
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
  L.total = up(L.part_o + U * kSekvMaxSplits * G * (size_t)D * 4);
  return L;
}

int sekv_splits(int U) {
  int S = (kSekvTargetCtas + U - 1) / U;
  return S < 1 ? 1 : (S > kSekvMaxSplits ? kSekvMaxSplits : S);
}

__device__ __forceinline__ float ex2s(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float warp_allsum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
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

// one warp per (kv head, span): expanded = max_h q_h . kbar / sqrt(D) >= theta
template <typename T, int DPL, int G>
__global__ void __launch_bounds__(kSekvWarps * 32)
    sekv_gate_kernel(const T* __restrict__ q, int Hq, int Hkv, int cap, const int32_t* counts,
                     const float* __restrict__ kbar, float scale, float theta, uint8_t* expanded) {
  constexpr int D = 32 * DPL;
  const int u = blockIdx.x, b = u / Hkv, kvh = u % Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nspans = counts[b * 2 + 1];
  float qx[G][DPL];
#pragma unroll
  for (int h = 0; h < G; ++h) load_dims<T, DPL>(q + ((size_t)b * Hq + (size_t)kvh * G + h) * D, lane, qx[h]);
  for (int i = blockIdx.y * kSekvWarps + warp; i < nspans; i += gridDim.y * kSekvWarps) {
    const float* kr = kbar + ((size_t)u * cap + i) * D + lane * DPL;
    float g = -INFINITY;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float d = 0.f;
#pragma unroll
      for (int j = 0; j < DPL; ++j) d = fmaf(qx[h][j], kr[j], d);
      g = fmaxf(g, warp_allsum(d) * scale);
    }
    if (lane == 0) expanded[(size_t)u * cap + i] = g >= theta ? 1 : 0;
  }
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
  int n, cap, Hq, Hkv, S;
  float scale_log2;
};

template <typename T, int DPL, int G>
__global__ void __launch_bounds__(kSekvWarps * 32) sekv_attend_kernel(SekvAttendArgs a) {
  constexpr int D = 32 * DPL;
  const int u = blockIdx.x / a.S, split = blockIdx.x % a.S;
  const int b = u / a.Hkv, kvh = u % a.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int A = a.counts[b * 2 + 0], NS = a.counts[b * 2 + 1], I = A + NS;
  const int i0 = (int)((long long)I * split / a.S), i1 = (int)((long long)I * (split + 1) / a.S);
  const T* Kb = reinterpret_cast<const T*>(a.K) + (size_t)u * a.n * D;
  const T* Vb = reinterpret_cast<const T*>(a.V) + (size_t)u * a.n * D;
  float qv[G][DPL];
#pragma unroll
  for (int h = 0; h < G; ++h)
    load_dims<T, DPL>(reinterpret_cast<const T*>(a.q) + ((size_t)b * a.Hq + (size_t)kvh * G + h) * D, lane, qv[h]);
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
    // reduce-scatter: at the level of partner distance o the lane keeps the lower or upper half
    // of its block (by bit o of its lane index) and adds the partner's copy of that half
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
    // all-gather, the same levels in reverse: blocks double until every lane holds all NP sums
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
  auto clear_slot = [&](float (&kx)[DPL], float (&vx)[DPL], float& bias) {
#pragma unroll
    for (int j = 0; j < DPL; ++j) kx[j] = vx[j] = 0.f;
    bias = -INFINITY;
  };
  // pass 1: the single-key items (anchors, summaries of spans that are not expanded), KB of
  // the warp's items per batch
  for (int base = i0 + warp; base < i1; base += KB * kSekvWarps) {
    float kx[KB][DPL], vx[KB][DPL], bias[KB];
#pragma unroll
    for (int k = 0; k < KB; ++k) {
      clear_slot(kx[k], vx[k], bias[k]);
      const int it = base + k * kSekvWarps;
      if (it >= i1) continue;
      if (it < A) {
        const int t = a.anchor_pos[(size_t)b * a.n + it];
        load_dims<T, DPL>(Kb + (size_t)t * D, lane, kx[k]);
        load_dims<T, DPL>(Vb + (size_t)t * D, lane, vx[k]);
        bias[k] = 0.f;
      } else {
        const int i = it - A;
        if (a.expanded[(size_t)u * a.cap + i]) continue;
        const int s = a.span_start[(size_t)b * a.cap + i], e = a.span_end[(size_t)b * a.cap + i];
        const float* kr = a.kbar + ((size_t)u * a.cap + i) * D + lane * DPL;
        const float* vr = a.vbar + ((size_t)u * a.cap + i) * D + lane * DPL;
#pragma unroll
        for (int j = 0; j < DPL; ++j) {
          kx[k][j] = kr[j];
          vx[k][j] = vr[j];
        }
        bias[k] = log2f((float)(e - s));  // the summary stands for e - s tokens
      }
    }
    take_batch(kx, vx, bias);
  }
  // pass 2: the tokens of the warp's expanded spans, KB per batch
  for (int it = i0 + warp; it < i1; it += kSekvWarps) {
    if (it < A) continue;
    const int i = it - A;
    if (!a.expanded[(size_t)u * a.cap + i]) continue;
    const int s = a.span_start[(size_t)b * a.cap + i], e = a.span_end[(size_t)b * a.cap + i];
    for (int t0 = s; t0 < e; t0 += KB) {
      float kx[KB][DPL], vx[KB][DPL], bias[KB];
#pragma unroll
      for (int k = 0; k < KB; ++k) {
        clear_slot(kx[k], vx[k], bias[k]);
        if (t0 + k < e) {
          load_dims<T, DPL>(Kb + (size_t)(t0 + k) * D, lane, kx[k]);
          load_dims<T, DPL>(Vb + (size_t)(t0 + k) * D, lane, vx[k]);
          bias[k] = 0.f;
        }
      }
      take_batch(kx, vx, bias);
    }
  }
  // merge the warps into the CTA partial
  __shared__ float wm[kSekvWarps][G], wl[kSekvWarps][G];
  __shared__ float wo[kSekvWarps][G][D];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    if (lane == 0) {
      wm[warp][h] = m[h];
      wl[warp][h] = l[h];
    }
#pragma unroll
    for (int j = 0; j < DPL; ++j) wo[warp][h][lane * DPL + j] = acc[h][j];
  }
  __syncthreads();
  for (int x = threadIdx.x; x < G * D; x += blockDim.x) {
    const int h = x / D, d = x % D;
    float M = wm[0][h];
#pragma unroll
    for (int w = 1; w < kSekvWarps; ++w) M = fmaxf(M, wm[w][h]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < kSekvWarps; ++w) {
      const float f = ex2s(wm[w][h] - M);
      L = fmaf(wl[w][h], f, L);
      O = fmaf(wo[w][h][d], f, O);
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
  const int U = B * Hkv, S = sekv_splits(U);
  const int32_t* counts = reinterpret_cast<const int32_t*>(st + L.counts);
  const float* kbar = reinterpret_cast<const float*>(st + L.kbar);
  uint8_t* expanded = st + L.expanded;
  const int ny = (L.cap + kSekvWarps - 1) / kSekvWarps;
  const dim3 ggrid(U, ny < kSekvSpanBlocks ? ny : kSekvSpanBlocks);
  sekv_gate_kernel<T, DPL, G><<<ggrid, kSekvWarps * 32, 0, s>>>(static_cast<const T*>(q), Hq, Hkv, L.cap, counts,
                                                                kbar, (float)(1.0 / sqrt((double)D)), theta,
                                                                expanded);
  QE_CUDA_TRY(cudaGetLastError());
  SekvAttendArgs a{};
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
  sekv_attend_kernel<T, DPL, G><<<U * S, kSekvWarps * 32, 0, s>>>(a);
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
