// Window routing under budgets shared by every layer and kv head of a sequence.
//
// "Make Each Token Count" - Metodologia 3 (Orçamento Global): one budget over all layers and
// heads instead of a fixed share per head, applied here to the window tiers of "Resumo Técnico:
// QEvict" - Metodologia (full / INT2 / evicted), with the two-stage selection of "Resumo
// Técnico: CriticalKV" - Algoritmo (Etapa 1: floor(alpha * b) by attention mass, Etapa 2: the
// rest by the perturbation score).
//
// One routing event: (1) for every layer (one context each) a kernel appends each live window's
// cumulative mass, perturbation and flat position (layer, kv head, window) to its sequence's
// candidate list (a unit claims its range with one atomic add, so the list holds live windows
// only, in no particular order); (2) one thread-block cluster per sequence selects Full = TwoStage(L, F) and
// INT2 = TwoStage(L minus Full, Q) over the list by exact radix selections on 64-bit keys (the
// score's order-preserving bits, then the complement of the flat position, so equal scores go to
// the lower position and the result does not depend on the list order) and writes each chosen
// tier at the window's flat position; (3) each layer's route kernel applies its part - page and
// ledger allocation, write-once quantisation, promotion - exactly as for per-unit routing.
#include <math.h>

#include "qe_internal.cuh"

namespace {

constexpr uint8_t kPick = 2, kFull = 4, kInt2 = 8;

struct GlobArgs {
  float* mass;       // [B][n] candidate list: cumulative attention mass,
  float* pert;       // [B][n] cumulative perturbation score,
  int32_t* pos;      // [B][n] flat position (layer * Hkv + kv head) * max_windows + window,
  uint8_t* flag;     // [B][n] kPick | kFull | kInt2
  int32_t* count;    // [B] list lengths
  uint8_t* decided;  // [B][n] QE_TIER_* by flat position (EVICTED where not chosen)
  int n;             // flat positions per sequence: layers * Hkv * max_windows
};

__device__ __forceinline__ uint32_t order_bits(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// higher score first, then the lower flat position; never 0 for a candidate
__device__ __forceinline__ unsigned long long cand_key(float score, int i) {
  return ((unsigned long long)order_bits(score) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)i);
}

__global__ void glob_keygen_kernel(DevState st, int layer, GlobArgs g) {
  const int u = blockIdx.x;
  const int b = u / st.Hkv, kvh = u % st.Hkv;
  const int nf = st.stacks[u * 4 + 2], nq = st.stacks[u * 4 + 3];
  const size_t ub = (size_t)u * st.Wmax;
  const int pos0 = (layer * st.Hkv + kvh) * st.Wmax;
  // a unit never holds more than max_windows live windows; anything else is a corrupted count
  const bool sane = nf >= 0 && nq >= 0 && nf + nq <= st.Wmax;
  const int cnt = sane ? nf + nq : 0;
  __shared__ int s_base;
  if (threadIdx.x == 0) {
    if (!sane) qe_record_error(st.status, QE_ERR_DEVICE_FAULT, u);
    s_base = atomicAdd(&g.count[b], cnt);
  }
  __syncthreads();
  const size_t base = (size_t)b * g.n + s_base;
  for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
    int win = i < nf ? st.full_list[ub + i] : st.int2_list[ub + i - nf];
    if (win < 0 || win >= st.Wmax) {
      qe_record_error(st.status, QE_ERR_DEVICE_FAULT, u);
      win = 0;  // keeps the list well formed; the status word reports the fault
    }
    g.mass[base + i] = st.mass[ub + win];
    g.pert[base + i] = st.pert[ub + win];
    g.pos[base + i] = pos0 + win;
    g.flag[base + i] = 0;
  }
}

// The selection of one sequence runs on one thread-block cluster of C CTAs (C up to 16): CTA r
// owns the r-th C-th of the candidate list. Every count and radix histogram is formed per CTA in
// shared memory and summed over the cluster through distributed shared memory, so every CTA
// takes the same decisions; flags are read and written only by the CTA that owns the entry.
constexpr int kSelThreadsG = 512;
constexpr int kSelMaxCluster = 16;

struct SelSh {
  unsigned int hist[256];  // this CTA's histogram of the current digit (read by the cluster)
  unsigned int tot[256];   // the cluster's histogram
  int cnt;                 // this CTA's member count (read by the cluster)
  int ctl[3];
  int red[kSelThreadsG / 32];
};

__device__ __forceinline__ void sel_cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t sel_ld_cluster(const uint32_t* local, uint32_t rank) {
  uint32_t a, v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(local)), "r"(rank));
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t sel_cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t sel_cluster_size() {
  uint32_t n;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(n));
  return n;
}

// the cluster-wide sum of v over every thread of every CTA
__device__ int cluster_count(int v, SelSh& sh) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) sh.red[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += sh.red[w];
    sh.cnt = t;
  }
  sel_cluster_sync();
  int t = 0;
  const uint32_t C = sel_cluster_size();
  for (uint32_t r = 0; r < C; ++r) t += (int)sel_ld_cluster(reinterpret_cast<const uint32_t*>(&sh.cnt), r);
  sel_cluster_sync();  // every CTA has read the counts before they change
  return t;
}

// Threshold of the k largest keys over the cluster's entries (1 <= k <= number of non-zero
// keys; non-zero keys distinct): key(i) is among them iff key(i) != 0 and
// (key(i) >> shift) >= (prefix >> shift). Most significant 8-bit digit first; a pass ends the
// search when the digit that holds the k-th key holds exactly the keys still needed. [i0, i1)
// are this CTA's entries.
template <typename KeyFn>
__device__ void topk_threshold(int i0, int i1, int k, KeyFn key, SelSh& sh, unsigned long long* prefix_out,
                               int* shift_out) {
  unsigned long long prefix = 0;
  int shift = 64;
  const uint32_t C = sel_cluster_size();
  for (int pass = 0; pass < 8; ++pass) {
    const int sft = 56 - 8 * pass;
    for (int d = threadIdx.x; d < 256; d += blockDim.x) sh.hist[d] = 0;
    __syncthreads();
    for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) {
      const unsigned long long kk = key(i);
      if (kk != 0 && (shift == 64 || (kk >> shift) == (prefix >> shift)))
        atomicAdd(&sh.hist[(kk >> sft) & 255], 1u);
    }
    sel_cluster_sync();
    for (int d = threadIdx.x; d < 256; d += blockDim.x) {
      uint32_t t = 0;
      for (uint32_t r = 0; r < C; ++r) t += sel_ld_cluster(&sh.hist[d], r);
      sh.tot[d] = t;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane l owns digits 255 - 8l .. 248 - 8l, highest first
      const int l = threadIdx.x;
      uint32_t c[8], loc = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = sh.tot[255 - 8 * l - j];
        loc += c[j];
      }
      uint32_t inc = loc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (l >= o) inc += y;
      }
      long long above = (long long)(inc - loc);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (above < k && above + c[j] >= k) {
          sh.ctl[0] = 255 - 8 * l - j;
          sh.ctl[1] = (int)above;
          sh.ctl[2] = (int)c[j];
        }
        above += c[j];
      }
    }
    __syncthreads();
    k -= sh.ctl[1];
    prefix |= (unsigned long long)sh.ctl[0] << sft;
    shift = sft;
    const bool done = sh.ctl[2] == k;
    sel_cluster_sync();  // every CTA has read the histograms before the next pass clears them
    if (done) break;
  }
  *prefix_out = prefix;
  *shift_out = shift;
}

// TwoStage(members, b) with stage-1 share b1: the chosen candidates get `out` in their flag
template <typename MemberFn>
__device__ void two_stage_global(int i0, int i1, int b, int b1, MemberFn member, const float* mass,
                                 const float* pert, const int32_t* pos, uint8_t* flag, uint8_t out, SelSh& sh) {
  int cnt_local = 0;
  for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) cnt_local += member(i) ? 1 : 0;
  const int cnt = cluster_count(cnt_local, sh);
  if (cnt <= b) {
    for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x)
      if (member(i)) flag[i] |= out;
    __syncthreads();
    return;
  }
  unsigned long long P;
  int S;
  if (b1 > 0) {
    auto k1 = [&](int i) -> unsigned long long { return member(i) ? cand_key(mass[i], pos[i]) : 0ull; };
    topk_threshold(i0, i1, b1, k1, sh, &P, &S);
    for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) {
      const unsigned long long kk = k1(i);
      if (kk != 0 && (kk >> S) >= (P >> S)) flag[i] |= kPick;
    }
    __syncthreads();
  }
  if (b - b1 > 0) {
    auto k2 = [&](int i) -> unsigned long long {
      return (member(i) && !(flag[i] & kPick)) ? cand_key(pert[i], pos[i]) : 0ull;
    };
    topk_threshold(i0, i1, b - b1, k2, sh, &P, &S);
    for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) {
      const unsigned long long kk = k2(i);
      if (kk != 0 && (kk >> S) >= (P >> S)) flag[i] |= out;
    }
    __syncthreads();
  }
  for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x)
    if (flag[i] & kPick) flag[i] = (uint8_t)((flag[i] & ~kPick) | out);
  __syncthreads();
}

// one cluster per sequence: grid = B * C CTAs, cluster size C
__global__ void __launch_bounds__(kSelThreadsG) glob_select_kernel(GlobArgs g, int F, int F1, int Q, int Q1) {
  __shared__ SelSh sh;
  const uint32_t C = sel_cluster_size(), rank = sel_cluster_rank();
  const int seq = blockIdx.x / C;
  const size_t base = (size_t)seq * g.n;
  const float* mass = g.mass + base;
  const float* pert = g.pert + base;
  const int32_t* pos = g.pos + base;
  uint8_t* flag = g.flag + base;
  uint8_t* decided = g.decided + base;
  const int n = g.count[seq];  // the list holds live windows only
  const int i0 = (int)((long long)n * rank / C), i1 = (int)((long long)n * (rank + 1) / C);
  two_stage_global(i0, i1, F, F1, [&](int) { return true; }, mass, pert, pos, flag, kFull, sh);
  two_stage_global(i0, i1, Q, Q1, [&](int i) { return (flag[i] & kFull) == 0; }, mass, pert, pos, flag, kInt2, sh);
  // chosen tiers by flat position (every other position was set to EVICTED beforehand)
  for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) {
    const uint8_t f = flag[i];
    decided[pos[i]] = (f & kFull) ? QE_TIER_FULL : ((f & kInt2) ? QE_TIER_INT2 : QE_TIER_EVICTED);
  }
}

// Cluster size of the selection: the largest C <= 16 whose B clusters can be resident at once
// (all of them, when possible), at least 1. Found once per device.
int glob_select_cluster(int B) {
  static QeOnce once;
  static int resident[QE_MAX_DEVICES][kSelMaxCluster + 1];
  int dev = 0;
  if (qe_once_per_device(once, &dev, [](int d) {
        QE_CUDA_TRY(cudaFuncSetAttribute(glob_select_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
        for (int C = 1; C <= kSelMaxCluster; ++C) {
          cudaLaunchConfig_t qc = {};
          cudaLaunchAttribute qa[1];
          qa[0].id = cudaLaunchAttributeClusterDimension;
          qa[0].val.clusterDim.x = C;
          qa[0].val.clusterDim.y = 1;
          qa[0].val.clusterDim.z = 1;
          qc.gridDim = dim3(C);
          qc.blockDim = dim3(kSelThreadsG);
          qc.attrs = qa;
          qc.numAttrs = 1;
          int nc = 0;
          if (cudaOccupancyMaxActiveClusters(&nc, glob_select_kernel, &qc) != cudaSuccess) {
            (void)cudaGetLastError();
            nc = 0;
          }
          resident[d][C] = nc;
        }
        return QE_OK;
      }) != QE_OK)
    return 1;
  for (int C = kSelMaxCluster; C > 1; --C)
    if (resident[dev][C] >= B) return C;
  for (int C = kSelMaxCluster; C > 1; --C)
    if (resident[dev][C] >= 1) return C;
  return 1;
}

struct GlobLayout {
  size_t mass, pert, pos, flag, count, decided, total;
};

GlobLayout glob_layout(int n_layers, int B, int Hkv, int max_windows) {
  const size_t n = (size_t)n_layers * Hkv * max_windows * B;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  GlobLayout L{};
  L.mass = 0;
  L.pert = up(L.mass + n * 4);
  L.pos = up(L.pert + n * 4);
  L.flag = up(L.pos + n * 4);
  L.count = up(L.flag + n);
  L.decided = up(L.count + (size_t)B * 4);
  L.total = up(L.decided + n);
  return L;
}

}  // namespace

extern "C" QE_API size_t qe_route_global_scratch_bytes(int n_layers, int B, int Hkv, int max_windows) {
  if (n_layers < 1 || B < 1 || Hkv < 1 || max_windows < 1) return 0;
  return glob_layout(n_layers, B, Hkv, max_windows).total;
}

extern "C" QE_API int qe_route_windows_global(qe_ctx* const* ctxs, int n_layers, int full_windows,
                                              int int2_windows, float alpha, void* scratch,
                                              size_t scratch_bytes, qe_stream_t stream) {
  if (!ctxs || n_layers < 1 || !scratch || full_windows < 0 || int2_windows < 0) return QE_ERR_INVALID_ARG;
  if (!(alpha >= 0.f && alpha <= 1.f)) return QE_ERR_INVALID_ARG;
  const qe_ctx* c0 = ctxs[0];
  for (int l = 0; l < n_layers; ++l) {
    const qe_ctx* c = ctxs[l];
    if (!c) return QE_ERR_INVALID_ARG;
    if (!c->loaded) return QE_ERR_STATE;
    if (c->cfg.B != c0->cfg.B || c->cfg.Hkv != c0->cfg.Hkv || c->lay.max_windows != c0->lay.max_windows)
      return QE_ERR_INVALID_ARG;
    for (int m = 0; m < l; ++m)
      if (ctxs[m] == c) return QE_ERR_INVALID_ARG;  // a layer listed twice
  }
  const int B = c0->cfg.B, Hkv = c0->cfg.Hkv, Wmax = c0->lay.max_windows;
  const long long n = (long long)n_layers * Hkv * Wmax;
  if (n * B >= (1ll << 31)) return QE_ERR_UNSUPPORTED_SHAPE;
  const GlobLayout L = glob_layout(n_layers, B, Hkv, Wmax);
  if (!qe_aligned(scratch, 256) || scratch_bytes < L.total) return QE_ERR_WORKSPACE;
  uint8_t* base = static_cast<uint8_t*>(scratch);
  GlobArgs g{};
  g.mass = reinterpret_cast<float*>(base + L.mass);
  g.pert = reinterpret_cast<float*>(base + L.pert);
  g.pos = reinterpret_cast<int32_t*>(base + L.pos);
  g.flag = base + L.flag;
  g.count = reinterpret_cast<int32_t*>(base + L.count);
  g.decided = base + L.decided;
  g.n = (int)n;
  cudaStream_t st = (cudaStream_t)stream;
  const int F1 = (int)floor((double)alpha * full_windows);
  const int Q1 = (int)floor((double)alpha * int2_windows);
  static_assert(QE_TIER_EVICTED == 0, "decided is cleared to EVICTED with a zero fill");
  QE_CUDA_TRY(cudaMemsetAsync(g.count, 0, (size_t)B * 4, st));
  QE_CUDA_TRY(cudaMemsetAsync(g.decided, 0, (size_t)n * B, st));
  for (int l = 0; l < n_layers; ++l) {
    const DevState s = make_state(ctxs[l]);
    glob_keygen_kernel<<<s.U, 256, 0, st>>>(s, l, g);
    QE_CUDA_TRY(cudaGetLastError());
  }
  {
    const int C = glob_select_cluster(B);
    cudaLaunchConfig_t lc = {};
    cudaLaunchAttribute la[1];
    la[0].id = cudaLaunchAttributeClusterDimension;
    la[0].val.clusterDim.x = C;
    la[0].val.clusterDim.y = 1;
    la[0].val.clusterDim.z = 1;
    lc.gridDim = dim3(B * C);
    lc.blockDim = dim3(kSelThreadsG);
    lc.stream = st;
    lc.attrs = la;
    lc.numAttrs = 1;
    QE_CUDA_TRY(cudaLaunchKernelEx(&lc, glob_select_kernel, g, full_windows, F1, int2_windows, Q1));
  }
  for (int l = 0; l < n_layers; ++l) {
    qe_ctx* c = ctxs[l];
    const int e = launch_route_decided(c, g.decided + (size_t)l * Hkv * Wmax, (size_t)n, st);
    if (e) return e;
    // per-unit tier sizes are no longer equal across units: keep upper bounds
    const int tot = c->n_full_max + c->n_int2_max;
    c->n_full_max = tot < full_windows ? tot : full_windows;
    c->n_int2_max = tot < int2_windows ? tot : int2_windows;
    c->counts_exact = 0;
    c->last_stream = st;
  }
  return QE_OK;
}
