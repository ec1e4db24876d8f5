// QEvict diagnostics: selection churn and global latent importance reactivation over
// consecutive tier maps, and the future missed mass of one decode step over a ghost cache.
//
// "Resumo Técnico: QEvict" - Principais Contribuições 1: Massa Perdida Futura (the share of
// future attention that falls on states a policy has already discarded), LIR Global (how often
// windows that left the active set come back to it) and Churn de Seleção (how unstable the
// assignments are between consecutive routing steps).
//
// Tier diagnostics: one CTA per (batch, kv-head) unit walks its windows once per routing
// event, compares the tier with the one it had at the previous event, updates two per-window
// flags (has exited the full tier, has re-entered it) and adds six integer counters.
//
// Future missed mass: the ghost cache holds every token's key at its original precision, so
// the softmax over all tokens so far is the attention the uncompressed model would pay. The
// unit's tokens are split over S CTAs; every warp streams 16-token tiles through its own ring
// of shared-memory stages (128-byte-swizzled TMA boxes, completion on an mbarrier) and forms
// S = Q K^T on the warp-level tensor cores (m16n8k16, the G query rows padded to 16, fp32
// accumulate). Each lane keeps, for its head, the running maximum (log2 domain), the sum of
// weights and the sum of weights of tokens in evicted windows; lanes, warps and finally the S
// CTAs are merged by rescaling to the common maximum. The pass reads each key once: it is
// bound by HBM bandwidth.
#include <math.h>

#include <type_traits>

#include <stdlib.h>

#include "qe_internal.cuh"
#include "tc_common.cuh"
#include "warp_mma.cuh"

namespace {

constexpr int kTierThreads = 256;
constexpr int kFmmWarps = 4;
constexpr int kFmmStages = 4;
constexpr int kFmmMaxSplits = 64;
constexpr size_t kFmmStatusBytes = 256;  // status word at the start of the scratch

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// flags bit 0: the window has left the full tier at some event; bit 1: it has re-entered it
__global__ void __launch_bounds__(kTierThreads)
    tier_diag_kernel(const uint8_t* __restrict__ tiers, uint8_t* __restrict__ prev, uint8_t* __restrict__ flags,
                     int W, int first, long long* __restrict__ counters) {
  const int u = blockIdx.x;
  const size_t base = (size_t)u * W;
  int c[6] = {0, 0, 0, 0, 0, 0};
  for (int w = threadIdx.x; w < W; w += blockDim.x) {
    const int now = tiers[base + w];
    if (first) {
      prev[base + w] = (uint8_t)now;
      flags[base + w] = 0;
      continue;
    }
    const int before = prev[base + w];
    int f = flags[base + w];
    if (before == QE_TIER_FULL || before == QE_TIER_INT2) {
      ++c[0];
      if (now != before) ++c[1];
    }
    if (before == QE_TIER_FULL && now != QE_TIER_FULL) {
      ++c[2];
      if (!(f & 1)) {
        ++c[4];
        f |= 1;
      }
    } else if (before != QE_TIER_FULL && now == QE_TIER_FULL && (f & 1)) {
      ++c[3];
      if (!(f & 2)) {
        ++c[5];
        f |= 2;
      }
    }
    prev[base + w] = (uint8_t)now;
    flags[base + w] = (uint8_t)f;
  }
  if (first) return;  // uniform over the block
  __shared__ int red[6][kTierThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 0; k < 6; ++k) {
    const int v = warp_sum_i(c[k]);
    if (lane == 0) red[k][warp] = v;
  }
  __syncthreads();
  if (threadIdx.x < 6) {
    long long s = 0;
    for (int x = 0; x < (int)(blockDim.x / 32); ++x) s += red[threadIdx.x][x];
    counters[(size_t)u * 6 + threadIdx.x] += s;
  }
}

struct FmmArgs {
  const void* q;          // [B][Hq][D]
  const uint8_t* tiers;   // [U][W]
  float4* part;           // [U][S][G]: (max log2, sum of weights, sum over evicted, 0)
  int32_t* status;
  long long n_stride;     // rows per unit in the ghost cache
  int n, W, window, Hq, Hkv, S;
  float scale_log2;       // log2(e) / sqrt(D)
};

template <int D>
struct FmmStage {
  static constexpr int BYTES = 16 * D * 2;  // one tile: 16 keys (1024-byte multiple)
  static constexpr size_t SMEM = 1024 + (size_t)kFmmWarps * kFmmStages * BYTES + kFmmWarps * kFmmStages * 8;
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(kFmmWarps * 32)
    fmm_partial_kernel(const __grid_constant__ CUtensorMap tmK, FmmArgs a) {
  constexpr int STAGE = FmmStage<D>::BYTES;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ float4 red[kFmmWarps][QE_MAX_G];
  const int u = blockIdx.x / a.S, split = blockIdx.x % a.S;
  const int b = u / a.Hkv, kvh = u % a.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int n_tiles = (a.n + 15) / 16;
  const int t0 = (int)((long long)n_tiles * split / a.S), t1 = (int)((long long)n_tiles * (split + 1) / a.S);
  // this warp's tiles: t0 + warp + kFmmWarps * r for r < n_own
  const int n_own = t1 - t0 > warp ? (t1 - t0 - warp + kFmmWarps - 1) / kFmmWarps : 0;
  uint8_t* ring = smem + warp * kFmmStages * STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kFmmWarps * kFmmStages * STAGE) + warp * kFmmStages;
  if (lane == 0) {
    for (int s = 0; s < kFmmStages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();

  // A operand: row g8 = query head g8 of the group (rows >= G and 8..15 are zero)
  uint32_t qa[D / 16][2];
  {
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
        reinterpret_cast<const T*>(a.q) + ((size_t)b * a.Hq + (size_t)kvh * G + (g8 < G ? g8 : 0)) * D);
#pragma unroll
    for (int kc = 0; kc < D / 16; ++kc) {
      qa[kc][0] = g8 < G ? qrow[kc * 8 + t4] : 0u;
      qa[kc][1] = g8 < G ? qrow[kc * 8 + 4 + t4] : 0u;
    }
  }
  const long long row_base = (long long)u * a.n_stride;
  auto issue = [&](int r) {
    const int s = r % kFmmStages;
    fence_proxy_async_smem();
    if (lane == 0) {
      const int tile = t0 + warp + kFmmWarps * r;
      mbar_arrive_expect_tx(&bars[s], STAGE);
#pragma unroll
      for (int xb = 0; xb < D / 64; ++xb)
        tc::tma_load_2d(ring + s * STAGE + xb * 2048, &tmK, xb * 64, (int)(row_base + (long long)tile * 16), &bars[s]);
    }
  };

  float mh = -1e30f, lh = 0.f, eh = 0.f;  // head g8: running max (log2), sums
  int issued = 0, r = 0;
  for (; issued < kFmmStages - 1 && issued < n_own; ++issued) issue(issued);
  bool ok = true;
  const uint8_t* tier_u = a.tiers + (size_t)u * a.W;
  for (; r < n_own; ++r) {
    if (issued < n_own) issue(issued++);
    const int s = r % kFmmStages;
    ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[s], (r / kFmmStages) & 1, a.status, 3000 + u));
    if (!ok) break;
    const uint8_t* stage = ring + s * STAGE;
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
    __syncwarp();
    // lane (g8, t4) holds head g8's scores of tokens 2t4, 2t4+1, 8+2t4, 9+2t4 of the tile.
    // With windows of at least 16 tokens a tile meets at most two windows: one division and
    // two tier loads per tile (shorter windows take one division per token).
    const int tile0 = (t0 + warp + kFmmWarps * r) * 16;
    const int tok0 = tile0 + 2 * t4;
    int w0 = 0, wb = 0;
    bool e0 = false, e1 = false;
    if (a.window >= 16) {
      w0 = tile0 / a.window;
      wb = (w0 + 1) * a.window;  // first token of the next window
      e0 = tier_u[w0] == QE_TIER_EVICTED;
      e1 = wb < a.n && tier_u[w0 + 1] == QE_TIER_EVICTED;
    }
    float sc[4] = {c0[0], c0[1], c1[0], c1[1]};
    bool ev[4];
    float mx = -1e30f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int tok = tok0 + (i & 1) + (i >> 1) * 8;
      const bool valid = tok < a.n;
      sc[i] = valid ? sc[i] * a.scale_log2 : -INFINITY;
      if (a.window >= 16)
        ev[i] = valid && (tok < wb ? e0 : e1);
      else
        ev[i] = valid && tier_u[tok / a.window] == QE_TIER_EVICTED;
      mx = fmaxf(mx, sc[i]);
    }
    if (mx > mh) {
      const float f = ex2f(mh - mx);
      lh *= f;
      eh *= f;
      mh = mx;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float p = ex2f(sc[i] - mh);
      lh += p;
      eh += ev[i] ? p : 0.f;
    }
  }
  if (!ok) {  // let the copies still in flight land before the CTA exits
    for (; r < issued; ++r) mbar_wait_bounded(&bars[r % kFmmStages], (r / kFmmStages) & 1, a.status, 4000 + u);
  }
  // merge the four lanes of a head, then the warps
#pragma unroll
  for (int o = 1; o < 4; o <<= 1) {
    const float om = __shfl_xor_sync(0xffffffffu, mh, o);
    const float ol = __shfl_xor_sync(0xffffffffu, lh, o);
    const float oe = __shfl_xor_sync(0xffffffffu, eh, o);
    const float M = fmaxf(mh, om);
    const float fa = ex2f(mh - M), fb = ex2f(om - M);
    lh = lh * fa + ol * fb;
    eh = eh * fa + oe * fb;
    mh = M;
  }
  if (t4 == 0 && g8 < G) red[warp][g8] = make_float4(mh, lh, eh, 0.f);
  __syncthreads();
  if (threadIdx.x < G) {
    const int h = threadIdx.x;
    float M = red[0][h].x;
#pragma unroll
    for (int x = 1; x < kFmmWarps; ++x) M = fmaxf(M, red[x][h].x);
    float L = 0.f, E = 0.f;
#pragma unroll
    for (int x = 0; x < kFmmWarps; ++x) {
      const float f = ex2f(red[x][h].x - M);
      L = fmaf(red[x][h].y, f, L);
      E = fmaf(red[x][h].z, f, E);
    }
    a.part[((size_t)u * a.S + split) * G + h] = make_float4(M, L, E, 0.f);
  }
}

// fmm[u] = (1/G) sum_h E_h / L_h over the S partials of unit u (0 for a head with no tokens)
__global__ void fmm_combine_kernel(const float4* __restrict__ part, int S, int G, float* __restrict__ fmm) {
  const int u = blockIdx.x, h = threadIdx.x;
  float f = 0.f;
  if (h < G) {
    float M = -1e30f;
    for (int s = 0; s < S; ++s) M = fmaxf(M, part[((size_t)u * S + s) * G + h].x);
    float L = 0.f, E = 0.f;
    for (int s = 0; s < S; ++s) {
      const float4 p = part[((size_t)u * S + s) * G + h];
      const float w = ex2f(p.x - M);
      L = fmaf(p.y, w, L);
      E = fmaf(p.z, w, E);
    }
    f = L > 0.f ? E / L : 0.f;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) f += __shfl_xor_sync(0xffffffffu, f, o);
  if (h == 0) fmm[u] = f / (float)G;
}

size_t fmm_scratch_bytes(int units, int G) {
  return kFmmStatusBytes + (size_t)units * kFmmMaxSplits * G * sizeof(float4);
}

template <typename T, int D, int G>
int launch_fmm(const void* q, const void* K, long long n_stride, int n, const uint8_t* tiers, int W, int window,
               int B, int Hq, int Hkv, float* fmm, uint8_t* scratch, cudaStream_t st) {
  constexpr size_t SMEM = FmmStage<D>::SMEM;
  auto kern = fmm_partial_kernel<T, D, G>;
  static QeOnce once;
  static int slots_of[QE_MAX_DEVICES];  // resident CTAs per device
  int dev = 0;
  int e = qe_once_per_device(once, &dev, [&](int d) {
    QE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM));
    int per_sm = 0, sms = 0;
    QE_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFmmWarps * 32, SMEM));
    QE_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, d));
    slots_of[d] = per_sm * sms > 0 ? per_sm * sms : 1;
    return QE_OK;
  });
  if (e) return e;
  const int U = B * Hkv;
  const long long rows = (long long)U * n_stride;
  CUtensorMap tm;
  e = tc::make_map(&tm, K, std::is_same<T, __nv_bfloat16>::value, D, (uint64_t)(rows > 0 ? rows : 1), 64, 16);
  if (e) return e;
  // as many splits as keep every CTA in one wave of resident slots (a second, partial wave
  // would double the pass), never more than the unit's tiles allow
  const int tiles = (n + 15) / 16;
  int S = slots_of[dev] / U;
  const int cap = (tiles + kFmmWarps - 1) / kFmmWarps;
  if (S > cap) S = cap;
  if (S > kFmmMaxSplits) S = kFmmMaxSplits;
  if (S < 1) S = 1;
  FmmArgs a{};
  a.q = q;
  a.tiers = tiers;
  a.part = reinterpret_cast<float4*>(scratch + kFmmStatusBytes);
  a.status = reinterpret_cast<int32_t*>(scratch);
  a.n_stride = n_stride;
  a.n = n;
  a.W = W;
  a.window = window;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.S = S;
  a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
  QE_CUDA_TRY(cudaMemsetAsync(scratch, 0, 8, st));
  fmm_partial_kernel<T, D, G><<<U * S, kFmmWarps * 32, SMEM, st>>>(tm, a);
  QE_CUDA_TRY(cudaGetLastError());
  fmm_combine_kernel<<<U, 32, 0, st>>>(a.part, S, G, fmm);
  QE_CUDA_TRY(cudaGetLastError());
  return QE_OK;
}

template <typename T, int D>
int launch_fmm_g(int G, const void* q, const void* K, long long ns, int n, const uint8_t* tiers, int W, int w, int B,
                 int Hq, int Hkv, float* fmm, uint8_t* scratch, cudaStream_t st) {
  switch (G) {
    case 1: return launch_fmm<T, D, 1>(q, K, ns, n, tiers, W, w, B, Hq, Hkv, fmm, scratch, st);
    case 2: return launch_fmm<T, D, 2>(q, K, ns, n, tiers, W, w, B, Hq, Hkv, fmm, scratch, st);
    case 4: return launch_fmm<T, D, 4>(q, K, ns, n, tiers, W, w, B, Hq, Hkv, fmm, scratch, st);
    case 5: return launch_fmm<T, D, 5>(q, K, ns, n, tiers, W, w, B, Hq, Hkv, fmm, scratch, st);
    case 8: return launch_fmm<T, D, 8>(q, K, ns, n, tiers, W, w, B, Hq, Hkv, fmm, scratch, st);
    default: return QE_ERR_UNSUPPORTED_SHAPE;
  }
}

}  // namespace

extern "C" QE_API int qe_diag_tiers(const uint8_t* tiers, uint8_t* prev, uint8_t* flags, int units, int W,
                                    int first, long long* counters, qe_stream_t stream) {
  if (!tiers || !prev || !flags || (!counters && !first) || units <= 0 || W <= 0) return QE_ERR_INVALID_ARG;
  tier_diag_kernel<<<units, kTierThreads, 0, (cudaStream_t)stream>>>(tiers, prev, flags, W, first ? 1 : 0,
                                                                    counters);
  return cudaGetLastError() == cudaSuccess ? QE_OK : QE_ERR_CUDA;
}

extern "C" QE_API int qe_diag_summary(const long long* counters, int units, qe_diag_stats* out,
                                      qe_stream_t s) {
  if (!counters || !out || units < 1) return QE_ERR_INVALID_ARG;
  long long* h = (long long*)malloc(sizeof(long long) * 6 * (size_t)units);
  if (!h) return QE_ERR_INVALID_ARG;
  const bool okc = cudaMemcpyAsync(h, counters, sizeof(long long) * 6 * (size_t)units, cudaMemcpyDeviceToHost,
                                   (cudaStream_t)s) == cudaSuccess &&
                   cudaStreamSynchronize((cudaStream_t)s) == cudaSuccess;
  if (!okc) {
    free(h);
    return QE_ERR_CUDA;
  }
  long long sum[6] = {0, 0, 0, 0, 0, 0};
  for (int u = 0; u < units; ++u)
    for (int i = 0; i < 6; ++i) sum[i] += h[(size_t)u * 6 + i];
  free(h);
  out->live_prev = sum[0];
  out->changed = sum[1];
  out->exits = sum[2];
  out->reentries = sum[3];
  out->windows_exited = sum[4];
  out->windows_reentered = sum[5];
  out->churn = sum[0] ? (double)sum[1] / (double)sum[0] : NAN;
  out->lir = sum[4] ? (double)sum[5] / (double)sum[4] : NAN;
  return QE_OK;
}

extern "C" QE_API size_t qe_diag_fmm_scratch_bytes(int units, int G) {
  if (units <= 0 || G <= 0 || G > QE_MAX_G) return 0;
  return fmm_scratch_bytes(units, G);
}

extern "C" QE_API int qe_diag_fmm(const void* q, const void* K_ghost, long long n_stride, int n,
                                  const uint8_t* tiers, int W, int window, int B, int Hq, int Hkv, int D,
                                  int dtype, float* fmm_out, void* scratch, size_t scratch_bytes,
                                  qe_stream_t stream) {
  if (!q || !K_ghost || !tiers || !fmm_out || !scratch) return QE_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || Hq <= 0 || Hq % Hkv || n < 0 || window <= 0 || W <= 0 || n_stride < n || n_stride < 1)
    return QE_ERR_INVALID_ARG;
  if (dtype != QE_FP16 && dtype != QE_BF16) return QE_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if (D != 64 && D != 128) return QE_ERR_UNSUPPORTED_SHAPE;
  if (((long long)n + window - 1) / window > W) return QE_ERR_INVALID_ARG;
  if ((long long)B * Hkv * n_stride + 16 >= (1ll << 31)) return QE_ERR_UNSUPPORTED_SHAPE;
  if (!qe_aligned(K_ghost, 16) || !qe_aligned(q, 4) || !qe_aligned(fmm_out, 4) || !qe_aligned(scratch, 16))
    return QE_ERR_INVALID_ARG;
  if (G > QE_MAX_G || scratch_bytes < fmm_scratch_bytes(B * Hkv, G)) return QE_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  uint8_t* sc = static_cast<uint8_t*>(scratch);
  const bool bf = dtype == QE_BF16;
  if (D == 128)
    return bf ? launch_fmm_g<__nv_bfloat16, 128>(G, q, K_ghost, n_stride, n, tiers, W, window, B, Hq, Hkv, fmm_out, sc, st)
              : launch_fmm_g<__half, 128>(G, q, K_ghost, n_stride, n, tiers, W, window, B, Hq, Hkv, fmm_out, sc, st);
  return bf ? launch_fmm_g<__nv_bfloat16, 64>(G, q, K_ghost, n_stride, n, tiers, W, window, B, Hq, Hkv, fmm_out, sc, st)
            : launch_fmm_g<__half, 64>(G, q, K_ghost, n_stride, n, tiers, W, window, B, Hq, Hkv, fmm_out, sc, st);
}
