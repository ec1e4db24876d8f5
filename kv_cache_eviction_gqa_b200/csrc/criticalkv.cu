// CriticalKV with a SnapKV-style observation window ("Resumo Técnico: CriticalKV", Algoritmo;
// Framework Teórico for the projected-value norms).
//
// Per unit (batch b, kv head kvh) with G query heads, n keys and the last n_obs positions as
// observation queries q_(h,j) (query j sits at position n - n_obs + j and sees keys 0..that):
//   A[h][i] = sum_j softmax_i(q_(h,j) . K / sqrt(D))                    (attention mass)
//   N[i][h] = || V_i W_O^h ||_1                                         (projected-value norm)
//   a_i = sum_h A[h][i],  p_i = sum_h A[h][i] N[i][h]
// and the budget b is filled in two stages: floor(alpha b) entries of highest a, then the
// rest of highest p among the others (ties to the lower index).
//
// The R = G n_obs query rows of a unit form a 128-row tensor-core tile, so S = Q K^T runs
// on tcgen05 twice over the keys:
//   pass 1 (obs_stats): A operand Q (query rows in TMEM lanes), B operand a 128-key tile;
//           each epilogue thread keeps its row's running max m and sum l of exp2(s c - m)
//           over its columns (c = log2(e)/sqrt(D)); splits of the key range write partials.
//   combine:          bias_r = m_r + log2(l_r) over the splits.
//   pass 2 (obs_mass): A operand the key tile (keys in TMEM lanes), B operand Q; a thread
//           owns one key and a 64-column half of the query rows (one head per 32-column
//           chunk when n_obs = 32, one head per half when n_obs = 64), and writes
//           A[h][key] = sum_j exp2(s c - bias_(h,j)) directly.
// Warp roles in both passes: warp 0 issues TMA loads (Q once, key tiles through a 2-stage
// ring), warp 1 owns TMEM (2 x 128 columns) and issues tcgen05.mma (M = N = 128, K = 16),
// warps 2-9 are the epilogue (lane quarter = warp % 4, column half = (warp - 2) / 4).
// Two CTAs share an SM. The selection then runs one CTA per unit: 64-bit keys
// (score bits, complemented index) go through an 8-bit radix select and a bitonic sort.
#include "tc_common.cuh"

namespace {

using namespace tc;

constexpr int kTile = 128;             // keys per tile
constexpr int kRows = 128;             // query rows per unit, padded
constexpr int kNST = 2;                // key-tile stages
constexpr int kEpiWarps = 8;
constexpr int kThreads = (2 + kEpiWarps) * 32;
constexpr int kTmemCols = 2 * kTile;   // two accumulator buffers of 128 columns
constexpr int kMaxSplits = 64;
constexpr int kMaxBudget = 8192;
constexpr int kSelThreads = 1024;

struct ObsArgs {
  int n, n_obs, R, G, Hq, Hkv, splits, tiles;
  float cs;                            // log2(e) / sqrt(D)
  float2* part;                        // [units][kMaxSplits][kRows] (m, l) of pass 1
  const float* bias;                   // [units][kRows]
  float* A;                            // [units][G][n]
  int32_t* status;
};

template <int D>
struct ObsSmem {
  static constexpr int KB = D / 64;                 // 64-element (128-byte) K boxes
  static constexpr int BOX = 128 * 128;             // 128 rows x 128 bytes
  static constexpr int FIX = KB * BOX;              // Q: 128 rows x D
  static constexpr int STAGE = KB * BOX;            // key tile: 128 rows x D
  static constexpr int BYTES = 1024 + FIX + kNST * STAGE + kRows * 4 + kRows * 8 + 256;
};

template <int D, bool BF16, int PASS>
__global__ void __launch_bounds__(kThreads, 2)
    obs_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, ObsArgs a) {
  using S = ObsSmem<D>;
  constexpr uint32_t IDESC = idesc_f16(BF16, false, 128, 128);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sFix = smem;
  uint8_t* sStage = smem + S::FIX;
  float* sBias = reinterpret_cast<float*>(sStage + kNST * S::STAGE);
  float2* sXch = reinterpret_cast<float2*>(sBias + kRows);
  uint64_t* full = reinterpret_cast<uint64_t*>(sXch + kRows);
  uint64_t* empty = full + kNST;
  uint64_t* accf = empty + kNST;
  uint64_t* acce = accf + 2;
  uint64_t* fixfull = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fixfull + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x % a.splits, u = blockIdx.x / a.splits;
  const int t0 = (int)((long long)a.tiles * split / a.splits);
  const int t1 = (int)((long long)a.tiles * (split + 1) / a.splits);
  const int NT = t1 - t0;
  const int qrow0 = ((u / a.Hkv) * a.Hq + (u % a.Hkv) * a.G) * a.n_obs;
  const int krow0 = u * a.n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], kEpiWarps);
    }
    mbar_init(fixfull, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (PASS == 2 && threadIdx.x < kRows) sBias[threadIdx.x] = a.bias[(size_t)u * kRows + threadIdx.x];
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(fixfull, S::FIX);
      for (int kb = 0; kb < S::KB; ++kb) tma_load_2d(sFix + kb * S::BOX, &tmQ, kb * 64, qrow0, fixfull);
      for (int i = 0; i < NT; ++i) {
        const int s = i % kNST;
        if (!wait_or_abort(&empty[s], ((i / kNST) & 1) ^ 1, abort_flag, a.status, 4001)) break;
        mbar_arrive_expect_tx(&full[s], S::STAGE);
        const int row = krow0 + (t0 + i) * kTile;
        for (int kb = 0; kb < S::KB; ++kb)
          tma_load_2d(sStage + s * S::STAGE + kb * S::BOX, &tmK, kb * 64, row, &full[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && wait_or_abort(fixfull, 0, abort_flag, a.status, 4002)) {
      tc_fence_after();
      for (int i = 0; i < NT; ++i) {
        const int s = i % kNST, b = i & 1;
        if (!wait_or_abort(&full[s], (i / kNST) & 1, abort_flag, a.status, 4003)) break;
        if (!wait_or_abort(&acce[b], ((i >> 1) & 1) ^ 1, abort_flag, a.status, 4004)) break;
        tc_fence_after();
        const uint8_t* opA = PASS == 1 ? sFix : sStage + s * S::STAGE;
        const uint8_t* opB = PASS == 1 ? sStage + s * S::STAGE : sFix;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k / 4) * S::BOX + (k % 4) * 32;
          mma_f16(tmem + (uint32_t)(b * kTile), sdesc(smem_u32(opA + off), 16, 1024),
                  sdesc(smem_u32(opB + off), 16, 1024), IDESC, k > 0 ? 1u : 0u);
        }
        mma_commit(&empty[s]);
        mma_commit(&accf[b]);
      }
    }
  } else {
    const int q = warp & 3, hf = (warp - 2) >> 2;
    const int lim0 = a.n - a.n_obs;     // last key every observation query sees
    float m = -1e30f, l = 0.f;          // pass 1 running stats of row 32q + lane
    for (int i = 0; i < NT; ++i) {
      const int b = i & 1;
      if (!__all_sync(0xffffffffu, wait_or_abort(&accf[b], (i >> 1) & 1, abort_flag, a.status, 4005))) break;
      tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * kTile + hf * 64);
      float x0[32], x1[32];
      tmem_ld32(taddr, x0);
      tmem_ld32(taddr + 32, x1);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[b]);
      const int tile_key0 = (t0 + i) * kTile;
      if (PASS == 1) {
        // row r = 32q + lane sees keys up to lim0 + (r % n_obs); columns are keys
        const int key0 = tile_key0 + hf * 64;
        if (key0 + 63 > lim0) {
          const int lim = lim0 + (q * 32 + lane) % a.n_obs;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            if (key0 + c > lim) x0[c] = -INFINITY;
            if (key0 + 32 + c > lim) x1[c] = -INFINITY;
          }
        }
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 32; ++c) mx = fmaxf(mx, fmaxf(x0[c], x1[c]));
        const float mn = fmaxf(m, mx * a.cs);
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          acc.x += exp2f(fmaf(x0[c], a.cs, -mn)) + exp2f(fmaf(x1[c], a.cs, -mn));
          acc.y += exp2f(fmaf(x0[c + 1], a.cs, -mn)) + exp2f(fmaf(x1[c + 1], a.cs, -mn));
        }
        l = l * exp2f(m - mn) + (acc.x + acc.y);
        m = mn;
      } else {
        // this thread's key; columns hf*64 + 32c + jj are query rows (one head per chunk)
        const int key = tile_key0 + q * 32 + lane;
        const bool open = tile_key0 + kTile - 1 <= lim0;  // every query sees every key of the tile
        // sum over the 32 query rows of chunk c (0 when the chunk is padding)
        auto chunk = [&](const float(&x)[32], int c) -> float {
          const int rb = hf * 64 + c * 32;
          if (rb >= a.R) return 0.f;
          const float4* bb = reinterpret_cast<const float4*>(sBias + rb);
          float2 acc = make_float2(0.f, 0.f);
          if (open) {
#pragma unroll
            for (int jj = 0; jj < 32; jj += 4) {
              const float4 bv = bb[jj / 4];
              acc.x += exp2f(fmaf(x[jj], a.cs, -bv.x)) + exp2f(fmaf(x[jj + 2], a.cs, -bv.z));
              acc.y += exp2f(fmaf(x[jj + 1], a.cs, -bv.y)) + exp2f(fmaf(x[jj + 3], a.cs, -bv.w));
            }
          } else {
            const int need_j = key - lim0 - rb % a.n_obs;  // query jb + jj sees the key iff jj >= need_j
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
              const float e = exp2f(fmaf(x[jj], a.cs, -sBias[rb + jj]));
              if (jj >= need_j) acc.x += e;
            }
          }
          return acc.x + acc.y;
        };
        const float v0 = chunk(x0, 0), v1 = chunk(x1, 1);
        if (key < a.n && hf * 64 < a.R) {
          float* dst = a.A + ((size_t)u * a.G + (hf * 64) / a.n_obs) * a.n + key;
          if (a.n_obs == 32) {
            dst[0] = v0;                                   // head of chunk 0
            if (hf * 64 + 32 < a.R) dst[a.n] = v1;         // next head
          } else {
            dst[0] = v0 + v1;                              // n_obs == 64: one head per half
          }
        }
      }
    }
    if (PASS == 1) {
      const int r = q * 32 + lane;
      if (hf == 1) sXch[r] = make_float2(m, l);
      // named barrier 1 over the epilogue warps only
      asm volatile("bar.sync 1, %0;" ::"r"(kEpiWarps * 32) : "memory");
      if (hf == 0 && r < a.R) {
        const float2 o = sXch[r];
        const float M = fmaxf(m, o.x);
        const float L = l * exp2f(m - M) + o.y * exp2f(o.x - M);
        a.part[((size_t)u * kMaxSplits + split) * kRows + r] = make_float2(M, L);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

__global__ void obs_combine(const float2* __restrict__ part, int splits, int R, float* __restrict__ bias) {
  const int u = blockIdx.x, r = threadIdx.x;
  if (r >= kRows) return;
  float M = -1e30f;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, part[((size_t)u * kMaxSplits + s) * kRows + r].x);
  float L = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float2 p = part[((size_t)u * kMaxSplits + s) * kRows + r];
    L += p.y * exp2f(p.x - M);
  }
  bias[(size_t)u * kRows + r] = r < R ? M + log2f(L) : INFINITY;
}

// ---------------------------------------------------------------------------------------
// selection
// ---------------------------------------------------------------------------------------

// 64-bit selection key: score bits above, complemented index below, so that a larger key
// means a larger score or, for equal scores, a lower index. Scores are >= 0; -0 joins +0.
__device__ __forceinline__ unsigned long long sel_key(float score, int i) {
  uint32_t b = __float_as_uint(score);
  if ((b << 1) == 0) b = 0;
  return (static_cast<unsigned long long>(b) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(i));
}

struct SelShared {
  uint32_t hist[256];
  int ctl[4];                          // digit found, count above, bin count
  int cnt;
  unsigned long long list[kMaxBudget];
};

// The k-th largest of key(i), i < n, with key(i) = 0 meaning "not a candidate". Returns the
// threshold as (prefix, shift): a key is among the k largest iff (key >> shift) >= (prefix >> shift).
template <typename KeyFn>
__device__ void radix_select(int n, long long k, KeyFn key, SelShared& sh, unsigned long long* prefix_out,
                             int* shift_out) {
  unsigned long long prefix = 0;
  int shift = 64;
  for (int pass = 0; pass < 8; ++pass) {
    const int sft = 56 - 8 * pass;
    for (int b = threadIdx.x; b < 256; b += blockDim.x) sh.hist[b] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const unsigned long long kk = key(i);
      if (kk == 0) continue;
      if (shift == 64 || (kk >> shift) == (prefix >> shift)) atomicAdd(&sh.hist[(kk >> sft) & 255], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane l owns bins 255 - 8l .. 248 - 8l (highest first)
      const int l = threadIdx.x;
      uint32_t c[8];
      uint32_t loc = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = sh.hist[255 - 8 * l - j];
        loc += c[j];
      }
      uint32_t inc = loc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (l >= o) inc += y;
      }
      long long above = inc - loc;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (above < k && above + c[j] >= k) {
          sh.ctl[0] = 255 - 8 * l - j;
          sh.ctl[1] = static_cast<int>(above);
          sh.ctl[2] = static_cast<int>(c[j]);
        }
        above += c[j];
      }
    }
    __syncthreads();
    const int d = sh.ctl[0];
    k -= sh.ctl[1];
    prefix |= static_cast<unsigned long long>(d) << sft;
    shift = sft;
    const bool done = sh.ctl[2] == k;
    __syncthreads();
    if (done) break;
  }
  *prefix_out = prefix;
  *shift_out = shift;
}

// Descending bitonic sort of sh.list[0..P), P a power of two.
__device__ void bitonic_desc(unsigned long long* v, int P) {
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = threadIdx.x; t < P / 2; t += blockDim.x) {
        const int lo = 2 * t - (t & (stride - 1));
        const int hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const unsigned long long x = v[lo], y = v[hi];
        if ((x < y) == desc) {
          v[lo] = y;
          v[hi] = x;
        }
      }
      __syncthreads();
    }
  }
}

// Gathers the keys at or above the threshold into sh.list, sorts them and writes the indices.
template <typename KeyFn>
__device__ void emit_sorted(int n, int count, KeyFn key, unsigned long long prefix, int shift, SelShared& sh,
                            int32_t* out) {
  int P = 1;
  while (P < count) P <<= 1;
  if (threadIdx.x == 0) sh.cnt = 0;
  for (int t = threadIdx.x; t < P; t += blockDim.x) sh.list[t] = 0;
  __syncthreads();
  const unsigned long long want = prefix >> shift;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const unsigned long long kk = key(i);
    if (kk != 0 && (kk >> shift) >= want) {
      const int at = atomicAdd(&sh.cnt, 1);
      if (at < count) sh.list[at] = kk;
    }
  }
  __syncthreads();
  bitonic_desc(sh.list, P);
  for (int t = threadIdx.x; t < count; t += blockDim.x)
    out[t] = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(sh.list[t] & 0xFFFFFFFFu));
  __syncthreads();
}

__global__ void __launch_bounds__(kSelThreads) ckv_select(const float* __restrict__ A, const float* __restrict__ N,
                                                          int n, int G, int budget, int b1, float* __restrict__ sa,
                                                          float* __restrict__ sp, int32_t* __restrict__ idx_out) {
  extern __shared__ uint8_t smem_raw[];
  SelShared& sh = *reinterpret_cast<SelShared*>(smem_raw);
  const int u = blockIdx.x;
  const float* Au = A + (size_t)u * G * n;
  const float* Nu = N + (size_t)u * n * G;
  float* au = sa + (size_t)u * n;
  float* pu = sp + (size_t)u * n;
  int32_t* out = idx_out + (size_t)u * budget;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    float s = 0.f, p = 0.f;
    for (int h = 0; h < G; ++h) {
      const float x = Au[(size_t)h * n + i];
      s += x;
      p = fmaf(x, Nu[(size_t)i * G + h], p);
    }
    au[i] = s;
    pu[i] = p;
  }
  __syncthreads();
  if (n <= budget) {
    for (int t = threadIdx.x; t < budget; t += blockDim.x) out[t] = t < n ? t : -1;
    return;
  }
  // stage 1
  unsigned long long T1 = ~0ull;
  int s1 = 64;
  auto key1 = [&](int i) { return sel_key(au[i], i); };
  if (b1 > 0) {
    radix_select(n, b1, key1, sh, &T1, &s1);
    emit_sorted(n, b1, key1, T1, s1, sh, out);
  }
  // stage 2: candidates are the keys below the stage-1 threshold
  const unsigned long long w1 = s1 == 64 ? ~0ull : (T1 >> s1);
  auto key2 = [&](int i) -> unsigned long long {
    if (s1 != 64 && (sel_key(au[i], i) >> s1) >= w1) return 0ull;
    return sel_key(pu[i], i);
  };
  const int b2 = budget - b1;
  if (b2 > 0) {
    unsigned long long T2;
    int s2;
    radix_select(n, b2, key2, sh, &T2, &s2);
    emit_sorted(n, b2, key2, T2, s2, sh, out + b1);
  }
}

template <int D, bool BF16>
int launch_obs(const void* q_obs, const void* K, int units, int B, int Hq, int Hkv, int n, int n_obs, float* A,
               float2* part, float* bias, int32_t* status, cudaStream_t st) {
  using S = ObsSmem<D>;
  auto k1 = obs_kernel<D, BF16, 1>;
  auto k2 = obs_kernel<D, BF16, 2>;
  static QeOnce once;
  static int sms_of[QE_MAX_DEVICES];
  int dev = 0;
  int e = qe_once_per_device(once, &dev, [&](int d) {
    QE_CUDA_TRY(cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, S::BYTES));
    QE_CUDA_TRY(cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, S::BYTES));
    QE_CUDA_TRY(cudaDeviceGetAttribute(&sms_of[d], cudaDevAttrMultiProcessorCount, d));
    return QE_OK;
  });
  if (e) return e;
  const int sms = sms_of[dev];
  CUtensorMap tmQ, tmK;
  e = make_map(&tmQ, q_obs, BF16, D, (uint64_t)B * Hq * n_obs, 64, kRows);
  if (e) return e;
  e = make_map(&tmK, K, BF16, D, (uint64_t)units * n, 64, kTile);
  if (e) return e;
  ObsArgs a{};
  a.n = n;
  a.n_obs = n_obs;
  a.G = Hq / Hkv;
  a.R = a.G * n_obs;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.tiles = (n + kTile - 1) / kTile;
  int splits = (2 * sms) / units;
  if (splits < 1) splits = 1;
  if (splits > a.tiles) splits = a.tiles;
  if (splits > kMaxSplits) splits = kMaxSplits;
  a.splits = splits;
  a.cs = 1.4426950408889634f / sqrtf((float)D);
  a.part = part;
  a.bias = bias;
  a.A = A;
  a.status = status;
  k1<<<units * splits, kThreads, S::BYTES, st>>>(tmQ, tmK, a);
  obs_combine<<<units, kRows, 0, st>>>(part, splits, a.R, bias);
  k2<<<units * splits, kThreads, S::BYTES, st>>>(tmQ, tmK, a);
  return cudaGetLastError() == cudaSuccess ? QE_OK : QE_ERR_CUDA;
}

struct CkvLayout {
  size_t status, part, bias, sa, sp, bytes;
  CkvLayout(int units, int n) {
    auto r = [](size_t x) { return (x + 255) & ~size_t(255); };
    status = 0;
    part = 256;
    bias = part + r((size_t)units * kMaxSplits * kRows * sizeof(float2));
    sa = bias + r((size_t)units * kRows * sizeof(float));
    sp = sa + r((size_t)units * n * sizeof(float));
    bytes = sp + r((size_t)units * n * sizeof(float));
  }
};

}  // namespace

QE_API size_t qe_criticalkv_scratch_bytes(int B, int Hq, int Hkv, int n, int n_obs) {
  (void)Hq;
  (void)n_obs;
  if (B < 1 || Hkv < 1 || n < 1) return 0;
  return CkvLayout(B * Hkv, n).bytes;
}

QE_API int qe_criticalkv_select(const void* q_obs, int n_obs, const void* K, const void* V, const void* W_O, int B,
                                int Hq, int Hkv, int n, int D, int hidden, int dtype, int budget, float alpha,
                                float* A_out, float* N_out, int32_t* idx_out, void* scratch, size_t scratch_bytes,
                                qe_stream_t stream) {
  if (!q_obs || !K || !V || !W_O || !A_out || !N_out || !idx_out || !scratch) return QE_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || n < 1 || budget < 1) return QE_ERR_INVALID_ARG;
  if (!(alpha >= 0.f && alpha <= 1.f)) return QE_ERR_INVALID_ARG;
  if (dtype != QE_FP16 && dtype != QE_BF16) return QE_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if (D != 64 && D != 128) return QE_ERR_UNSUPPORTED_SHAPE;
  if ((n_obs != 32 && n_obs != 64) || G * n_obs > kRows || n_obs > n) return QE_ERR_UNSUPPORTED_SHAPE;
  if (budget > kMaxBudget || G > QE_MAX_G || hidden < 64 || hidden % 64) return QE_ERR_UNSUPPORTED_SHAPE;
  if ((long long)B * Hkv * n >= (1ll << 31)) return QE_ERR_UNSUPPORTED_SHAPE;
  if (!qe_aligned(q_obs, 16) || !qe_aligned(K, 16) || !qe_aligned(V, 16) || !qe_aligned(W_O, 16) ||
      !qe_aligned(scratch, 256))
    return QE_ERR_INVALID_ARG;
  const int units = B * Hkv;
  const CkvLayout L(units, n);
  if (scratch_bytes < L.bytes) return QE_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(scratch);
  int32_t* status = reinterpret_cast<int32_t*>(base + L.status);
  QE_CUDA_TRY(cudaMemsetAsync(status, 0, 16, st));
  // N[u][i][h] = ||V_i W_O^h||_1
  int e = launch_vwo(V, units, n, D, dtype, W_O, Hq, Hkv, hidden, N_out, (long long)n * G, status, st);
  if (e) return e;
  float2* part = reinterpret_cast<float2*>(base + L.part);
  float* bias = reinterpret_cast<float*>(base + L.bias);
  const bool bf = dtype == QE_BF16;
  if (D == 128)
    e = bf ? launch_obs<128, true>(q_obs, K, units, B, Hq, Hkv, n, n_obs, A_out, part, bias, status, st)
           : launch_obs<128, false>(q_obs, K, units, B, Hq, Hkv, n, n_obs, A_out, part, bias, status, st);
  else
    e = bf ? launch_obs<64, true>(q_obs, K, units, B, Hq, Hkv, n, n_obs, A_out, part, bias, status, st)
           : launch_obs<64, false>(q_obs, K, units, B, Hq, Hkv, n, n_obs, A_out, part, bias, status, st);
  if (e) return e;
  const int b1 = (int)floor((double)alpha * (double)budget);
  const size_t smem = sizeof(SelShared);
  static QeOnce once;
  int dev = 0;
  e = qe_once_per_device(once, &dev, [&](int) {
    QE_CUDA_TRY(cudaFuncSetAttribute(ckv_select, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    return QE_OK;
  });
  if (e) return e;
  ckv_select<<<units, kSelThreads, smem, st>>>(A_out, N_out, n, G, budget, b1,
                                               reinterpret_cast<float*>(base + L.sa),
                                               reinterpret_cast<float*>(base + L.sp), idx_out);
  return cudaGetLastError() == cudaSuccess ? QE_OK : QE_ERR_CUDA;
}
