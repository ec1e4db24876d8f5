// DBTrimKV global trim of a paged, variable-length cache ("Make Each Token Count",
// Metodologia 2-4). Entry i of a head carries a retention rate beta_i and a position pos_i;
// at step t its retention is beta_i^(t - pos_i). The cache keeps the M entries of highest
// retention over all heads, ranked in float64 on log r = (t - pos) * ln(beta), ties to the
// lower flat index, and compacts every head's survivors in their original order.
//
// Pipeline (one stream, nothing allocated; all state in the caller's scratch):
//   T0 trim_init     1 CTA: validate lengths, exclusive scan -> flat offsets, reset state.
//   T1 trim_keygen   (chunk, head) CTAs: key -> order-preserving u64 at its flat index,
//                    fused with radix pass 0 (top 11 bits); the last CTA picks the digit.
//   T2 trim_hist     passes 1..5 over the flat key array (persistent grid); each pass
//                    histograms the next digit of the keys that share the decided prefix and
//                    its last CTA picks the digit holding the M-th key. A pass whose chosen
//                    bin is kept whole ends the search early; later passes return at once.
//   T3 trim_count    (chunk, head): keys above / equal to the threshold per chunk.
//   T4 trim_scan     1 CTA: equal keys are kept in flat order up to the remaining count;
//                    per-head exclusive scan of survivors -> destination base per chunk.
//   T5 trim_move     (chunk, head): stable in-chunk ranks, copy K/V rows, beta, pos.
// Keys (8 B per entry) stay L2-resident across the passes; K/V rows move once.
#include "qe_internal.cuh"

namespace {

constexpr int kCH = 2048;             // entries per chunk CTA
constexpr int kCT = 256;              // threads per chunk CTA
constexpr int kEPT = kCH / kCT;       // entries per thread
constexpr int kDigit = 11;            // radix digit width
constexpr int kBins = 1 << kDigit;
constexpr int kPasses = 6;            // 5 x 11 + 9 = 64 bits
constexpr int kHT = 512;              // threads per histogram CTA

// modes of the selection
constexpr int kSelect = 0;            // threshold not yet found
constexpr int kFound = 1;             // threshold prefix found; keep keys above it and `need` equal
constexpr int kKeepAll = 2;           // M >= total
constexpr int kKeepNone = 3;          // M == 0

__host__ __device__ constexpr int pass_shift(int p) {
  return 64 - kDigit * (p + 1) > 0 ? 64 - kDigit * (p + 1) : 0;
}
__host__ __device__ constexpr int pass_width(int p) {
  return p < kPasses - 1 ? kDigit : 64 - kDigit * (kPasses - 1);
}

struct TrimState {
  int32_t status[4];                  // {code, detail}: the first device-side error
  unsigned long long prefix;          // decided high bits of the threshold key (ordered form)
  long long need;                     // keys equal to the prefix still to keep (flat order)
  int32_t total;                      // valid entries over all heads
  int32_t shift;                      // keys compare on (ordered >> shift)
  int32_t mode;
  uint32_t ticket[kPasses];
};

struct TrimScratch {
  TrimState* st;
  uint32_t* hist;                     // [kBins]
  int32_t* off;                       // [n_heads + 1] flat offset of each head
  unsigned long long* keys;           // [total] ordered keys, flat order
  int4* ctab;                         // [n_heads][nch] {gt, eq, kept ties, destination base}
};

__host__ __device__ inline size_t rup256(size_t x) { return (x + 255) & ~size_t(255); }

struct ScratchLayout {
  size_t st, hist, off, keys, ctab, bytes;
  ScratchLayout(int n_heads, int max_pages) {
    const size_t cap = size_t(max_pages) * QE_PAGE;
    const size_t nch = (cap + kCH - 1) / kCH;
    st = 0;
    hist = rup256(sizeof(TrimState));
    off = hist + rup256(sizeof(uint32_t) * kBins);
    keys = off + rup256(sizeof(int32_t) * (size_t(n_heads) + 1));
    ctab = keys + rup256(sizeof(unsigned long long) * size_t(n_heads) * cap);
    bytes = ctab + rup256(sizeof(int4) * size_t(n_heads) * nch);
  }
};

__device__ __forceinline__ void trim_error(TrimState* st, int code, int detail) {
  if (atomicCAS(&st->status[0], 0, code) == 0) st->status[1] = detail;
}

// Order-preserving image of a float64 key: larger key <-> larger u64. -0 maps with +0,
// NaN to 0 (below every other key).
__device__ __forceinline__ unsigned long long ordered_key(double key) {
  unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(key));
  if ((b << 1) == 0) b = 0;
  if (key != key) return 0ull;
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

// Block-wide exclusive scan of one int per thread; *total receives the sum.
// sm: at least 32 ints of shared memory, reused (the call ends with a barrier).
template <int NT>
__device__ __forceinline__ int block_excl_scan(int v, int* total, int* sm) {
  static_assert(NT % 32 == 0 && NT <= 1024, "block size");
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sm[w] = x;
  __syncthreads();
  if (w == 0) {
    int s = lane < NT / 32 ? sm[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < NT / 32) sm[lane] = s;
  }
  __syncthreads();
  const int before = w ? sm[w - 1] : 0;
  *total = sm[NT / 32 - 1];
  __syncthreads();
  return before + x - v;
}

// Adds one to bin `digit` of a shared histogram (plain shared-memory atomics: aggregating
// equal digits with a warp match vote cost more than the contention it saves).
__device__ __forceinline__ void hist_add(uint32_t* sh, uint32_t digit, bool valid) {
  if (valid) atomicAdd(&sh[digit], 1u);
}

// Run by the last CTA of pass p once every CTA's counts are in `hist`: find the digit whose
// bin holds the need-th largest key among those sharing the prefix, extend the prefix, and
// reset the histogram for the next pass.
template <int NT>
__device__ void select_digit(TrimScratch s, int p, int* sm) {
  constexpr int per = kBins / NT;
  const int tid = threadIdx.x;
  const long long k = s.st->need;
  // thread tid owns bins [hi - per, hi), the highest bins going to thread 0
  const int hi = kBins - tid * per;
  uint32_t c[per];
  int local = 0;
#pragma unroll
  for (int j = 0; j < per; ++j) {
    c[j] = __ldcg(&s.hist[hi - 1 - j]);
    local += static_cast<int>(c[j]);
  }
  int sum_all;
  const int above0 = block_excl_scan<NT>(local, &sum_all, sm);
  long long above = above0;
#pragma unroll
  for (int j = 0; j < per; ++j) {
    if (above < k && above + c[j] >= k) {
      const int d = hi - 1 - j;
      const long long rest = k - above;
      s.st->prefix |= static_cast<unsigned long long>(d) << pass_shift(p);
      s.st->shift = pass_shift(p);
      s.st->need = rest;
      if (static_cast<long long>(c[j]) == rest || p == kPasses - 1) s.st->mode = kFound;
    }
    above += c[j];
  }
  __syncthreads();
  for (int b = tid; b < kBins; b += NT) s.hist[b] = 0;
}

// T0: lengths -> offsets, state reset.
__global__ void __launch_bounds__(1024) trim_init(const int32_t* __restrict__ lengths, int n_heads,
                                                  int cap, long long M, TrimScratch s) {
  __shared__ int sm[32];
  const int tid = threadIdx.x;
  if (tid < 4) s.st->status[tid] = 0;
  if (tid < kPasses) s.st->ticket[tid] = 0;
  for (int b = tid; b < kBins; b += 1024) s.hist[b] = 0;
  int carry = 0;
  for (int base = 0; base < n_heads; base += 1024) {
    const int h = base + tid;
    int len = 0;
    if (h < n_heads) {
      len = lengths[h];
      if (len < 0 || len > cap) {
        trim_error(s.st, QE_ERR_INVALID_ARG, h);
        len = 0;
      }
    }
    int tot;
    const int ex = block_excl_scan<1024>(len, &tot, sm);
    if (h < n_heads) s.off[h] = carry + ex;
    carry += tot;
  }
  if (tid == 0) {
    s.off[n_heads] = carry;
    s.st->total = carry;
    s.st->prefix = 0;
    s.st->shift = 64;
    s.st->need = M;
    s.st->mode = M == 0 ? kKeepNone : (M >= carry ? kKeepAll : kSelect);
  }
}

__device__ __forceinline__ int head_length(const TrimScratch& s, int h) {
  return s.off[h + 1] - s.off[h];
}

// T1: keys of chunk blockIdx.x of head blockIdx.y, and the histogram of their top digit.
__global__ void __launch_bounds__(kCT) trim_keygen(const float* __restrict__ beta,
                                                   const int32_t* __restrict__ pos,
                                                   const int32_t* __restrict__ page_table,
                                                   int max_pages, int n_pages_total, int t,
                                                   TrimScratch s) {
  __shared__ uint32_t sh[kBins];
  __shared__ int sm[32];
  __shared__ int last;
  const int tid = threadIdx.x, h = blockIdx.y;
  const int len = head_length(s, h);
  const int e0 = blockIdx.x * kCH;
  const bool do_hist = s.st->mode == kSelect;
  for (int b = tid; b < kBins; b += kCT) sh[b] = 0;
  __syncthreads();
  if (e0 < len) {
    const int32_t* pt = page_table + static_cast<size_t>(h) * max_pages;
    unsigned long long* kout = s.keys + s.off[h];
    // every load of the thread's entries is issued before any is used: page ids, then the
    // entries' beta and pos
    int pgv[kEPT];
#pragma unroll
    for (int j = 0; j < kEPT; ++j) {
      const int e = e0 + j * kCT + tid;
      pgv[j] = e < len ? pt[e >> 4] : -1;
    }
    float bv[kEPT];
    int32_t pv[kEPT];
#pragma unroll
    for (int j = 0; j < kEPT; ++j) {
      const int e = e0 + j * kCT + tid;
      const bool good = pgv[j] >= 0 && pgv[j] < n_pages_total;
      const size_t at = good ? static_cast<size_t>(pgv[j]) * QE_PAGE + (e & 15) : 0;
      bv[j] = good ? beta[at] : 1.f;
      pv[j] = good ? pos[at] : 0;
    }
#pragma unroll
    for (int j = 0; j < kEPT; ++j) {
      const int e = e0 + j * kCT + tid;
      const bool valid = e < len;
      unsigned long long ok = 0;
      if (valid) {
        if (pgv[j] < 0 || pgv[j] >= n_pages_total) {
          trim_error(s.st, QE_ERR_DEVICE_FAULT, h);
        } else {
          const double age = static_cast<double>(t) - static_cast<double>(pv[j]);
          ok = ordered_key(age * log(static_cast<double>(bv[j])));
        }
        kout[e] = ok;
      }
      if (do_hist) hist_add(sh, static_cast<uint32_t>(ok >> pass_shift(0)), valid);
    }
  }
  __syncthreads();
  if (do_hist)
    for (int b = tid; b < kBins; b += kCT)
      if (sh[b]) atomicAdd(&s.hist[b], sh[b]);
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    last = atomicAdd(&s.st->ticket[0], 1u) == gridDim.x * gridDim.y - 1;
  }
  __syncthreads();
  if (last && do_hist) {
    __threadfence();
    select_digit<kCT>(s, 0, sm);
  }
}

// T2: radix pass p >= 1 over the flat key array.
__global__ void __launch_bounds__(kHT) trim_hist(TrimScratch s, int p) {
  __shared__ uint32_t sh[kBins];
  __shared__ int sm[32];
  __shared__ int last;
  if (s.st->mode != kSelect) return;  // uniform over the grid: state fixed before launch
  const int tid = threadIdx.x;
  const int total = s.st->total;
  const int cmp = s.st->shift;        // bits above this are decided
  const unsigned long long want = s.st->prefix >> cmp;
  const int sft = pass_shift(p);
  const uint32_t mask = (1u << pass_width(p)) - 1u;
  for (int b = tid; b < kBins; b += kHT) sh[b] = 0;
  __syncthreads();
  // each warp takes 256 consecutive keys per step (8 per lane, four 16-byte loads issued
  // together); the bound is warp-uniform so every lane reaches the warp-wide votes in hist_add
  const int lane = tid & 31;
  const int stride = gridDim.x * kHT * 8;
  for (int wb = (blockIdx.x * kHT + (tid & ~31)) * 8; wb < total; wb += stride) {
    ulonglong2 v[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int i0 = wb + c * 64 + lane * 2;
      v[c] = make_ulonglong2(0ull, 0ull);
      if (i0 + 1 < total)
        v[c] = __ldcg(reinterpret_cast<const ulonglong2*>(s.keys + i0));
      else if (i0 < total)
        v[c].x = __ldcg(s.keys + i0);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int i0 = wb + c * 64 + lane * 2;
      const bool m0 = i0 < total && (v[c].x >> cmp) == want;
      const bool m1 = i0 + 1 < total && (v[c].y >> cmp) == want;
      hist_add(sh, static_cast<uint32_t>(v[c].x >> sft) & mask, m0);
      hist_add(sh, static_cast<uint32_t>(v[c].y >> sft) & mask, m1);
    }
  }
  __syncthreads();
  for (int b = tid; b < kBins; b += kHT)
    if (sh[b]) atomicAdd(&s.hist[b], sh[b]);
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    last = atomicAdd(&s.st->ticket[p], 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (last) {
    __threadfence();
    select_digit<kHT>(s, p, sm);
  }
}

// Classification of one key against the final state: 2 = above the threshold, 1 = equal to
// it (kept in flat order up to `need`), 0 = dropped.
struct Classifier {
  int mode, shift;
  unsigned long long want;
  __device__ Classifier(const TrimState* st) {
    mode = st->mode;
    shift = st->shift;
    want = mode == kFound ? (st->prefix >> shift) : 0;
  }
  __device__ __forceinline__ int operator()(unsigned long long k) const {
    if (mode == kKeepAll) return 2;
    if (mode != kFound) return 0;
    const unsigned long long v = k >> shift;
    return v > want ? 2 : (v == want ? 1 : 0);
  }
};

// Loads the kEPT consecutive keys of this thread's entries (flat index f0.., valid below n).
__device__ __forceinline__ void load_keys(const unsigned long long* keys, int f0, int n,
                                          unsigned long long (&k)[kEPT]) {
  // f0 is a multiple of kEPT but the head offset need not be 16-byte aligned: plain loads.
#pragma unroll
  for (int j = 0; j < kEPT; ++j) k[j] = j < n ? __ldcg(keys + f0 + j) : 0ull;
}

// T3: per chunk, keys above and equal to the threshold.
__global__ void __launch_bounds__(kCT) trim_count(TrimScratch s, int nch) {
  __shared__ int sm[32];
  const int tid = threadIdx.x, h = blockIdx.y, c = blockIdx.x;
  const int len = head_length(s, h);
  const int e0 = c * kCH + tid * kEPT;
  const Classifier cls(s.st);
  int gt = 0, eq = 0;
  if (e0 < len) {
    unsigned long long k[kEPT];
    load_keys(s.keys + s.off[h], e0, len - e0, k);
#pragma unroll
    for (int j = 0; j < kEPT; ++j) {
      if (e0 + j >= len) break;
      const int r = cls(k[j]);
      gt += r == 2;
      eq += r == 1;
    }
  }
  int tg, te;
  block_excl_scan<kCT>(gt, &tg, sm);
  block_excl_scan<kCT>(eq, &te, sm);
  if (tid == 0) s.ctab[static_cast<size_t>(h) * nch + c] = make_int4(tg, te, 0, 0);
}

// T4: ties kept in flat order; destination base of each chunk; new lengths.
__global__ void __launch_bounds__(1024) trim_scan(TrimScratch s, int n_heads, int nch,
                                                  int32_t* __restrict__ new_lengths) {
  __shared__ int sm[32];
  const int tid = threadIdx.x;
  const long long need = s.st->mode == kFound ? s.st->need : 0;
  const int n = n_heads * nch;
  long long carry = 0;
  for (int base = 0; base < n; base += 1024) {
    const int i = base + tid;
    int4 ct = i < n ? s.ctab[i] : make_int4(0, 0, 0, 0);
    int tot;
    const long long before = carry + block_excl_scan<1024>(ct.y, &tot, sm);
    const long long kept = need - before;
    ct.z = static_cast<int>(kept <= 0 ? 0 : (kept >= ct.y ? ct.y : kept));
    ct.w = ct.x + ct.z;  // survivors of the chunk, replaced by the base below
    if (i < n) s.ctab[i] = ct;
    carry += tot;
  }
  __syncthreads();
  for (int h = tid; h < n_heads; h += 1024) {
    int b = 0;
    for (int c = 0; c < nch; ++c) {
      int4& ct = s.ctab[static_cast<size_t>(h) * nch + c];
      const int sv = ct.w;
      ct.w = b;
      b += sv;
    }
    new_lengths[h] = b;
  }
}

// T5: stable compaction of chunk blockIdx.x of head blockIdx.y. R = 16-byte words per row.
template <int R>
__global__ void __launch_bounds__(kCT) trim_move(const float* __restrict__ beta,
                                                 const int32_t* __restrict__ pos,
                                                 const int32_t* __restrict__ page_table,
                                                 int max_pages, int n_pages_total,
                                                 const uint4* __restrict__ kv_in,
                                                 uint4* __restrict__ kv_out,
                                                 float* __restrict__ beta_out,
                                                 int32_t* __restrict__ pos_out, TrimScratch s,
                                                 int nch) {
  constexpr int kPg = kCH / QE_PAGE;  // logical pages of a chunk
  __shared__ int sm[32];
  __shared__ int16_t src_of[kCH];     // in-chunk entry of each survivor, in order
  __shared__ int32_t spg[kPg];        // physical page of each source page of the chunk
  __shared__ int32_t dpg[kPg + 1];    // physical page of each destination page touched
  const int tid = threadIdx.x, h = blockIdx.y, c = blockIdx.x;
  const int len = head_length(s, h);
  const int e0 = c * kCH;
  if (e0 >= len) return;
  const int4 ct = s.ctab[static_cast<size_t>(h) * nch + c];
  const Classifier cls(s.st);
  if (cls.mode == kKeepNone) return;
  const int32_t* pt = page_table + static_cast<size_t>(h) * max_pages;

  // ranks: ties first (kept while their in-chunk rank is below ct.z), then survivors
  const int et = e0 + tid * kEPT;
  unsigned long long k[kEPT];
  load_keys(s.keys + s.off[h], et, len - et, k);
  int r[kEPT];
  int neq = 0;
#pragma unroll
  for (int j = 0; j < kEPT; ++j) {
    r[j] = et + j < len ? cls(k[j]) : 0;
    neq += r[j] == 1;
  }
  int tot;
  int tie = block_excl_scan<kCT>(neq, &tot, sm);
  int nkeep = 0;
#pragma unroll
  for (int j = 0; j < kEPT; ++j) {
    if (r[j] == 1) r[j] = tie++ < ct.z ? 2 : 0;
    nkeep += r[j] == 2;
  }
  int ns;
  int rank = block_excl_scan<kCT>(nkeep, &ns, sm);
#pragma unroll
  for (int j = 0; j < kEPT; ++j)
    if (r[j] == 2) src_of[rank++] = static_cast<int16_t>(tid * kEPT + j);

  // page tables of the source chunk and of the destination range
  const int p0 = e0 / QE_PAGE;
  const int q0 = ct.w / QE_PAGE;
  const int nq = ns ? (ct.w + ns - 1) / QE_PAGE - q0 + 1 : 0;
  for (int i = tid; i < kPg; i += kCT) {
    int pg = -1;
    if (p0 + i < max_pages && (p0 + i) * QE_PAGE < len) {
      pg = pt[p0 + i];
      if (pg < 0 || pg >= n_pages_total) {
        trim_error(s.st, QE_ERR_DEVICE_FAULT, h);
        pg = -1;
      }
    }
    spg[i] = pg;
  }
  for (int i = tid; i < nq; i += kCT) {
    int pg = pt[q0 + i];
    if (pg < 0 || pg >= n_pages_total) {
      trim_error(s.st, QE_ERR_DEVICE_FAULT, h);
      pg = -1;
    }
    dpg[i] = pg;
  }
  __syncthreads();

  // K and V rows: 2R words per survivor, consecutive threads on consecutive words
  const int items = ns * 2 * R;
  constexpr int kU = 4;
  for (int i0 = tid; i0 < items; i0 += kCT * kU) {
    uint4 w[kU];
    size_t dst[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u * kCT;
      dst[u] = ~size_t(0);
      if (i < items) {
        const int sv = i / (2 * R), rem = i - sv * 2 * R;
        const int part = rem / R, word = rem - part * R;
        const int se = src_of[sv];
        const int de = ct.w + sv;
        const int sp = spg[se / QE_PAGE], dp = dpg[de / QE_PAGE - q0];
        if (sp >= 0 && dp >= 0) {
          w[u] = __ldcs(kv_in + ((static_cast<size_t>(sp) * 2 + part) * QE_PAGE + (se & 15)) * R +
                        word);
          dst[u] = ((static_cast<size_t>(dp) * 2 + part) * QE_PAGE + (de & 15)) * R + word;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u)
      if (dst[u] != ~size_t(0)) __stcs(kv_out + dst[u], w[u]);
  }
  for (int sv = tid; sv < ns; sv += kCT) {
    const int se = src_of[sv], de = ct.w + sv;
    const int sp = spg[se / QE_PAGE], dp = dpg[de / QE_PAGE - q0];
    if (sp < 0 || dp < 0) continue;
    const size_t a = static_cast<size_t>(sp) * QE_PAGE + (se & 15);
    const size_t b = static_cast<size_t>(dp) * QE_PAGE + (de & 15);
    beta_out[b] = beta[a];
    pos_out[b] = pos[a];
  }
}

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

}  // namespace

QE_API size_t qe_trim_scratch_bytes(int n_heads, int max_pages_per_head) {
  if (n_heads < 1 || max_pages_per_head < 1) return 0;
  return ScratchLayout(n_heads, max_pages_per_head).bytes;
}

QE_API int qe_trim_global_topm(const float* beta, const int32_t* pos, const int32_t* page_table,
                               const int32_t* lengths, int n_heads, int max_pages_per_head,
                               int n_pages_total, int D, int dtype, int t, long long M,
                               const void* kv_in, void* kv_out, float* beta_out,
                               int32_t* pos_out, int32_t* new_lengths, void* scratch,
                               size_t scratch_bytes, qe_stream_t stream) {
  if (!beta || !pos || !page_table || !lengths || !kv_in || !kv_out || !beta_out || !pos_out ||
      !new_lengths || !scratch)
    return QE_ERR_INVALID_ARG;
  if (n_heads < 1 || max_pages_per_head < 1 || n_pages_total < 1 || M < 0)
    return QE_ERR_INVALID_ARG;
  if (n_heads > 65535) return QE_ERR_UNSUPPORTED_SHAPE;
  if (dtype != QE_FP16 && dtype != QE_BF16) return QE_ERR_INVALID_ARG;
  if (D != 64 && D != 128 && D != 256) return QE_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<long long>(n_heads) * max_pages_per_head * QE_PAGE >= (1ll << 31))
    return QE_ERR_UNSUPPORTED_SHAPE;
  if (!qe_aligned(kv_in, 16) || !qe_aligned(kv_out, 16) || !qe_aligned(scratch, 256))
    return QE_ERR_INVALID_ARG;
  const ScratchLayout L(n_heads, max_pages_per_head);
  if (scratch_bytes < L.bytes) return QE_ERR_WORKSPACE;
  const size_t kv_bytes = static_cast<size_t>(n_pages_total) * 2 * QE_PAGE * D * 2;
  const size_t meta_bytes = static_cast<size_t>(n_pages_total) * QE_PAGE * 4;
  if (overlap(kv_in, kv_bytes, kv_out, kv_bytes) || overlap(beta, meta_bytes, beta_out, meta_bytes) ||
      overlap(pos, meta_bytes, pos_out, meta_bytes))
    return QE_ERR_INVALID_ARG;
  const int sms = sm_count();
  if (sms <= 0) return QE_ERR_CUDA;

  uint8_t* base = static_cast<uint8_t*>(scratch);
  TrimScratch s;
  s.st = reinterpret_cast<TrimState*>(base + L.st);
  s.hist = reinterpret_cast<uint32_t*>(base + L.hist);
  s.off = reinterpret_cast<int32_t*>(base + L.off);
  s.keys = reinterpret_cast<unsigned long long*>(base + L.keys);
  s.ctab = reinterpret_cast<int4*>(base + L.ctab);
  const int cap = max_pages_per_head * QE_PAGE;
  const int nch = (cap + kCH - 1) / kCH;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  trim_init<<<1, 1024, 0, st>>>(lengths, n_heads, cap, M, s);
  trim_keygen<<<dim3(nch, n_heads), kCT, 0, st>>>(beta, pos, page_table, max_pages_per_head,
                                                  n_pages_total, t, s);
  for (int p = 1; p < kPasses; ++p) trim_hist<<<2 * sms, kHT, 0, st>>>(s, p);
  trim_count<<<dim3(nch, n_heads), kCT, 0, st>>>(s, nch);
  trim_scan<<<1, 1024, 0, st>>>(s, n_heads, nch, new_lengths);
  const uint4* in = static_cast<const uint4*>(kv_in);
  uint4* out = static_cast<uint4*>(kv_out);
  const dim3 grid(nch, n_heads);
  if (D == 64)
    trim_move<8><<<grid, kCT, 0, st>>>(beta, pos, page_table, max_pages_per_head, n_pages_total,
                                       in, out, beta_out, pos_out, s, nch);
  else if (D == 128)
    trim_move<16><<<grid, kCT, 0, st>>>(beta, pos, page_table, max_pages_per_head, n_pages_total,
                                        in, out, beta_out, pos_out, s, nch);
  else
    trim_move<32><<<grid, kCT, 0, st>>>(beta, pos, page_table, max_pages_per_head, n_pages_total,
                                        in, out, beta_out, pos_out, s, nch);
  return cudaGetLastError() == cudaSuccess ? QE_OK : QE_ERR_CUDA;
}
