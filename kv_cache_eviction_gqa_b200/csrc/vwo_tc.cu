// ||V_i W_O^h||_1 on the 5th-generation tensor cores (tcgen05, accumulators in TMEM).
//
// "Resumo Técnico: CriticalKV", Framework Teórico: the perturbation bound depends on the
// projected values V W_O; Algoritmo, Etapa 2 scores an entry by A_i * ||V_i W_O||_1.
//
// out[g][r][j] = sum_c | sum_d V[g][r][d] * W_O[(kvh*G + j)*D + d][c] |,  kvh = g % Hkv.
//
// One CTA owns 256 rows (two 128-row M-tiles) of one group and a range of N-tiles of
// 128 columns over (query head j, hidden tile). Warp roles:
//   warp 0     one elected thread issues TMA loads: the 256 x D block of V once (K-major,
//              128-byte swizzle), then W_O^h tiles [D rows][128 columns] through a 4-stage
//              ring. W_O is read in its natural row-major layout as an MN-major operand.
//   warp 1     allocates 512 TMEM columns; one elected thread issues tcgen05.mma
//              (kind::f16, M = 128, N = 128, K = 16) into one of two accumulator buffers
//              (2 M-tiles x 128 columns each) and commits to mbarriers.
//   warps 2-9  epilogue: each thread owns one accumulator row (TMEM lane), reads 128 fp32
//              columns with tcgen05.ld, adds their absolute values to a running row sum and
//              releases the buffer; at the end of a head's columns the row sum is written.
// The product V W_O (rows x G*hidden) is never stored. All waits are bounded: a wait that
// gives up records QE_ERR_TIMEOUT, raises a CTA-wide abort flag and the CTA winds down.
#include "tc_common.cuh"

namespace {

using namespace tc;

constexpr int kMT = 2;          // 128-row M-tiles per CTA
constexpr int kBM = 128;
constexpr int kBN = 128;        // N tile = TMEM columns per accumulator
constexpr int kNST = 4;         // W_O stages
constexpr int kEpiWarps = 4 * kMT;
constexpr int kThreads = (2 + kEpiWarps) * 32;
constexpr int kTmemCols = 2 * kMT * kBN;  // two accumulator buffers = 512 columns

struct VwoArgs {
  float* out;
  long long ogs;
  int rows, G, Hkv;
  int ntiles_per_head;  // hidden / kBN
  int mpairs;           // ceil(rows / 256)
  int nsplit;           // N-tile ranges per (group, row block)
  int ntot;             // G * ntiles_per_head
  int nparts;           // column parts per head (each writes its own partial row sums)
  long long pstride;    // elements between the partial outputs of consecutive parts
  int atomic;           // several CTAs add into one output element (never set: splits are whole heads)
  int32_t* status;
};

template <int D, bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
    vwo_tc_kernel(const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmW, VwoArgs a) {
  constexpr int KB = D / 64;               // 64-element (128-byte) K boxes
  constexpr int A_BOX = kBM * 128;         // one box: 128 rows x 128 bytes
  constexpr int A_BYTES = kMT * KB * A_BOX;
  constexpr int B_BOX = D * 128;           // one box: D rows x 64 columns x 2 bytes
  constexpr int B_STAGE = (kBN / 64) * B_BOX;
  constexpr uint32_t FMT = BF16 ? 1u : 0u;
  // kind::f16 instruction descriptor: D fp32, A/B fp16|bf16, A K-major, B MN-major, M=128, N=128
  constexpr uint32_t IDESC = (1u << 4) | (FMT << 7) | (FMT << 10) | (1u << 16) | ((uint32_t)(kBN >> 3) << 17) |
                             ((uint32_t)(kBM >> 4) << 24);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kNST * B_STAGE);
  uint64_t* empty = full + kNST;
  uint64_t* accf = empty + kNST;
  uint64_t* acce = accf + 2;
  uint64_t* afull = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(afull + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int item = blockIdx.x;
  const int split = item % a.nsplit;
  item /= a.nsplit;
  const int p = item % a.mpairs, g = item / a.mpairs, kvh = g % a.Hkv;
  const int n0 = (int)((long long)a.ntot * split / a.nsplit), n1 = (int)((long long)a.ntot * (split + 1) / a.nsplit);
  const int NT = n1 - n0;
  const int row0 = p * kMT * kBM;
  const int grow0 = g * a.rows + row0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], kEpiWarps);
    }
    mbar_init(afull, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---- producer ----
      mbar_arrive_expect_tx(afull, A_BYTES);
      for (int mt = 0; mt < kMT; ++mt)
        for (int kb = 0; kb < KB; ++kb) tma_load_2d(sA + (mt * KB + kb) * A_BOX, &tmV, kb * 64, grow0 + mt * kBM, afull);
      for (int i = 0; i < NT; ++i) {
        const int s = i % kNST;
        if (!wait_or_abort(&empty[s], ((i / kNST) & 1) ^ 1, abort_flag, a.status, 3001)) break;
        const int n = n0 + i, j = n / a.ntiles_per_head, nt = n % a.ntiles_per_head;
        const int hrow = (kvh * a.G + j) * D, col = nt * kBN;
        mbar_arrive_expect_tx(&full[s], B_STAGE);
        for (int c = 0; c < kBN / 64; ++c) tma_load_2d(sB + s * B_STAGE + c * B_BOX, &tmW, col + c * 64, hrow, &full[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issuer ----
      if (wait_or_abort(afull, 0, abort_flag, a.status, 3002)) {
        tc_fence_after();
        for (int i = 0; i < NT; ++i) {
          const int s = i % kNST, b = i & 1;
          if (!wait_or_abort(&full[s], (i / kNST) & 1, abort_flag, a.status, 3003)) break;
          if (!wait_or_abort(&acce[b], ((i >> 1) & 1) ^ 1, abort_flag, a.status, 3004)) break;
          tc_fence_after();
#pragma unroll
          for (int mt = 0; mt < kMT; ++mt) {
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const uint64_t ad = sdesc(smem_u32(sA + (mt * KB + k / 4) * A_BOX + (k % 4) * 32), 16, 1024);
              const uint64_t bd = sdesc(smem_u32(sB + s * B_STAGE + k * 16 * 128), B_BOX, 1024);
              mma_f16(tmem + (uint32_t)(b * kMT * kBN + mt * kBN), ad, bd, IDESC, k > 0 ? 1u : 0u);
            }
          }
          mma_commit(&empty[s]);
          mma_commit(&accf[b]);
        }
      }
    }
  } else {
    // ---- epilogue ----
    const int ew = warp - 2, mt = ew / 4, q = warp & 3;
    const int r = row0 + mt * kBM + q * 32 + lane;
    float rowsum = 0.f;
    for (int i = 0; i < NT; ++i) {
      const int b = i & 1;
      if (!__all_sync(0xffffffffu, wait_or_abort(&accf[b], (i >> 1) & 1, abort_flag, a.status, 3005))) break;
      tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * kMT * kBN + mt * kBN);
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) rowsum += tmem_abs_sum32(taddr + c * 32);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[b]);
      const int n = n0 + i;
      if (n % a.ntiles_per_head == a.ntiles_per_head - 1 || i == NT - 1) {
        const int j = n / a.ntiles_per_head;
        if (r < a.rows) {
          float* o = a.out + (size_t)(split % a.nparts) * a.pstride + (size_t)g * a.ogs + (size_t)r * a.G + j;
          if (a.atomic) atomicAdd(o, rowsum);
          else *o = rowsum;
        }
        rowsum = 0.f;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

template <int D, bool BF16>
int launch_tc(const void* V, int n_groups, int rows, const void* W, int Hq, int Hkv, int hidden, float* out,
              long long ogs, int nparts, long long pstride, int32_t* status, cudaStream_t s) {
  constexpr int KB = D / 64;
  // at least 120 KB so that two CTAs never share an SM (each holds all 512 TMEM columns)
  constexpr size_t SMEM_USE = 1024 + (size_t)kMT * KB * kBM * 128 + (size_t)kNST * (kBN / 64) * D * 128 + 256;
  constexpr size_t SMEM = SMEM_USE > 120 * 1024 ? SMEM_USE : 120 * 1024;
  auto kern = vwo_tc_kernel<D, BF16>;
  static QeOnce once;
  static int sms_of[QE_MAX_DEVICES];
  int dev = 0;
  int e = qe_once_per_device(once, &dev, [&](int d) {
    QE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM));
    QE_CUDA_TRY(cudaDeviceGetAttribute(&sms_of[d], cudaDevAttrMultiProcessorCount, d));
    return QE_OK;
  });
  if (e) return e;
  const int sms = sms_of[dev];
  CUtensorMap tmV, tmW;
  e = make_map(&tmV, V, BF16, D, (uint64_t)n_groups * rows, 64, kBM);
  if (e) return e;
  e = make_map(&tmW, W, BF16, hidden, (uint64_t)Hq * D, 64, D);
  if (e) return e;
  VwoArgs a{};
  a.out = out;
  a.ogs = ogs;
  a.rows = rows;
  a.G = Hq / Hkv;
  a.Hkv = Hkv;
  a.ntiles_per_head = hidden / kBN;
  a.mpairs = (rows + kMT * kBM - 1) / (kMT * kBM);
  a.ntot = a.G * a.ntiles_per_head;
  const long long items = (long long)n_groups * a.mpairs;
  // Few row blocks: split the columns over several CTAs, at whole query heads only (a divisor
  // of G), so that every output element is written by one CTA and results do not depend on
  // the order in which CTAs finish.
  int want = 1;
  if (items < 2ll * sms) want = (int)((2ll * sms + items - 1) / items);
  int nsplit = 1;
  for (int d = 1; d <= a.G; ++d)
    if (a.G % d == 0 && d <= want) nsplit = d;
  // with column parts, every head's tiles are split into nparts ranges of their own
  if (nparts > 1) {
    if (a.ntiles_per_head % nparts) return QE_ERR_UNSUPPORTED_SHAPE;
    nsplit = a.G * nparts;
  }
  a.nsplit = nsplit;
  a.nparts = nparts > 1 ? nparts : 1;
  a.pstride = pstride;
  a.atomic = 0;
  a.status = status;
  kern<<<(unsigned)(items * nsplit), kThreads, SMEM, s>>>(tmV, tmW, a);
  return cudaGetLastError() == cudaSuccess ? QE_OK : QE_ERR_CUDA;
}

}  // namespace

// Tensor-core path for hidden % 128 == 0; status may be NULL (errors then go nowhere).
int launch_vwo_tc(const void* V, int n_groups, int rows, int D, int dtype, const void* W_O, int Hq, int Hkv,
                  int hidden, float* out, long long ogs, int32_t* status, cudaStream_t s, int nparts,
                  long long pstride) {
  if (hidden % kBN) return QE_ERR_UNSUPPORTED_SHAPE;
  if ((long long)n_groups * rows > 0x7fffffffll) return QE_ERR_UNSUPPORTED_SHAPE;
  const bool bf = dtype == QE_BF16;
  if (D == 128)
    return bf ? launch_tc<128, true>(V, n_groups, rows, W_O, Hq, Hkv, hidden, out, ogs, nparts, pstride, status, s)
              : launch_tc<128, false>(V, n_groups, rows, W_O, Hq, Hkv, hidden, out, ogs, nparts, pstride, status, s);
  return bf ? launch_tc<64, true>(V, n_groups, rows, W_O, Hq, Hkv, hidden, out, ogs, nparts, pstride, status, s)
            : launch_tc<64, false>(V, n_groups, rows, W_O, Hq, Hkv, hidden, out, ogs, nparts, pstride, status, s);
}

// Column parts for a launch of few row blocks: the largest power of two that divides the
// hidden tiles of a head and keeps items * G * parts within one wave of the SMs.
int vwo_tc_parts(int n_groups, int rows, int Hq, int Hkv, int hidden, int max_parts, int sms) {
  if (hidden % kBN) return 1;
  const long long items = (long long)n_groups * ((rows + kMT * kBM - 1) / (kMT * kBM));
  const int G = Hq / Hkv, tph = hidden / kBN;
  int P = 1;
  while (2 * P <= max_parts && tph % (2 * P) == 0 && items * G * 2 * P <= sms) P *= 2;
  return P;
}
