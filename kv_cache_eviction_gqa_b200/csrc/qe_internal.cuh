// Internal declarations shared by the CUDA translation units of libqevict.
// Device helpers (bulk copies, mbarriers, bounded waits, dtype conversion) and the
// host-side context. Nothing here is part of the C ABI (see include/qevict.h).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <mutex>

#include "../../include/qevict.h"

#define QE_PAGE 16

// floats of one window's score partials in the decode kernel's scratch: {max, sum p, sum p n}
// per query head of the group, relative to that max
__host__ __device__ constexpr int win_part_floats(int D, int G) { return (void)D, 3 * G; }
// column parts of a completed window's V W_O norms (partial row sums, added by finalize)
constexpr int kTailNormParts = 8;
#define QE_MAX_G 8
#define QE_MAX_SPLITS 64

// status word slots
#define QE_ST_CODE 0
#define QE_ST_DETAIL 1

// ----------------------------------------------------------------------------
// host context
// ----------------------------------------------------------------------------
struct qe_ctx {
  qe_config cfg;
  qe_layout lay;
  int G;
  uint8_t* ws;          // workspace base [dev]
  const void* W_O;      // [Hq*D][hidden] [dev]
  // host mirror of the length / step (identical for every unit)
  int n;                // tokens per unit
  int step;             // decode steps since prefill
  int complete;         // windows complete and in the tier lists (the tail is window `complete`)
  int loaded;           // prefill done
  int n_full_max;       // upper bound of full-tier windows over units
  int n_int2_max;       // upper bound of INT2-tier windows over units
  int counts_exact;     // every unit holds exactly n_full_max / n_int2_max windows (per-unit
                        // routing keeps the units in step; host-given transitions and the
                        // global budget do not)
  cudaStream_t last_stream;
  // scratch sub-buffers [dev]
  float* win_part;      // [U][max_windows][win_part_floats(D, G)]
  float* tail_s;        // [U][window][G]
  int32_t* xlist;       // [U][max_windows] transition lists (quantise) [win]
  int32_t* plist;       // [U][max_windows] transition lists (promote)  [win]
  int32_t* xcount;      // [U][4] counts: quantise, promote
  int32_t* host_ids;    // [max_windows] staging for host-given window ids
  uint8_t* tailV;       // [Hkv][B][window][D] dtype: V of the tail window (for its norms)
  float* tail_norm;     // [kTailNormParts][Hkv][B*window][G] partial norms of a just-completed window
  // typed views of the state arrays
  template <typename T> T* at(size_t off) const { return reinterpret_cast<T*>(ws + off); }
};

// ----------------------------------------------------------------------------
// device state view passed by value to kernels
// ----------------------------------------------------------------------------
struct DevState {
  uint8_t* pages;       // [U][P][2][16][D] T
  int32_t* page_free;   // [U][P]
  int32_t* win_pages;   // [U][Wmax][ppw]
  uint8_t* win_tier;    // [U][Wmax]
  int32_t* win_slot;    // [U][Wmax]
  uint8_t* slots;       // [U][S][window*D]
  int32_t* slot_free;   // [U][S]
  float* mass;          // [U][Wmax]
  float* pert;          // [U][Wmax]
  float* norms;         // [U][max_ctx][G]
  int32_t* full_list;   // [U][Wmax]
  int32_t* int2_list;   // [U][Wmax]
  float* tail_p;        // [U][window][G]
  int32_t* stacks;      // [U][4] page top, slot top, n_full, n_int2
  int32_t* route_stats; // [U][8]
  int32_t* status;      // [4]
  int P, S, Wmax, ppw, window, D, G, max_ctx, norm_pitch, U, B, Hkv, Hq;
  size_t page_bytes, slot_bytes;
};

DevState make_state(const qe_ctx* c);

// ----------------------------------------------------------------------------
// device helpers
// ----------------------------------------------------------------------------
__device__ __forceinline__ void qe_record_error(int32_t* status, int code, int detail) {
  if (atomicCAS(&status[QE_ST_CODE], 0, code) == 0) status[QE_ST_DETAIL] = detail;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// 1-D bulk copy global -> shared of this CTA, completion signalled on an mbarrier.
// src, dst 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// One test of an mbarrier phase. The thread may be suspended in it until the phase completes
// or about a millisecond has passed (the suspend-time hint), so a waiting warp takes no issue
// slots from the others while its copy is in flight.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(1000000u)
      : "memory");
  return ok != 0;
}

// Bounded wait on an mbarrier phase: gives up after ~2^31 clock cycles (about a
// second), records QE_ERR_TIMEOUT and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, int32_t* status,
                                                  int where) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > (1ll << 31)) {
      qe_record_error(status, QE_ERR_TIMEOUT, where);
      return false;
    }
  }
  return true;
}

// dtype traits: 16-bit element -> float
template <typename T> struct Elem;
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float lo(uint32_t w) { return __uint_as_float(w << 16); }
  static __device__ __forceinline__ float hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
  static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};
template <> struct Elem<__half> {
  static __device__ __forceinline__ float lo(uint32_t w) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xffffu)));
  }
  static __device__ __forceinline__ float hi(uint32_t w) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16)));
  }
  static __device__ __forceinline__ float to_f(__half x) { return __half2float(x); }
  static __device__ __forceinline__ __half from_f(float x) { return __float2half_rn(x); }
};

// ----------------------------------------------------------------------------
// host helpers
// ----------------------------------------------------------------------------
#define QE_CUDA_TRY(expr)                         \
  do {                                            \
    cudaError_t _e = (expr);                      \
    if (_e != cudaSuccess) return QE_ERR_CUDA;    \
  } while (0)

// One-time host set-up of a kernel (attributes, occupancy queries) for each device this
// process launches on. setup(dev) runs under a lock on the first call for that device and is
// retried on the next call if it failed; results it stores per device are visible to every
// thread once this returns QE_OK.
#define QE_MAX_DEVICES 64
struct QeOnce {
  std::mutex mu;
  bool done[QE_MAX_DEVICES] = {};
};
template <typename F>
int qe_once_per_device(QeOnce& once, int* dev_out, F&& setup) {
  int dev = 0;
  QE_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= QE_MAX_DEVICES) return QE_ERR_UNSUPPORTED_SHAPE;
  *dev_out = dev;
  std::lock_guard<std::mutex> g(once.mu);
  if (once.done[dev]) return QE_OK;
  const int e = setup(dev);
  if (e == QE_OK) once.done[dev] = true;
  return e;
}

static inline bool qe_aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

// launchers (defined in the .cu files)
int launch_prefill(qe_ctx* c, const void* K, const void* V, int ctx_len, const float* norms,
                   cudaStream_t st);
int launch_append(qe_ctx* c, const void* k, const void* v, cudaStream_t st);
// k_new / v_new non-null: the decode launch also appends the step's token (position c->n - 1,
// c->n already advanced by the caller)
int launch_decode(qe_ctx* c, const void* q, float* out, cudaStream_t st, const void* k_new = nullptr,
                  const void* v_new = nullptr);
int launch_finalize(qe_ctx* c, int tail_win, cudaStream_t st);
int launch_route(qe_ctx* c, cudaStream_t st);
// route with the tier of every candidate window given: window w of unit (b, kvh) takes
// decided[b * dec_stride + kvh * max_windows + w] (QE_TIER_FULL, _INT2 or _EVICTED)
int launch_route_decided(qe_ctx* c, const uint8_t* decided, size_t dec_stride, cudaStream_t st);
int launch_set_tier(qe_ctx* c, int unit, const int32_t* ids_host, int n, int tier, cudaStream_t st);
int launch_vwo(const void* V, int n_groups, int rows, int D, int dtype, const void* W_O, int Hq,
               int Hkv, int hidden, float* out, long long out_group_stride, int32_t* status,
               cudaStream_t st);
int launch_vwo_tc(const void* V, int n_groups, int rows, int D, int dtype, const void* W_O, int Hq,
                  int Hkv, int hidden, float* out, long long out_group_stride, int32_t* status,
                  cudaStream_t st, int nparts = 1, long long part_stride = 0);
// column parts for the tensor-core launch of few rows (1 when the launch already fills the GPU)
int vwo_tc_parts(int n_groups, int rows, int Hq, int Hkv, int hidden, int max_parts, int sms);
int launch_int2_quantize(const void* x, int T, int D, int dtype, uint8_t* codes, uint32_t* meta,
                         cudaStream_t st);
int launch_ledger_read(qe_ctx* c, int unit, int win, uint8_t* codes_k, uint32_t* meta_k, uint8_t* codes_v,
                       uint32_t* meta_v, int32_t* found, cudaStream_t st);
