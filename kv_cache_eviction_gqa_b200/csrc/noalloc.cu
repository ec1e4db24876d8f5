// Allocation-free variant of qe_decode_attend_and_score.
//
// Some callers cannot give this library extra device memory at run time: for example an
// inference engine that hands a plugin only its input and output buffers and forbids any
// allocation while a request executes, or a process whose device memory is entirely owned
// by another allocator. For them this entry point runs the split-K decode kernel with its
// per-call scratch (per-window score partials and tail-token scores) in a fixed array that is
// part of the library image, instead of the scratch region of the context workspace. The
// cache state itself still lives in the caller's workspace, and q / out are the caller's
// buffers. (The splits of a unit merge through distributed shared memory, so no split
// partials or completion counters are needed.)
//
// The array is a file-scope __device__ object of kStaticScratchBytes: every GPU that loads
// this library holds that much memory until the process exits. All calls on one GPU share
// it, and it keeps whatever the last call left. Nothing needs clearing: a call folds a window
// partial into the cumulative scores only if every CTA of the window's unit finished all its
// waits, and each such partial was written earlier in the same call; when a bounded wait gives
// up (QE_ERR_TIMEOUT in the status word) the step's score update is skipped for that unit, so
// values left by another call are never read into the scores. Two calls whose kernels overlap
// on the same GPU (for example two contexts on two streams) race on the array: issue them one
// after the other. A config whose scratch needs more
// than kStaticScratchBytes is rejected with QE_ERR_INVALID_ARG before anything is enqueued.
// The first call on a device looks up the array's device address (cudaGetSymbolAddress with
// that device current) and caches it; make that first call before any stream capture.
#include "qe_internal.cuh"

namespace {

constexpr size_t kStaticScratchBytes = 16u << 20;  // 16 MiB
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

uint8_t* g_scratch_ptr[QE_MAX_DEVICES];  // device address of g_static_scratch per device

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Device address of the static scratch on the current device. The first call on a device
// resolves it with cudaGetSymbolAddress (with that device current) and caches it.
int static_scratch(uint8_t** out) {
  static QeOnce once;
  int dev = 0;
  const int e = qe_once_per_device(once, &dev, [](int d) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return (int)QE_ERR_CUDA;
    g_scratch_ptr[d] = static_cast<uint8_t*>(p);
    return (int)QE_OK;
  });
  if (e) return e;
  *out = g_scratch_ptr[dev];
  return QE_OK;
}

}  // namespace

extern "C" QE_API int qe_decode_attend_and_score_noalloc(qe_ctx* c, const void* q, float* out,
                                                         qe_stream_t s) {
  if (!c || !q || !out) return QE_ERR_INVALID_ARG;
  // the decode kernel's per-call scratch, laid out like the workspace scratch
  const size_t U = c->lay.units, G = c->G, w = c->cfg.window, W = c->lay.max_windows;
  const size_t b_win = round256(U * W * win_part_floats(c->cfg.D, c->G) * 4);
  const size_t b_tail = round256(U * w * G * 4);
  if (b_win + b_tail > kStaticScratchBytes) return QE_ERR_INVALID_ARG;
  uint8_t* base = nullptr;
  int e = static_scratch(&base);
  if (e) return e;
  // run the regular entry point with the context's scratch pointers aimed at the array
  float* wp = c->win_part;
  float* ts = c->tail_s;
  c->win_part = reinterpret_cast<float*>(base);
  c->tail_s = reinterpret_cast<float*>(base + b_win);
  e = qe_decode_attend_and_score(c, q, out, s);
  c->win_part = wp;
  c->tail_s = ts;
  return e;
}
