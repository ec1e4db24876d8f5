// C ABI of libqevict: configuration checks, workspace layout, context lifetime and the
// host-side sequencing of one decode step. Every kernel launch lives in the other files.
#include <stdlib.h>
#include <string.h>

#include "qe_internal.cuh"

namespace {

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int check_config(const qe_config* c) {
  if (!c) return QE_ERR_INVALID_ARG;
  if (c->B < 1 || c->Hq < 1 || c->Hkv < 1 || c->Hq % c->Hkv) return QE_ERR_INVALID_ARG;
  const int G = c->Hq / c->Hkv;
  if (G > QE_MAX_G) return QE_ERR_UNSUPPORTED_SHAPE;
  if (c->D != 64 && c->D != 128) return QE_ERR_UNSUPPORTED_SHAPE;
  if (c->dtype != QE_FP16 && c->dtype != QE_BF16) return QE_ERR_INVALID_ARG;
  if (c->page != QE_PAGE) return QE_ERR_UNSUPPORTED_SHAPE;
  if (c->window != 16 && c->window != 32 && c->window != 64) return QE_ERR_UNSUPPORTED_SHAPE;
  if (c->full_windows < 0 || c->int2_windows < 0) return QE_ERR_INVALID_ARG;
  if (!(c->alpha >= 0.f && c->alpha <= 1.f)) return QE_ERR_INVALID_ARG;
  if (c->route_every < 0) return QE_ERR_INVALID_ARG;  // 0: the caller routes
  if (c->hidden < 1 || c->hidden % 64) return QE_ERR_UNSUPPORTED_SHAPE;
  if (c->max_ctx < c->window) return QE_ERR_INVALID_ARG;
  if (c->pages_per_unit < c->window / QE_PAGE) return QE_ERR_INVALID_ARG;
  if (c->slots_per_unit < 0) return QE_ERR_INVALID_ARG;
  if (c->max_splits < 1 || c->max_splits > QE_MAX_SPLITS) return QE_ERR_INVALID_ARG;
  return QE_OK;
}

// Sizes of the scratch buffers, in workspace order (qe_plan reserves them, qe_create points
// into them): window partials (win_part_floats per window),
// tail scores, quantise list, promote list, list counts, host-given ids, tail-window V rows,
// tail-window norms.
constexpr int kScratchParts = 8;
void scratch_sizes(const qe_config* c, size_t (&sz)[kScratchParts]) {
  const size_t G = c->Hq / c->Hkv, D = c->D, w = c->window;
  const size_t U = (size_t)c->B * c->Hkv;
  const size_t Wmax = (c->max_ctx + w - 1) / w;
  sz[0] = U * Wmax * win_part_floats((int)D, (int)G) * 4;
  sz[1] = U * w * G * 4;
  sz[2] = U * Wmax * 4;
  sz[3] = U * Wmax * 4;
  sz[4] = U * 4 * 4;
  sz[5] = Wmax * 4;
  sz[6] = (size_t)c->Hkv * c->B * w * D * 2;
  sz[7] = (size_t)kTailNormParts * c->Hkv * c->B * w * G * 4;
}

int finalize_tail(qe_ctx* c, cudaStream_t st) {
  int e = launch_finalize(c, c->complete, st);
  if (e) return e;
  c->complete += 1;
  c->n_full_max += 1;
  return QE_OK;
}

}  // namespace

extern "C" {

QE_API int qe_plan(const qe_config* c, qe_layout* L) {
  int e = check_config(c);
  if (e) return e;
  if (!L) return QE_ERR_INVALID_ARG;
  memset(L, 0, sizeof(*L));
  const size_t U = (size_t)c->B * c->Hkv, G = c->Hq / c->Hkv, D = c->D, P = c->pages_per_unit,
               S = c->slots_per_unit, w = c->window;
  const size_t Wmax = (c->max_ctx + w - 1) / w, ppw = w / QE_PAGE;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  L->pages = take(U * P * 2 * QE_PAGE * D * 2);
  L->page_free = take(U * P * 4);
  L->win_pages = take(U * Wmax * ppw * 4);
  L->win_tier = take(U * Wmax);
  L->win_slot = take(U * Wmax * 4);
  L->slots = take(U * S * w * D);
  L->slot_free = take(U * S * 4);
  L->mass = take(U * Wmax * 4);
  L->pert = take(U * Wmax * 4);
  L->norms = take(U * align_up((size_t)c->max_ctx, 16) * G * 4);
  L->full_list = take(U * Wmax * 4);
  L->int2_list = take(U * Wmax * 4);
  L->tail_p = take(U * w * G * 4);
  L->stacks = take(U * 4 * 4);
  L->route_stats = take(U * 8 * 4);
  L->status = take(16);
  const size_t s0 = off;
  L->scratch = s0;
  size_t sz[kScratchParts];
  scratch_sizes(c, sz);
  for (int i = 0; i < kScratchParts; ++i) take(sz[i]);
  L->scratch_bytes = off - s0;
  L->total = off;
  L->max_windows = (int)Wmax;
  L->units = (int)U;
  return QE_OK;
}

QE_API size_t qe_workspace_bytes(const qe_config* c) {
  qe_layout L;
  return qe_plan(c, &L) == QE_OK ? L.total : 0;
}

QE_API int qe_create(const qe_config* cfg, void* ws, size_t bytes, const void* W_O, qe_ctx** out) {
  if (!cfg || !ws || !W_O || !out) return QE_ERR_INVALID_ARG;
  if (!qe_aligned(ws, 256) || !qe_aligned(W_O, 16)) return QE_ERR_INVALID_ARG;
  qe_layout L;
  int e = qe_plan(cfg, &L);
  if (e) return e;
  if (bytes < L.total) return QE_ERR_WORKSPACE;
  qe_ctx* c = (qe_ctx*)calloc(1, sizeof(qe_ctx));
  if (!c) return QE_ERR_INVALID_ARG;
  c->cfg = *cfg;
  c->lay = L;
  c->G = cfg->Hq / cfg->Hkv;
  c->ws = (uint8_t*)ws;
  c->W_O = W_O;
  const size_t U = L.units, G = c->G, D = cfg->D, w = cfg->window, Wmax = L.max_windows;
  size_t off = L.scratch;
  auto take = [&](size_t b) {
    size_t o = off;
    off = align_up(off + b, 256);
    return c->ws + o;
  };
  size_t sz[kScratchParts];
  scratch_sizes(cfg, sz);
  c->win_part = (float*)take(sz[0]);
  c->tail_s = (float*)take(sz[1]);
  c->xlist = (int32_t*)take(sz[2]);
  c->plist = (int32_t*)take(sz[3]);
  c->xcount = (int32_t*)take(sz[4]);
  c->host_ids = (int32_t*)take(sz[5]);
  c->tailV = (uint8_t*)take(sz[6]);
  c->tail_norm = (float*)take(sz[7]);
  *out = c;
  return QE_OK;
}

QE_API int qe_destroy(qe_ctx* c) {
  if (!c) return QE_ERR_INVALID_ARG;
  free(c);
  return QE_OK;
}

QE_API int qe_load_prefill(qe_ctx* c, const void* K, const void* V, int ctx_len, const float* norms,
                           qe_stream_t s) {
  if (!c || !K || !V) return QE_ERR_INVALID_ARG;
  if (!qe_aligned(K, 16) || !qe_aligned(V, 16) || !qe_aligned(norms, 4)) return QE_ERR_INVALID_ARG;
  if (ctx_len < 1 || ctx_len > c->cfg.max_ctx) return QE_ERR_INVALID_ARG;
  if ((ctx_len + QE_PAGE - 1) / QE_PAGE > c->cfg.pages_per_unit) return QE_ERR_POOL_EXHAUSTED;
  cudaStream_t st = (cudaStream_t)s;
  int e = launch_prefill(c, K, V, ctx_len, norms, st);
  if (e) return e;
  c->n = ctx_len;
  c->complete = ctx_len / c->cfg.window;
  c->step = 0;
  c->loaded = 1;
  c->n_full_max = ctx_len / c->cfg.window;
  c->n_int2_max = 0;
  c->counts_exact = 1;
  c->last_stream = st;
  return QE_OK;
}

QE_API int qe_kv_append(qe_ctx* c, const void* k, const void* v, qe_stream_t s) {
  if (!c || !k || !v) return QE_ERR_INVALID_ARG;
  if (!c->loaded) return QE_ERR_STATE;
  if (!qe_aligned(k, 16) || !qe_aligned(v, 16)) return QE_ERR_INVALID_ARG;
  if (c->n >= c->cfg.max_ctx) return QE_ERR_POOL_EXHAUSTED;
  cudaStream_t st = (cudaStream_t)s;
  int e;
  // a complete tail that no decode call has finalised yet is finalised first
  if (c->n - c->complete * c->cfg.window == c->cfg.window && (e = finalize_tail(c, st))) return e;
  e = launch_append(c, k, v, st);
  if (e) return e;
  c->n += 1;
  c->last_stream = st;
  return QE_OK;
}

QE_API int qe_decode_attend_and_score(qe_ctx* c, const void* q, float* out, qe_stream_t s) {
  if (!c || !q || !out) return QE_ERR_INVALID_ARG;
  if (!c->loaded) return QE_ERR_STATE;
  if (!qe_aligned(q, 16) || !qe_aligned(out, 16)) return QE_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)s;
  int e = launch_decode(c, q, out, st);
  if (e) return e;
  c->last_stream = st;
  // the tail window just became complete: compute its norms, move it to the full tier
  if (c->n - c->complete * c->cfg.window == c->cfg.window) return finalize_tail(c, st);
  return QE_OK;
}

QE_API int qe_route_windows(qe_ctx* c, qe_stream_t s) {
  if (!c) return QE_ERR_INVALID_ARG;
  if (!c->loaded) return QE_ERR_STATE;
  cudaStream_t st = (cudaStream_t)s;
  int e = launch_route(c, st);
  if (e) return e;
  const int tot = c->n_full_max + c->n_int2_max;
  c->n_full_max = tot < c->cfg.full_windows ? tot : c->cfg.full_windows;
  const int rest = tot - c->n_full_max;
  c->n_int2_max = rest < c->cfg.int2_windows ? rest : c->cfg.int2_windows;
  c->last_stream = st;
  return QE_OK;
}

QE_API int qe_decode_step(qe_ctx* c, const void* q, const void* k, const void* v, float* out,
                          qe_stream_t s) {
  // append + decode in one launch: the CTA that streams a unit's tail window first writes the
  // new token (same results as qe_kv_append followed by qe_decode_attend_and_score)
  if (!c || !q || !out || !k || !v) return QE_ERR_INVALID_ARG;
  if (!c->loaded) return QE_ERR_STATE;
  if (!qe_aligned(q, 16) || !qe_aligned(out, 16) || !qe_aligned(k, 16) || !qe_aligned(v, 16))
    return QE_ERR_INVALID_ARG;
  if (c->n >= c->cfg.max_ctx) return QE_ERR_POOL_EXHAUSTED;
  cudaStream_t st = (cudaStream_t)s;
  int e;
  if (c->n - c->complete * c->cfg.window == c->cfg.window && (e = finalize_tail(c, st))) return e;
  c->n += 1;
  e = launch_decode(c, q, out, st, k, v);
  if (e) {
    c->n -= 1;
    return e;
  }
  c->last_stream = st;
  if (c->n - c->complete * c->cfg.window == c->cfg.window && (e = finalize_tail(c, st))) return e;
  if (c->cfg.route_every > 0 && c->step % c->cfg.route_every == 0) {
    e = qe_route_windows(c, s);
    if (e) return e;
  }
  c->step += 1;
  return QE_OK;
}

QE_API int qe_quantize_once(qe_ctx* c, int unit, const int32_t* ids, int n, qe_stream_t s) {
  if (!c || (!ids && n > 0) || n < 0) return QE_ERR_INVALID_ARG;
  if (!c->loaded) return QE_ERR_STATE;
  if (unit < 0 || unit >= c->lay.units || n > c->lay.max_windows) return QE_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i)
    if (ids[i] < 0 || ids[i] >= c->lay.max_windows) return QE_ERR_INVALID_ARG;
  if (n == 0) return QE_OK;
  int e = launch_set_tier(c, unit, ids, n, QE_TIER_INT2, (cudaStream_t)s);
  if (e) return e;
  c->n_int2_max += n;
  c->counts_exact = 0;
  c->last_stream = (cudaStream_t)s;
  return QE_OK;
}

QE_API int qe_promote(qe_ctx* c, int unit, const int32_t* ids, int n, qe_stream_t s) {
  if (!c || (!ids && n > 0) || n < 0) return QE_ERR_INVALID_ARG;
  if (!c->loaded) return QE_ERR_STATE;
  if (unit < 0 || unit >= c->lay.units || n > c->lay.max_windows) return QE_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i)
    if (ids[i] < 0 || ids[i] >= c->lay.max_windows) return QE_ERR_INVALID_ARG;
  if (n == 0) return QE_OK;
  int e = launch_set_tier(c, unit, ids, n, QE_TIER_FULL, (cudaStream_t)s);
  if (e) return e;
  c->n_full_max += n;
  c->counts_exact = 0;
  c->last_stream = (cudaStream_t)s;
  return QE_OK;
}

QE_API int qe_int2_quantize(const void* x, int T, int D, int dtype, uint8_t* codes, uint32_t* meta,
                            qe_stream_t s) {
  if (!x || !codes || !meta || T < 0 || D < 16 || D % 16 || D > 1024) return QE_ERR_INVALID_ARG;
  if (dtype != QE_FP16 && dtype != QE_BF16) return QE_ERR_INVALID_ARG;
  if (T == 0) return QE_OK;
  return launch_int2_quantize(x, T, D, dtype, codes, meta, (cudaStream_t)s);
}

QE_API int qe_vwo_l1norm(const void* V, int n_groups, int rows, int D, int dtype, const void* W_O,
                         int Hq, int Hkv, int hidden, float* out, long long out_group_stride,
                         qe_stream_t s) {
  if (!V || !W_O || !out || n_groups < 1 || rows < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv)
    return QE_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return QE_ERR_UNSUPPORTED_SHAPE;
  if (Hq / Hkv > QE_MAX_G || hidden < 64 || hidden % 64) return QE_ERR_UNSUPPORTED_SHAPE;
  if (dtype != QE_FP16 && dtype != QE_BF16) return QE_ERR_INVALID_ARG;
  if (!qe_aligned(V, 16) || !qe_aligned(W_O, 16)) return QE_ERR_INVALID_ARG;
  if (out_group_stride < (long long)rows * (Hq / Hkv)) return QE_ERR_INVALID_ARG;
  if (rows == 0) return QE_OK;
  return launch_vwo(V, n_groups, rows, D, dtype, W_O, Hq, Hkv, hidden, out, out_group_stride, nullptr,
                    (cudaStream_t)s);
}

QE_API int qe_ledger_read(qe_ctx* c, int unit, int win, uint8_t* codes_k, uint32_t* meta_k, uint8_t* codes_v,
                          uint32_t* meta_v, int32_t* found, qe_stream_t s) {
  if (!c || !codes_k || !meta_k || !codes_v || !meta_v || !found) return QE_ERR_INVALID_ARG;
  if (!c->loaded) return QE_ERR_STATE;
  if (unit < 0 || unit >= c->lay.units || win < 0 || win >= c->lay.max_windows) return QE_ERR_INVALID_ARG;
  if (!qe_aligned(meta_k, 4) || !qe_aligned(meta_v, 4) || !qe_aligned(found, 4)) return QE_ERR_INVALID_ARG;
  c->last_stream = (cudaStream_t)s;
  return launch_ledger_read(c, unit, win, codes_k, meta_k, codes_v, meta_v, found, (cudaStream_t)s);
}

// ---- checkpoint of a context ----
namespace {
struct StateHeader {  // 256 bytes, little endian as the host
  char magic[4];      // "QEVS"
  int32_t version;    // 1
  qe_config cfg;
  int32_t n, step, complete, n_full_max, n_int2_max, counts_exact;
  uint64_t state_bytes;  // bytes of workspace that follow the header (all of it)
};
constexpr size_t kHeaderBytes = 256;
static_assert(sizeof(StateHeader) <= kHeaderBytes, "state header");
constexpr int32_t kStateVersion = 1;
bool same_config(const qe_config& a, const qe_config& b) { return memcmp(&a, &b, sizeof(qe_config)) == 0; }
}  // namespace

QE_API size_t qe_state_bytes(const qe_ctx* c) { return c ? kHeaderBytes + c->lay.total : 0; }

QE_API int qe_state_export(qe_ctx* c, void* dst, size_t bytes, qe_stream_t s) {
  if (!c || !dst) return QE_ERR_INVALID_ARG;
  if (!c->loaded) return QE_ERR_STATE;
  if (bytes < qe_state_bytes(c)) return QE_ERR_WORKSPACE;
  StateHeader h;
  memset(&h, 0, sizeof(h));
  memcpy(h.magic, "QEVS", 4);
  h.version = kStateVersion;
  h.cfg = c->cfg;
  h.n = c->n;
  h.step = c->step;
  h.complete = c->complete;
  h.n_full_max = c->n_full_max;
  h.n_int2_max = c->n_int2_max;
  h.counts_exact = c->counts_exact;
  h.state_bytes = c->lay.total;
  cudaStream_t st = (cudaStream_t)s;
  // the header from pageable host memory: the copy consumes it before returning
  QE_CUDA_TRY(cudaMemcpyAsync(dst, &h, sizeof(h), cudaMemcpyDefault, st));
  QE_CUDA_TRY(cudaMemcpyAsync((uint8_t*)dst + kHeaderBytes, c->ws, c->lay.total, cudaMemcpyDefault, st));
  c->last_stream = st;
  return QE_OK;
}

QE_API int qe_state_import(qe_ctx* c, const void* src, size_t bytes, qe_stream_t s) {
  if (!c || !src) return QE_ERR_INVALID_ARG;
  if (bytes < kHeaderBytes) return QE_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)s;
  StateHeader h;
  QE_CUDA_TRY(cudaMemcpyAsync(&h, src, sizeof(h), cudaMemcpyDefault, st));
  QE_CUDA_TRY(cudaStreamSynchronize(st));
  if (memcmp(h.magic, "QEVS", 4) != 0 || h.version != kStateVersion) return QE_ERR_INVALID_ARG;
  if (!same_config(h.cfg, c->cfg) || h.state_bytes != c->lay.total) return QE_ERR_INVALID_ARG;
  if (bytes < kHeaderBytes + h.state_bytes) return QE_ERR_WORKSPACE;
  QE_CUDA_TRY(cudaMemcpyAsync(c->ws, (const uint8_t*)src + kHeaderBytes, h.state_bytes, cudaMemcpyDefault, st));
  c->n = h.n;
  c->step = h.step;
  c->complete = h.complete;
  c->n_full_max = h.n_full_max;
  c->n_int2_max = h.n_int2_max;
  c->counts_exact = h.counts_exact;
  c->loaded = 1;
  c->last_stream = st;
  return QE_OK;
}

QE_API int qe_status(qe_ctx* c, int* detail) {
  if (!c) return QE_ERR_INVALID_ARG;
  int32_t h[4] = {0, 0, 0, 0};
  if (cudaStreamSynchronize(c->last_stream) != cudaSuccess) return QE_ERR_CUDA;
  if (cudaMemcpy(h, c->ws + c->lay.status, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess)
    return QE_ERR_CUDA;
  if (detail) *detail = h[QE_ST_DETAIL];
  return h[QE_ST_CODE];
}

QE_API int qe_step_index(const qe_ctx* c) { return c ? c->step : QE_ERR_INVALID_ARG; }
QE_API int qe_length(const qe_ctx* c) { return c ? c->n : QE_ERR_INVALID_ARG; }
QE_API int qe_list_counts(const qe_ctx* c, int* nf, int* nq) {
  if (!c) return QE_ERR_INVALID_ARG;
  if (nf) *nf = c->n_full_max;
  if (nq) *nq = c->n_int2_max;
  return QE_OK;
}

QE_API const char* qe_strerror(int code) {
  switch (code) {
    case QE_OK: return "ok";
    case QE_ERR_INVALID_ARG: return "invalid argument";
    case QE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case QE_ERR_POOL_EXHAUSTED: return "page pool exhausted";
    case QE_ERR_LEDGER_FULL: return "INT2 ledger full";
    case QE_ERR_CUDA: return "CUDA runtime error";
    case QE_ERR_TIMEOUT: return "bounded device wait gave up";
    case QE_ERR_DEVICE_FAULT: return "device index out of range";
    case QE_ERR_WORKSPACE: return "workspace too small";
    case QE_ERR_STATE: return "call out of order";
    default: return "unknown error";
  }
}

}  // extern "C"

DevState make_state(const qe_ctx* c) {
  DevState s;
  const qe_layout& L = c->lay;
  s.pages = c->ws + L.pages;
  s.page_free = c->at<int32_t>(L.page_free);
  s.win_pages = c->at<int32_t>(L.win_pages);
  s.win_tier = c->at<uint8_t>(L.win_tier);
  s.win_slot = c->at<int32_t>(L.win_slot);
  s.slots = c->ws + L.slots;
  s.slot_free = c->at<int32_t>(L.slot_free);
  s.mass = c->at<float>(L.mass);
  s.pert = c->at<float>(L.pert);
  s.norms = c->at<float>(L.norms);
  s.full_list = c->at<int32_t>(L.full_list);
  s.int2_list = c->at<int32_t>(L.int2_list);
  s.tail_p = c->at<float>(L.tail_p);
  s.stacks = c->at<int32_t>(L.stacks);
  s.route_stats = c->at<int32_t>(L.route_stats);
  s.status = c->at<int32_t>(L.status);
  s.P = c->cfg.pages_per_unit;
  s.S = c->cfg.slots_per_unit;
  s.Wmax = L.max_windows;
  s.ppw = c->cfg.window / QE_PAGE;
  s.window = c->cfg.window;
  s.D = c->cfg.D;
  s.G = c->G;
  s.max_ctx = c->cfg.max_ctx;
  s.norm_pitch = (c->cfg.max_ctx + 15) / 16 * 16;
  s.U = L.units;
  s.B = c->cfg.B;
  s.Hkv = c->cfg.Hkv;
  s.Hq = c->cfg.Hq;
  s.page_bytes = (size_t)2 * QE_PAGE * c->cfg.D * 2;
  s.slot_bytes = (size_t)c->cfg.window * c->cfg.D;
  return s;
}
