/*
 * qevict.h - C ABI of the tiered KV-cache decode library (libqevict.so, sm_100a).
 *
 * One decode step of grouped-query attention over a window-partitioned paged KV
 * cache that holds a full-precision tier (fp16/bf16) and a recoverable INT2 tier,
 * fused with cumulative window scoring, budgeted two-stage routing of every window
 * to full / INT2 / evicted, and a write-once INT2 ledger. Sources:
 *   "Resumo Técnico: QEvict"  - Metodologia (three tiers under a fixed budget),
 *       Mecanismos Principais (window-level routing, cumulative scoring, demotion,
 *       promotion, write-once quantisation ledger, GQA decode path).
 *   "Resumo Técnico: CriticalKV" - Framework Teórico (perturbation L = ||o - o_hat||_1,
 *       projected values V W_O), Algoritmo (two-stage greedy, b' = alpha*b, alpha = 0.5,
 *       then A_i * ||V_i W_O||_1 on the remaining budget).
 *   "Make Each Token Count" (DBTrimKV) - Metodologia 2 (retention r = beta^(t-i)),
 *       3 (one global budget M over layers and heads), 4 (paged variable-length heads).
 *
 * Conventions (every entry point):
 *   - Pointers marked [dev] are device pointers, [host] are host pointers. The caller
 *     owns every buffer; the library never allocates device memory (cudaMalloc) itself.
 *   - Every call that takes a cudaStream_t is asynchronous on that stream and returns
 *     after enqueueing. Arguments are validated on the host before anything is enqueued.
 *   - Return value: QE_OK (0) or a negative QE_ERR_*. Errors found by a kernel (pool
 *     exhausted, an index out of range, a bounded wait that gave up) are recorded in the
 *     context's device status word; read them with qe_status() after synchronising.
 *     No kernel traps or asserts; a failing kernel records the error and returns.
 *   - Row-major layouts. The cache dtype (fp16 or bf16) is fixed at qe_create.
 *   - No C++ exception crosses this boundary.
 */
#ifndef QEVICT_H
#define QEVICT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QE_API __attribute__((visibility("default")))

typedef struct CUstream_st* qe_stream_t; /* a cudaStream_t; NULL = legacy default stream */

enum {
  QE_OK = 0,
  QE_ERR_INVALID_ARG = -1,      /* NULL pointer, bad size, misaligned buffer        */
  QE_ERR_UNSUPPORTED_SHAPE = -2,/* D not in {64,128}, G > 8, window not in {16..64} */
  QE_ERR_POOL_EXHAUSTED = -3,   /* a unit's page free list ran empty (device)       */
  QE_ERR_LEDGER_FULL = -4,      /* a unit's INT2 ledger ran out of slots (device)   */
  QE_ERR_CUDA = -5,             /* a CUDA runtime call failed                        */
  QE_ERR_TIMEOUT = -6,          /* a bounded device wait gave up (device)            */
  QE_ERR_DEVICE_FAULT = -7,     /* an index read from device state was out of range  */
  QE_ERR_WORKSPACE = -8,        /* workspace smaller than qe_workspace_bytes()       */
  QE_ERR_STATE = -9             /* call out of order (e.g. decode before prefill)    */
};

enum { QE_FP16 = 0, QE_BF16 = 1 };

/* Window tiers as stored in the tier map (one byte per window). */
enum { QE_TIER_EVICTED = 0, QE_TIER_INT2 = 1, QE_TIER_FULL = 2, QE_TIER_TAIL = 3 };

/*
 * qe_config - shape and budgets of one decode context (one attention layer).
 * A "unit" is one (batch b, kv-head g) pair; units are independent and numbered
 * u = b*Hkv + g. Budgets are per unit and counted in windows.
 */
typedef struct {
  int B, Hq, Hkv, D;          /* batch, query heads, KV heads, head dim (64 or 128)      */
  int dtype;                  /* QE_FP16 or QE_BF16: cache, query and W_O element type   */
  int page;                   /* tokens per page; must be 16                              */
  int window;                 /* tokens per routing window: 16, 32 or 64                  */
  int full_windows;           /* F: full-precision budget per unit (windows)              */
  int int2_windows;           /* Q: INT2 budget per unit (windows)                        */
  float alpha;                /* stage-1 share of each budget (0.5 on the pages)          */
  int route_every;            /* R: route after attention on decode steps s % R == 0; 0: qe_decode_step never routes (the caller does, e.g. qe_route_windows_global) */
  int hidden;                 /* columns of W_O                                           */
  int max_ctx;                /* capacity in tokens per unit (prefill + decode)           */
  int pages_per_unit;         /* page-pool capacity per unit (>= ceil(prefill/16) + margin)*/
  int slots_per_unit;         /* INT2 ledger capacity per unit (>= F + Q)                 */
  int max_splits;             /* upper bound on split-K CTAs per unit (1..64; the kernel uses
                                 at most 16, one thread-block cluster per unit)             */
} qe_config;

/* Byte offsets of the state arrays inside the caller's workspace (see qe_layout). */
typedef struct {
  size_t total;               /* bytes the workspace must hold                            */
  size_t pages;               /* [U][pages_per_unit][2][16][D] cache dtype: K rows, V rows */
  size_t page_free;           /* [U][pages_per_unit] int32 free-page stack per unit       */
  size_t win_pages;           /* [U][max_windows][window/16] int32 page of each window    */
  size_t win_tier;            /* [U][max_windows] uint8 QE_TIER_*                          */
  size_t win_slot;            /* [U][max_windows] int32 ledger slot or -1                 */
  size_t slots;               /* [U][slots_per_unit][window*D] bytes: INT2 ledger entries  */
  size_t slot_free;           /* [U][slots_per_unit] int32 free-slot stack per unit       */
  size_t mass;                /* [U][max_windows] float cumulative attention mass         */
  size_t pert;                /* [U][max_windows] float cumulative perturbation score     */
  size_t norms;               /* [U][max_ctx][G] float ||V_i W_O^h||_1 per token and head */
  size_t full_list;           /* [U][max_windows] int32 windows in the full tier          */
  size_t int2_list;           /* [U][max_windows] int32 windows in the INT2 tier          */
  size_t tail_p;              /* [U][window][G] float cumulative attention of tail tokens */
  size_t stacks;              /* [U][4] int32: page-stack top, slot-stack top, -, -       */
  size_t route_stats;         /* [U][8] int32: promotions, new demotions, reused demotions,
                                 evictions, full kept, int2 kept, -, stage-1 mass x 1e6    */
  size_t status;              /* [4] int32 device status word (first error, detail)       */
  size_t scratch;             /* split-K partials, window partials, transition lists       */
  size_t scratch_bytes;
  int max_windows;            /* ceil(max_ctx / window)                                    */
  int units;                  /* B * Hkv                                                   */
} qe_layout;

typedef struct qe_ctx qe_ctx; /* opaque host object; owns no device memory */

/* qe_plan - fill *out with the workspace size and state-array offsets for *cfg.
 * [host] cfg, out. Returns QE_ERR_UNSUPPORTED_SHAPE / QE_ERR_INVALID_ARG on a bad config. */
QE_API int qe_plan(const qe_config* cfg, qe_layout* out);

/* qe_workspace_bytes - bytes of device workspace qe_create needs (0 on a bad config). */
QE_API size_t qe_workspace_bytes(const qe_config* cfg);

/* qe_create - bind a context to a caller-allocated device workspace.
 *   workspace [dev]: at least qe_workspace_bytes(cfg) bytes, 256-byte aligned; the
 *                    library keeps every piece of state in it and never frees it.
 *   W_O [dev]:       [Hq*D][hidden] in the cache dtype; y = concat_h(o_h) @ W_O, so the
 *                    rows h*D..h*D+D-1 are W_O^h. Must outlive the context.
 *   out [host]:      receives the context.
 * The context is host-only state (shape, step counter, pointers into the workspace). */
QE_API int qe_create(const qe_config* cfg, void* workspace, size_t workspace_bytes,
                     const void* W_O, qe_ctx** out);

/* qe_destroy - free the host context. The workspace stays the caller's. */
QE_API int qe_destroy(qe_ctx* ctx);

/* qe_load_prefill - reset the context and load a prefill cache of ctx_len tokens.
 *   K, V [dev]: [B][Hkv][ctx_len][D] cache dtype. Every complete window goes to the
 *   full tier; an incomplete last window becomes the tail. Scores start at 0.
 *   norms [dev, may be NULL]: [B][Hkv][ctx_len][G] float ||V_i W_O^h||_1 of the prefill
 *   tokens (e.g. from qe_vwo_l1norm); NULL computes them here on tensor cores.
 * (QEvict, Metodologia: the cache before decoding starts.) */
QE_API int qe_load_prefill(qe_ctx* ctx, const void* K, const void* V, int ctx_len,
                           const float* norms, qe_stream_t stream);

/* qe_kv_append - append one token per unit at position n (the current length).
 *   k_new, v_new [dev]: [B][Hkv][D] cache dtype. Takes a fresh page from the unit's free
 *   list at every 16th token. (QEvict, Metodologia: states appended during decoding.) */
QE_API int qe_kv_append(qe_ctx* ctx, const void* k_new, const void* v_new, qe_stream_t stream);

/* qe_decode_attend_and_score - GQA decode attention over every live token of both tiers.
 *   q [dev]: [B][Hq][D] cache dtype; query head h uses kv head h / (Hq/Hkv).
 *   out [dev]: [B][Hq][D] float32 attention output o_h = sum_i p_{h,i} V_i.
 *   INT2 tokens are dequantised in registers (code*s + z). Fused with the scoring of
 *   "Resumo Técnico: QEvict" (Pontuação Cumulativa) and "Resumo Técnico: CriticalKV"
 *   (Etapa 2): for every live window w of unit (b,g),
 *     mass[w] += sum_{h in g} sum_{i in w} p_{h,i}
 *     pert[w] += sum_{h in g} sum_{i in w} p_{h,i} * ||V_i W_O^h||_1.
 *   When this step completes the tail window, its norms are computed (tensor cores) and it
 *   joins the full tier as a routing candidate. */
QE_API int qe_decode_attend_and_score(qe_ctx* ctx, const void* q, float* out,
                                      qe_stream_t stream);

/* qe_decode_attend_and_score_noalloc - the same computation, arguments and results as
 * qe_decode_attend_and_score, for callers that cannot provide device memory beyond their
 * inputs and outputs while a step runs (an engine that gives a plugin only its buffers and
 * forbids allocation during execution, or a process whose memory belongs to another
 * allocator). The pages have no counterpart to this entry point: it only changes where the
 * decode kernel keeps its per-call scratch (per-window score partials, tail scores): in a
 * fixed 16 MiB array inside the library image instead of the workspace scratch region.
 * It calls no cudaMalloc/cudaFree. Every GPU that loads the library keeps that array until
 * exit; all calls on one GPU share it, so calls whose kernels overlap on that GPU race and
 * must be serialised. Returns QE_ERR_INVALID_ARG if the context's scratch would exceed
 * 16 MiB. The first call on a device resolves the array's address (cudaGetSymbolAddress);
 * make it before any stream capture. */
QE_API int qe_decode_attend_and_score_noalloc(qe_ctx* ctx, const void* q, float* out,
                                              qe_stream_t stream);

/* qe_route_windows - two-stage budgeted routing of every live complete window, then the
 * tier transitions (QEvict Metodologia + CriticalKV Algoritmo):
 *   Full = TwoStage(L, F); INT2 = TwoStage(L \ Full, Q); the rest is evicted for good.
 *   TwoStage(S, b): all of S if |S| <= b, else the floor(alpha*b) highest mass, then the
 *   b - floor(alpha*b) highest pert among the rest; ties go to the lower window index.
 * Demotions quantise only windows with no ledger entry yet (write-once); promotions write
 * dequant(ledger) rounded to the cache dtype into fresh pages and keep the entry.
 * Per-unit counts of the event land in the layout's route_stats array. */
QE_API int qe_route_windows(qe_ctx* ctx, qe_stream_t stream);

/* qe_route_windows_global - one routing event under budgets shared by every layer and kv head
 * of a sequence ("Make Each Token Count", Metodologia 3: Orçamento Global, applied to the
 * window tiers of "Resumo Técnico: QEvict", Metodologia). For each batch element b, the live
 * complete windows of all contexts (one per layer, in the order given) and all kv heads compete:
 *   Full = TwoStage(L_b, full_windows); INT2 = TwoStage(L_b \ Full, int2_windows); the rest
 *   is evicted. Window w of kv head h of layer l has the flat position (l*Hkv + h)*W + w
 *   (W = max_windows); equal scores go to the lower position. TwoStage is the rule of
 *   qe_route_windows with alpha given here. Each context then applies its transitions exactly
 *   as qe_route_windows does (write-once quantisation, promotion, page and ledger reuse).
 *   ctxs [host]: n_layers distinct loaded contexts with equal B, Hkv and max_windows; their own
 *     full_windows / int2_windows are not used. Give each context page and ledger pools large
 *     enough for the share a unit may receive (e.g. slots_per_unit = max_windows); a unit whose
 *     pool runs out records QE_ERR_POOL_EXHAUSTED / QE_ERR_LEDGER_FULL in its context's status.
 *   scratch [dev]: qe_route_global_scratch_bytes(n_layers, B, Hkv, max_windows) bytes,
 *     256-byte aligned, not shared by concurrent calls.
 * Host-side errors: QE_ERR_INVALID_ARG (null, repeated or mismatched contexts, negative
 * budgets, alpha outside [0, 1]), QE_ERR_STATE (a context not loaded), QE_ERR_UNSUPPORTED_SHAPE
 * (B * n_layers * Hkv * max_windows >= 2^31), QE_ERR_WORKSPACE (small or misaligned scratch).
 * Use route_every = 0 in the contexts so that qe_decode_step leaves routing to this call.
 * After it, qe_list_counts gives upper bounds of the per-unit tier sizes. Asynchronous on
 * `stream`; allocates nothing. */
QE_API size_t qe_route_global_scratch_bytes(int n_layers, int B, int Hkv, int max_windows);
QE_API int qe_route_windows_global(qe_ctx* const* ctxs, int n_layers, int full_windows,
                                   int int2_windows, float alpha, void* scratch,
                                   size_t scratch_bytes, qe_stream_t stream);

/* qe_decode_step - one whole decode step: kv_append, decode_attend_and_score and, on steps
 * s % R == 0 (s counted from the prefill), route_windows. Arguments as above. */
QE_API int qe_decode_step(qe_ctx* ctx, const void* q, const void* k_new, const void* v_new,
                          float* out, qe_stream_t stream);

/* qe_quantize_once - demote the listed windows of one unit to the INT2 tier.
 *   win_ids [host]: n window indices of unit `unit`, each currently in the full tier.
 *   A window that already has a ledger entry reuses it (no re-quantisation).
 * (QEvict, Hierarquia Recuperável: Rebaixamento + write-once ledger.) */
QE_API int qe_quantize_once(qe_ctx* ctx, int unit, const int32_t* win_ids, int n,
                            qe_stream_t stream);

/* qe_promote - promote the listed INT2 windows of one unit back to the full tier; their
 * pages receive dequant(ledger) rounded to the cache dtype; the ledger entry is kept.
 * (QEvict, Hierarquia Recuperável: Promoção.) */
QE_API int qe_promote(qe_ctx* ctx, int unit, const int32_t* win_ids, int n,
                      qe_stream_t stream);

/* qe_int2_quantize - standalone INT2 group quantiser (the one the ledger uses).
 *   x [dev]: [T][D] cache dtype, D a multiple of 16. codes [dev]: [T][D/4] bytes, byte j of
 *   a token holds elements 4j..4j+3, element 4j+e in bits 2e..2e+1. meta [dev]: [T][D/16]
 *   pairs of fp16 (scale s, zero z), s in the low half. Per 16-element group:
 *   s = fp16(f32(max-min)/3), z = fp16(min), code = clamp(rint(f32(x-z)/s), 0, 3), 0 if s==0. */
QE_API int qe_int2_quantize(const void* x, int T, int D, int dtype, uint8_t* codes,
                            uint32_t* meta, qe_stream_t stream);

/* qe_ledger_read - the write-once INT2 ledger entry of one window ("Resumo Técnico: QEvict",
 * Hierarquia Recuperável: Livro de Registro de Quantização de Escrita Única), in the row-major
 * form of qe_int2_quantize. Inside the workspace an entry is stored in 16-token blocks arranged
 * for the decode kernel's tensor-core operands; this call is how a caller inspects it.
 *   unit in [0, B*Hkv), win in [0, max_windows).
 *   codes_k, codes_v [dev]: [window][D/4] bytes (element 4j+e of a token in bits 2e of byte j).
 *   meta_k, meta_v [dev]: [window][D/16] u32 = fp16 scale (low half) | fp16 zero (high half).
 *   found [dev, int32]: 1 when the window has a ledger entry (the outputs are then written),
 *     0 when it has none (nothing else is written).
 * QE_ERR_INVALID_ARG for a null or misaligned pointer or an index out of range; QE_ERR_STATE
 * before the prefill. Asynchronous on `stream`; allocates nothing. */
QE_API int qe_ledger_read(qe_ctx* ctx, int unit, int win, uint8_t* codes_k, uint32_t* meta_k,
                          uint8_t* codes_v, uint32_t* meta_v, int32_t* found, qe_stream_t stream);

/* qe_vwo_l1norm - N[g][r][j] = || V[g][r][:] @ W_O^{h} ||_1 with h = (g % Hkv)*G + j, on
 * tensor cores (tcgen05, accumulators in TMEM).
 *   V [dev]: [n_groups][rows][D] dtype. W_O [dev]: [Hq*D][hidden] dtype.
 *   out [dev]: float, element (g, r, j) at out[g*out_group_stride + r*G + j].
 * ("Resumo Técnico: CriticalKV", Framework Teórico: projected values V W_O.) */
QE_API int qe_vwo_l1norm(const void* V, int n_groups, int rows, int D, int dtype,
                         const void* W_O, int Hq, int Hkv, int hidden, float* out,
                         long long out_group_stride, qe_stream_t stream);

/* qe_criticalkv_select - CriticalKV two-stage selection per (batch, kv head) with a
 * SnapKV-style observation window ("Resumo Técnico: CriticalKV", Algoritmo, Etapas 1 e 2;
 * Framework Teórico for the projected values V W_O).
 * Per unit (b, kvh) with query heads h = kvh*G .. kvh*G+G-1 (G = Hq/Hkv):
 *   A[h][i] = sum_j softmax_i(q_(h,j) . K_i / sqrt(D)), query j at position n - n_obs + j seeing
 *             keys 0 .. n - n_obs + j (causal);
 *   N[i][h] = || V_i W_O^h ||_1, W_O^h = rows h*D .. h*D+D-1 of W_O;
 *   a_i = sum_h A[h][i], p_i = sum_h A[h][i] N[i][h] (float32);
 *   stage 1 keeps floor(alpha * budget) entries of highest a, stage 2 the remaining budget
 *   entries of highest p among the rest; equal scores go to the lower index.
 *   q_obs [dev]: [B][Hq][n_obs][D] queries of the last n_obs positions.
 *   K, V [dev]: [B][Hkv][n][D]. W_O [dev]: [Hq*D][hidden]. All of one dtype, 16-byte aligned.
 *   A_out [dev, float]: [B][Hkv][G][n].  N_out [dev, float]: [B][Hkv][n][G].
 *   idx_out [dev, int32]: [B][Hkv][budget]: stage-1 picks in descending a, then stage-2 picks in
 *   descending p. When n <= budget every entry is kept: idx_out = 0..n-1, then -1.
 *   scratch [dev]: qe_criticalkv_scratch_bytes() bytes, 256-byte aligned, owned by the caller;
 *   its first 8 bytes receive a status word {int32 code, int32 detail}: 0, or QE_ERR_TIMEOUT if a
 *   bounded wait inside a tensor-core kernel gave up. Read it after synchronising.
 * Supported: D in {64, 128}; n_obs in {32, 64} with G * n_obs <= 128 and n_obs <= n;
 * budget <= 8192; hidden a multiple of 64 (tensor cores when a multiple of 128); alpha in
 * [0, 1]. Otherwise QE_ERR_UNSUPPORTED_SHAPE / QE_ERR_INVALID_ARG, nothing launched.
 * Asynchronous on `stream`; allocates nothing. */
QE_API size_t qe_criticalkv_scratch_bytes(int B, int Hq, int Hkv, int n, int n_obs);
QE_API int qe_criticalkv_select(const void* q_obs, int n_obs, const void* K, const void* V,
                                const void* W_O, int B, int Hq, int Hkv, int n, int D,
                                int hidden, int dtype, int budget, float alpha,
                                float* A_out, float* N_out, int32_t* idx_out,
                                void* scratch, size_t scratch_bytes, qe_stream_t stream);

/* qe_trim_global_topm - DBTrimKV global trim of a paged, variable-length cache ("Make Each
 * Token Count", Metodologia 2-4: the retention of entry i at step t is beta_i^(t - pos_i); the
 * cache keeps the M entries of highest retention over every (layer, head) and drops the rest).
 * Each entry's key is log r = (t - pos) * ln(beta), computed in float64 (beta widened from
 * float32 exactly, ln in float64). Entries are ranked by key, descending; equal keys go to the
 * lower flat index, where the flat index runs over heads first (head 0's entries, then head 1's,
 * ...) and then over a head's entries in logical order. The first M are kept (all of them when
 * M is at least the total; none when M == 0).
 *   beta [dev, float], pos [dev, int32]: [n_pages_total][16], indexed by physical page and slot.
 *     beta is expected in (0, 1]; a key that is NaN ranks below every other key.
 *   page_table [dev, int32]: [n_heads][max_pages_per_head]; entry (h, p) is the physical page of
 *     head h's logical page p. Entry e of head h lives in logical page e/16, slot e%16.
 *   lengths [dev, int32]: [n_heads] entries per head, each in [0, 16*max_pages_per_head].
 *   kv_in [dev]: [n_pages_total][2][16][D] dtype (K rows of a page, then its V rows).
 *   kv_out, beta_out, pos_out [dev]: same shapes as kv_in, beta, pos, and must not overlap them.
 *     Head h's survivors are written in their original order to its logical entries 0..L_h-1,
 *     through the same page table. Nothing else in the outputs is written.
 *   new_lengths [dev, int32]: [n_heads] survivor count L_h of each head.
 *   scratch [dev]: qe_trim_scratch_bytes(n_heads, max_pages_per_head) bytes, 256-byte aligned,
 *     owned by the caller and not shared by concurrent calls. Its first 8 bytes receive a status
 *     word {int32 code, int32 detail}: 0 after a clean run, otherwise the first device-side error
 *     (QE_ERR_INVALID_ARG for a length out of range, QE_ERR_DEVICE_FAULT for a page-table entry
 *     outside [0, n_pages_total); detail = the head). The caller reads it after synchronising.
 * Host-side errors (returned, nothing launched): QE_ERR_INVALID_ARG for a null or misaligned
 * pointer (kv 16-byte aligned), M < 0, overlapping in/out buffers or a small scratch;
 * QE_ERR_UNSUPPORTED_SHAPE for D not in {64, 128, 256} or n_heads * 16 * max_pages_per_head
 * at or above 2^31. Asynchronous on `stream`; allocates nothing. */
QE_API size_t qe_trim_scratch_bytes(int n_heads, int max_pages_per_head);
QE_API int qe_trim_global_topm(const float* beta, const int32_t* pos, const int32_t* page_table,
                               const int32_t* lengths, int n_heads, int max_pages_per_head,
                               int n_pages_total, int D, int dtype, int t, long long M,
                               const void* kv_in, void* kv_out, float* beta_out, int32_t* pos_out,
                               int32_t* new_lengths, void* scratch, size_t scratch_bytes,
                               qe_stream_t stream);

/* qe_diag_tiers - selection churn and global latent importance reactivation between two
 * consecutive routing events ("Resumo Técnico: QEvict", Principais Contribuições 1: Churn de
 * Seleção, LIR Global). The active set is the full-precision tier.
 *   tiers [dev, uint8]: [units][W] QE_TIER_* of every window after this event (a context's
 *     win_tier array, or any map in that encoding; EVICTED also marks windows not created yet).
 *   prev [dev, uint8]: [units][W] the map at the previous event; overwritten with `tiers`.
 *   flags [dev, uint8]: [units][W] per-window history (bit 0: has left the full tier, bit 1:
 *     has re-entered it); owned by the caller, kept across calls.
 *   first: nonzero on the first event of a run: copies tiers to prev, zeroes flags, counts
 *     nothing (counters may then be NULL).
 *   counters [dev, int64]: [units][6], ADDED to (the caller zeroes them once):
 *     0 live_prev  windows FULL or INT2 at the previous event
 *     1 changed    of those, windows whose tier differs now
 *     2 exits      windows FULL before and not FULL now
 *     3 reentries  windows not FULL before, FULL now, that had exited at an earlier event
 *     4 windows_exited, 5 windows_reentered: first exit / first re-entry of a window
 *   churn = sum(changed) / sum(live_prev); LIR = sum(windows_reentered) / sum(windows_exited),
 *   pooled over units and events.
 * QE_ERR_INVALID_ARG for a null pointer or a non-positive size. Asynchronous on `stream`;
 * allocates nothing. */
QE_API int qe_diag_tiers(const uint8_t* tiers, uint8_t* prev, uint8_t* flags, int units, int W,
                         int first, long long* counters, qe_stream_t stream);

/* qe_diag_fmm - future missed mass of one decode step ("Resumo Técnico: QEvict", Principais
 * Contribuições 1: Massa Perdida Futura): for each (b, kvh) unit, the share of the ghost
 * attention that falls on tokens of evicted windows, averaged over the unit's G query heads:
 *   fmm[u] = (1/G) sum_h sum_{i < n, tiers[u][i / window] == EVICTED} p_{h,i},
 *   p_{h,.} = softmax_i(q_h . K_i / sqrt(D)) over all n tokens of the ghost cache; 0 if n == 0.
 *   q [dev]: [B][Hq][D] dtype, query head h = kvh * G + g of unit (b, kvh).
 *   K_ghost [dev]: [B][Hkv][n_stride][D] dtype, 16-byte aligned: every token's key at its
 *     original precision (the caller appends each step's key; evicted windows stay in it).
 *   tiers [dev, uint8]: [B*Hkv][W] QE_TIER_*; token i lies in window i / window.
 *   fmm_out [dev, float]: [B*Hkv].
 *   scratch [dev]: qe_diag_fmm_scratch_bytes(B*Hkv, G) bytes, 16-byte aligned, not shared by
 *     concurrent calls; its first 8 bytes receive a status word {int32 code, int32 detail}: 0,
 *     or QE_ERR_TIMEOUT if a bounded wait gave up (detail = where and the unit).
 * Host-side errors (returned, nothing launched): QE_ERR_INVALID_ARG for a null or misaligned
 * pointer, Hq not a multiple of Hkv, n < 0, n_stride < n, ceil(n / window) > W or a bad dtype;
 * QE_ERR_UNSUPPORTED_SHAPE for D not in {64, 128}, G not in {1, 2, 4, 5, 8} or
 * B * Hkv * n_stride + 16 >= 2^31; QE_ERR_WORKSPACE for a small scratch. Asynchronous on `stream`;
 * allocates nothing. */
/* qe_diag_summary - the pooled diagnostics of qe_diag_tiers' counters ("Resumo Técnico: QEvict",
 * Principais Contribuições 1): sums over units of the six counters, churn = changed / live_prev
 * and LIR = windows_reentered / windows_exited (NaN when the denominator is 0).
 *   counters [dev, int64]: [units][6] as qe_diag_tiers keeps them. out [host]: filled.
 * Synchronises `stream` (the counters are read back). QE_ERR_INVALID_ARG for a null pointer or
 * units < 1; QE_ERR_CUDA when the copy fails. */
typedef struct {
  long long live_prev, changed, exits, reentries, windows_exited, windows_reentered;
  double churn, lir;
} qe_diag_stats;
QE_API int qe_diag_summary(const long long* counters, int units, qe_diag_stats* out, qe_stream_t stream);

QE_API size_t qe_diag_fmm_scratch_bytes(int units, int G);
QE_API int qe_diag_fmm(const void* q, const void* K_ghost, long long n_stride, int n,
                       const uint8_t* tiers, int W, int window, int B, int Hq, int Hkv, int D,
                       int dtype, float* fmm_out, void* scratch, size_t scratch_bytes,
                       qe_stream_t stream);

/* SEKV-style mixed-resolution attention ("Resumo Técnico: SEKV", Metodologia 1-3).
 * qe_sekv_build (once per cache): for each sequence b, tokens with surprisal H[b][t] >= tau are
 *   anchors (full resolution) and every maximal run of non-anchor tokens is a span; for each
 *   (b, kv head) and span S the summary key is sum_{t in S} H_t K_t / sum_{t in S} H_t (the
 *   plain mean when that sum is 0) and the summary value the same mean of V, in float32.
 * qe_sekv_attend (every step): span S of kv head h is expanded when
 *   max over the G query heads of h of q . kbar_S / sqrt(D) >= theta; the output of query head
 *   (b, hq) is the softmax attention over the anchors' K/V, the tokens of expanded spans and
 *   the summaries of the other spans, a summary's score raised by ln|S| (it stands for |S|
 *   tokens). The trained routing projections and thresholds and the CPU low-rank rebuild are
 *   not part of this call: theta stands for the learned threshold and an expanded span
 *   contributes the tokens in K/V.
 *   q [dev]: [B][Hq][D]; K, V [dev]: [B][Hkv][n][D] (16-byte aligned), fp16 or bf16 (dtype);
 *   H [dev, float]: [B][n] surprisal per token; out [dev, float]: [B][Hq][D].
 *   state [dev]: qe_sekv_state_bytes(B, Hq, Hkv, n, D) bytes, 256-byte aligned, written by
 *   build and read (expansion flags and partials written) by attend; qe_sekv_state_offsets
 *   gives the byte offsets of its arrays: [0] counts [B][2] int32 (anchors, spans), [1] anchor
 *   positions [B][n] int32, [2] span starts, [3] span ends (exclusive) [B][cap] int32, [4] summary
 *   keys, [5] summary values [B][Hkv][cap][D] float, [6] expansion flags [B][Hkv][cap] uint8,
 *   and [7] cap = (n + 1) / 2.
 * Errors (returned, nothing launched): QE_ERR_INVALID_ARG (null or misaligned pointer, n < 1,
 * Hq not a multiple of Hkv, bad dtype), QE_ERR_UNSUPPORTED_SHAPE (D not in {64, 128}, G not in
 * {1, 2, 4, 5, 8}, n > 500000), QE_ERR_WORKSPACE (small state). Asynchronous; allocates nothing. */
QE_API size_t qe_sekv_state_bytes(int B, int Hq, int Hkv, int n, int D);
QE_API int qe_sekv_state_offsets(int B, int Hq, int Hkv, int n, int D, size_t* offsets);
QE_API int qe_sekv_build(const void* K, const void* V, const float* H, int B, int Hq, int Hkv, int n,
                         int D, int dtype, float tau, void* state, size_t state_bytes,
                         qe_stream_t stream);
QE_API int qe_sekv_attend(const void* q, const void* K, const void* V, int B, int Hq, int Hkv, int n,
                          int D, int dtype, float theta, void* state, size_t state_bytes,
                          float* out, qe_stream_t stream);

/* qe_state_bytes / qe_state_export / qe_state_import - checkpoint and restore of one context:
 * the persistent state the pages describe ("Resumo Técnico: QEvict", Hierarquia Recuperável:
 * the write-once INT2 ledger; Pontuação Cumulativa: the cumulative window scores), together with
 * the page pool, page tables, tier map, tier lists and free stacks that give it meaning, and the
 * host-side counters (tokens, decode steps, complete windows).
 * Format: a 256-byte header (magic "QEVS", version, the qe_config, the host counters, the byte
 * count that follows) and then the whole workspace verbatim (qe_layout.total bytes: the state
 * arrays, and the scratch region, which also carries the V rows of the incomplete tail window
 * that its norms are computed from when it completes).
 *   qe_state_bytes: bytes of a checkpoint of this context (0 for a NULL context).
 *   qe_state_export: dst [host or dev] of at least qe_state_bytes(ctx) bytes; asynchronous on
 *     `stream` for device memory and pinned host memory (the caller keeps dst alive and reads it
 *     after synchronising); the state copied is the one every earlier call on `stream` leaves.
 *     QE_ERR_STATE before the prefill, QE_ERR_WORKSPACE for a small buffer.
 *   qe_state_import: src [host or dev] of a checkpoint taken from a context with an equal
 *     qe_config (and the same W_O, which is not part of the checkpoint). Reads the header
 *     (synchronising `stream`), checks it, then copies the state into this context's workspace
 *     on `stream` and restores the host counters. QE_ERR_INVALID_ARG for a bad magic, version or
 *     config (nothing is changed then); QE_ERR_WORKSPACE for a small buffer. */
QE_API size_t qe_state_bytes(const qe_ctx* ctx);
QE_API int qe_state_export(qe_ctx* ctx, void* dst, size_t bytes, qe_stream_t stream);
QE_API int qe_state_import(qe_ctx* ctx, const void* src, size_t bytes, qe_stream_t stream);

/* qe_status - copy the device status word to the host (synchronises the context's last
 * stream) and return the first recorded error, or QE_OK. *detail (may be NULL) receives the
 * failing index or unit. */
QE_API int qe_status(qe_ctx* ctx, int* detail);

/* qe_step_index - decode steps taken since the last prefill; qe_length - tokens per unit. */
QE_API int qe_step_index(const qe_ctx* ctx);
QE_API int qe_length(const qe_ctx* ctx);
/* qe_list_counts - full-tier and INT2-tier window counts (identical for every unit under
 * per-unit routing; upper bounds over units after qe_route_windows_global). */
QE_API int qe_list_counts(const qe_ctx* ctx, int* n_full, int* n_int2);

/* qe_strerror - static message for a QE_* code. */
QE_API const char* qe_strerror(int code);

#ifdef __cplusplus
}
#endif
#endif /* QEVICT_H */
