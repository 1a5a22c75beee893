/*
 * sdm_fp8.h -- C ABI of the B200 (sm_100a) FP8 in-context-learning attention
 * layer: fused LogScale/GatedLogScale query scaling, FP8 e4m3 quantisation
 * with context-derived per-head scales, FP8 flash attention, and cached
 * prediction against a resident FP8 K/V cache with split-KV.
 *
 * Sources (web pages, cited by title and section):
 *   "Fuse shared-length query scaling during inference" (structured-data-models
 *     PR #1168), "Problem identified" and "Solution": LogScale/GatedLogScale,
 *     float32 length arithmetic, per-head conversion, query multiply and gate
 *     fused, every eager rounding boundary preserved.
 *   "[FP8 3/4] Integrate FP8 attention and caching into TabICLv2"
 *     (structured-data-models PR #879), opening section and usage example:
 *     FP8 attention of the intermediate ICL layers, Q scales derived from the
 *     context only, fit once / predict many with a quantised K/V cache, and a
 *     RuntimeError when a cache is misused (here: SDM_ERR_CACHE_MISMATCH).
 *   "[TRTLLM-15160][feat] ... make trtllm::kda_decode inplace-only"
 *     (TensorRT-LLM PR #18375), walkthrough: results go only into
 *     caller-owned output storage, checked for device, dtype and layout before
 *     launch.
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are device memory of the CURRENT CUDA device,
 *     allocated and owned by the caller, 16-byte aligned (workspace: 256-byte
 *     aligned), row-major and contiguous in the layout stated.  The library
 *     allocates nothing and writes only to the outputs, the cache buffers and
 *     the workspace it is given.
 *   - fp16 data is IEEE binary16; e4m3 data is OCP FP8 E4M3 ("fn": max 448,
 *     0x7F/0xFF NaN) stored one code per byte.
 *   - head_dim must be 64 (SDM_ERR_UNSUPPORTED otherwise); 1 <= heads <= 128.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and the call returns without synchronising.  Argument errors are
 *     reported before anything is enqueued.  A bounded in-kernel wait that
 *     gives up ORs a flag into the error word (the first 4 bytes of the
 *     workspace); sdm_sync_status() reports it as SDM_ERR_TIMEOUT and clears
 *     it.  A workspace's first 256 bytes must be zero before its first use.
 *   - Layout symbols: B batch, N context rows, M query rows, T = N + M,
 *     H heads, d = 64.  Context rows are rows [0, N) of every row-indexed
 *     tensor; query rows are [N, T).
 */
#ifndef SDM_FP8_H
#define SDM_FP8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SDM_OK = 0,
  SDM_ERR_INVALID_ARG = 1,     /* null pointer, bad size, misaligned pointer */
  SDM_ERR_UNSUPPORTED = 2,     /* head_dim != 64, heads outside [1,128], sizes past the kernels' limits */
  SDM_ERR_WORKSPACE = 3,       /* workspace missing or smaller than sdm_workspace_size() */
  SDM_ERR_DEVICE_MISMATCH = 4, /* a pointer is not device memory of the current device */
  SDM_ERR_CACHE_MISMATCH = 5,  /* cache shape/device disagrees with the call, or cache not filled */
  SDM_ERR_TIMEOUT = 6,         /* an in-kernel bounded wait gave up (from sdm_sync_status) */
  SDM_ERR_CUDA = 7             /* a CUDA runtime call or launch failed */
} sdm_status;

/* Operations, for sdm_workspace_size(). */
typedef enum {
  SDM_OP_QUANTIZE_CONTEXT = 0,
  SDM_OP_ICL_ATTENTION = 1,
  SDM_OP_CACHED_ATTENTION = 2,
  SDM_OP_ICL_ATTENTION_F16 = 3,
  SDM_OP_CACHED_ATTENTION_OFFLOAD = 4,
  SDM_OP_CACHED_PARTIALS = 5
} sdm_op;

/* Keys per online-softmax block (blocks start at key 0, or at the chunk start
 * on the cached path). */
#define SDM_KV_TILE 128

/*
 * FP8 K/V cache: the fitted state that cached prediction reads (the analogue
 * of the pages' quantised KV cache entry).  The caller allocates the three
 * buffers with the sizes from sdm_cache_layout() on one device and fills in
 * every field; sdm_fp8_quantize_context(), sdm_icl_attention() or
 * sdm_icl_attention_ragged() writes the contents and sets `filled` to 1 and
 * `ragged` to 0 or 1 (initialise both to 0).
 *   k8     [B][H][N][64]   e4m3, keys row-major (rows past n_b: zero codes)
 *   v8t    [B][H][64][ld_v] e4m3, V transposed (keys contiguous);
 *          ld_v = N rounded up to a multiple of 128; keys [n_b, ld_v) are zero
 *   scales the scales block, fp32 words: [3][B][H] s_q, s_k, s_v (amax/448
 *          over the context rows), then, for a ragged cache, n_b as int32 [B]
 *          and fp32 ln(n_b) [B]; size from sdm_cache_layout()
 */
typedef struct {
  uint8_t* k8;
  uint8_t* v8t;
  float* scales;
  int64_t n_ctx;
  int64_t ld_v;
  int32_t batch;
  int32_t heads;
  int32_t head_dim;
  int32_t device;
  int32_t filled;
  int32_t ragged; /* 1: per-batch context lengths n_b are stored in the scales block */
} sdm_fp8_cache;

/* Human-readable name of a status code (static storage). */
const char* sdm_status_string(sdm_status status);

/* Library version as major*10000 + minor*100 + patch. */
int32_t sdm_version(void);

/*
 * Keys per split-KV chunk of cached prediction for a context of n_ctx keys:
 * min(16384, max(1024, 128 * ceil(n_ctx / 4096))) -- about 32 chunks.  It
 * depends on the context length only, so a query's cached prediction does not
 * depend on how the queries are batched.  Returns 0 for n_ctx < 1.
 */
int64_t sdm_split_keys(int64_t n_ctx);

/*
 * Byte sizes of the three cache buffers for B x N x H x d, and ld_v.
 * Returns SDM_ERR_INVALID_ARG / SDM_ERR_UNSUPPORTED for bad shapes.
 */
sdm_status sdm_cache_layout(int32_t batch, int64_t n_ctx, int32_t heads, int32_t head_dim, size_t* k8_bytes,
                            size_t* v8t_bytes, size_t* scales_bytes, int64_t* ld_v);

/*
 * Workspace bytes `op` needs for these sizes (0 on invalid sizes).  For
 * SDM_OP_ICL_ATTENTION, keep_cache == 0 means the call gets no cache and the
 * workspace also holds K8/V8/scales; for the other ops keep_cache is ignored.
 * n_query is M for SDM_OP_CACHED_ATTENTION.
 */
size_t sdm_workspace_size(sdm_op op, int32_t batch, int64_t n_ctx, int64_t n_query, int32_t heads,
                          int32_t head_dim, int32_t keep_cache);

/*
 * Step 1 -- fused LogScale / GatedLogScale ("Fuse shared-length query scaling
 * during inference", "Solution").  For every row r, head h and element e:
 *   lam = fp32 ln(max(n_len, 1))            (the shared integer key length)
 *   s_h = fp16(fp32(c_h[h] * lam))           (per-head conversion)
 *   q1  = fp16(fp32(q * s_h))
 *   gated: u = fp16(tanh(gate)), w = fp16(1 + u), q_out = fp16(q1 * w)
 * with one round-to-nearest-even per eager operation.
 *   q, q_out  [B][rows][H][d] fp16 (may alias exactly: in place)
 *   c_h       [H] fp32, device
 *   gate      [B][rows][H] fp16, or NULL for LogScale
 *   n_len     >= 1
 */
sdm_status sdm_qscale_fused(const void* q, void* q_out, int32_t batch, int64_t rows, int32_t heads,
                            int32_t head_dim, int64_t n_len, const float* c_h, const void* gate, void* stream);

/*
 * Step 2 -- context-derived FP8 quantisation ("[FP8 3/4] ...", opening
 * section).  Per (b, h): s_X = amax(|X| over context rows [0, N) and all d)
 * / 448 for X in {Q', K, V} (1 if the amax is 0), then
 * X8 = e4m3_rne_satfinite(fp32(X) / s_X) with IEEE division.
 *   q_scaled  [B][T][H][d] fp16, already query-scaled (step 1); T = N + M
 *   k, v      [B][N][H][d] fp16 (context rows only)
 *   q8        [B][H][T][d] e4m3 out; query rows use the context scale and saturate
 *   cache     out: k8, v8t, scales written, `filled` set; shape fields must match
 *   ws        >= sdm_workspace_size(SDM_OP_QUANTIZE_CONTEXT, ...) bytes
 */
sdm_status sdm_fp8_quantize_context(const void* q_scaled, const void* k, const void* v, int32_t batch,
                                    int64_t n_ctx, int64_t n_query, int32_t heads, int32_t head_dim, uint8_t* q8,
                                    sdm_fp8_cache* cache, void* ws, size_t ws_bytes, void* stream);

/*
 * Step 3 alone -- FP8 flash attention of already-quantised rows to the cache
 * ("[FP8 3/4] ...", opening section).  For each row i and head h, over keys
 * j < N of the cache, in 128-key blocks:
 *   z_j = sum_e q8[e]*k8_j[e] (fp32 tensor-core accumulation)
 *   c2 = fp32(fp32(s_q*s_k) * fp32(log2(e)/8));  m = running max z;
 *   P_j = e4m3(2^(fma(z_j, c2, -fp32(m*c2))))  -- probabilities in (0, 1]
 *   l = sum_j P_j, acc = sum_j P_j * v8_j (rescaled by 2^(m2_old - m2_new)
 *   whenever the running max rises); out = fp16(acc * s_v / l).
 *   q8     [B][H][rows][d] e4m3
 *   cache  filled FP8 cache (k8, v8t, scales)
 *   out    [B][rows][H][d] fp16
 *   split  0: one pass over all keys; 1: split-KV in sdm_split_keys(N)-key
 *          chunks combined in chunk order (the cached-prediction arithmetic)
 *   ws     >= sdm_workspace_size(SDM_OP_CACHED_ATTENTION, B, N, rows, ...)
 */
sdm_status sdm_fp8_attention(const uint8_t* q8, int32_t batch, int64_t rows, const sdm_fp8_cache* cache, void* out,
                             int32_t split, void* ws, size_t ws_bytes, void* stream);

/*
 * Steps 1-3 -- one call of the FP8 ICL attention layer ("model(context,
 * labels, queries)" on "[FP8 3/4] ...").  Query scaling with n = N is fused
 * into the amax and quantisation passes; context rows attend to all context
 * rows (themselves included) and query rows attend to the context rows.
 *   q     [B][T][H][d] fp16 (raw, before query scaling), T = N + M
 *   k, v  [B][N][H][d] fp16
 *   c_h   [H] fp32 device;  gate [B][T][H] fp16 or NULL (LogScale)
 *   out   [B][T][H][d] fp16
 *   cache NULL: the FP8 K/V and scales live in the workspace and are
 *         discarded; non-NULL: "fit" -- they are written to the cache's
 *         buffers, which the caller then reuses for sdm_cached_attention.
 *   ws    >= sdm_workspace_size(SDM_OP_ICL_ATTENTION, ..., cache != NULL)
 */
sdm_status sdm_icl_attention(const void* q, const void* k, const void* v, int32_t batch, int64_t n_ctx,
                             int64_t n_query, int32_t heads, int32_t head_dim, const float* c_h, const void* gate,
                             void* out, sdm_fp8_cache* cache, void* ws, size_t ws_bytes, void* stream);

/*
 * Batched estimators with ragged contexts ("unmasked context rows",
 * "[FP8 3/4] ...", opening section): batch b has n_b = ctx_len[b] context
 * rows (1 <= n_b <= N); its rows [n_b, N) are padding.  Each batch is the
 * layer of sdm_icl_attention on its own unmasked rows: query scaling with
 * n = n_b, scales from rows [0, n_b) only, context rows [0, n_b) and query
 * rows [N, T) attend to keys [0, n_b).  Padding rows never reach a scale or a
 * softmax (their contents, NaN included, cannot change a result) and their
 * outputs are written as zeros.
 *   ctx_len  HOST array of B int64 (read during the call; not kept)
 *   other arguments as sdm_icl_attention; a cache given here is marked ragged
 *   and keeps n_b, so sdm_cached_attention masks and scales by batch.
 */
sdm_status sdm_icl_attention_ragged(const void* q, const void* k, const void* v, int32_t batch, int64_t n_ctx,
                                    int64_t n_query, int32_t heads, int32_t head_dim, const int64_t* ctx_len,
                                    const float* c_h, const void* gate, void* out, sdm_fp8_cache* cache, void* ws,
                                    size_t ws_bytes, void* stream);

/*
 * Step 4 -- cached prediction ("model.predict(queries)" after "model.fit" on
 * "[FP8 3/4] ...").  The M query rows are query-scaled with n = cache->n_ctx,
 * quantised with the cache's context-derived s_q, and attend to the cache's
 * keys with split-KV (sdm_split_keys(N)-key chunks, a fixed-order combine), so a
 * query's output is identical however the queries are batched.
 *   q    [B][M][H][d] fp16 raw;  gate [B][M][H] fp16 or NULL;  c_h [H] fp32
 *   out  [B][M][H][d] fp16
 *   ws   >= sdm_workspace_size(SDM_OP_CACHED_ATTENTION, B, cache->n_ctx, M, ...)
 * With a ragged cache, batch b's queries are scaled with n = n_b and attend to
 * its keys [0, n_b).
 * Returns SDM_ERR_CACHE_MISMATCH if the cache is unfilled, on another device,
 * or its batch/heads/head_dim differ from the call's.
 */
sdm_status sdm_cached_attention(const void* q, int32_t batch, int64_t n_query, int32_t heads, int32_t head_dim,
                                const sdm_fp8_cache* cache, const float* c_h, const void* gate, void* out, void* ws,
                                size_t ws_bytes, void* stream);

/*
 * Precision rule ("[FP8 3/4] Integrate FP8 attention and caching into
 * TabICLv2", opening section): FP8 attention serves the intermediate ICL
 * layers only, and only above 8,192 unmasked context rows; the final ICL
 * layer and shorter contexts keep normal-precision attention.  Returns 1 when
 * a layer with `n_unmasked_ctx` unmasked context rows (final_layer != 0 for
 * the last ICL layer) takes sdm_icl_attention, 0 when it takes
 * sdm_icl_attention_f16.  Pure host function; no CUDA call.
 */
#define SDM_FP8_MIN_CONTEXT 8192
int32_t sdm_fp8_eligible(int64_t n_unmasked_ctx, int32_t final_layer);

/*
 * Normal-precision ICL attention: the path the precision rule keeps for the
 * final ICL layer and for contexts of at most 8,192 rows ("[FP8 3/4] ...",
 * opening section; the pages run it through the framework's scaled
 * dot-product attention).  Same rows, masking and query scaling as
 * sdm_icl_attention: out = softmax(q' k^T / sqrt(d)) v over the N context
 * keys, with fp16 q', k, v on the tensor cores, fp32 logits and accumulation,
 * fp16 probabilities in the P.V product, fp16 output.  No quantisation and
 * no cache.
 *   q     [B][T][H][d] fp16 raw, T = N + M
 *   k, v  [B][N][H][d] fp16
 *   c_h   [H] fp32 device: query scaling with n = N (gate [B][T][H] fp16 or
 *         NULL); or c_h = NULL: no query scaling, q is used as given and gate
 *         must be NULL
 *   out   [B][T][H][d] fp16
 *   ws    >= sdm_workspace_size(SDM_OP_ICL_ATTENTION_F16, B, N, M, H, d, 0)
 */
sdm_status sdm_icl_attention_f16(const void* q, const void* k, const void* v, int32_t batch, int64_t n_ctx,
                                 int64_t n_query, int32_t heads, int32_t head_dim, const float* c_h,
                                 const void* gate, void* out, void* ws, size_t ws_bytes, void* stream);

/* sdm_icl_attention_f16 with ragged contexts: ctx_len as for
 * sdm_icl_attention_ragged (host array, 1 <= n_b <= N); padding rows out 0. */
sdm_status sdm_icl_attention_f16_ragged(const void* q, const void* k, const void* v, int32_t batch, int64_t n_ctx,
                                        int64_t n_query, int32_t heads, int32_t head_dim, const int64_t* ctx_len,
                                        const float* c_h, const void* gate, void* out, void* ws, size_t ws_bytes,
                                        void* stream);

/*
 * Step 4 from a cache held off the device ("Cache chunking, CPU offloading
 * ... are supported", "[FP8 3/4] ...", opening section).  Same result, bit
 * for bit, as sdm_cached_attention on the same cache: the K8 / V8^T buffers
 * (cache->k8, cache->v8t; page-locked host memory, or device memory) are
 * streamed one split-KV chunk of sdm_split_keys(N) keys at a time into two
 * staging slots of the workspace; chunk c's attention writes partial c and the
 * fixed-order combine follows.  Only the scales block must be on the device.
 * Copies run on `copy_stream` and overlap the attention of the previous chunk
 * on `stream` (copy_stream NULL or equal to stream: one stream, no overlap);
 * the call creates and releases its own events.  The cache must have been
 * filled on the device (the caller copies k8 / v8t out; `filled` stays 1).
 *   ws  >= sdm_workspace_size(SDM_OP_CACHED_ATTENTION_OFFLOAD, B, N, M, H, d, 0)
 *       (holds 2 x B x H x 128 x sdm_split_keys(N) bytes of staging)
 */
sdm_status sdm_cached_attention_offload(const void* q, int32_t batch, int64_t n_query, int32_t heads,
                                        int32_t head_dim, const sdm_fp8_cache* cache, const float* c_h,
                                        const void* gate, void* out, void* ws, size_t ws_bytes, void* stream,
                                        void* copy_stream);

/*
 * Ragged grouped-query prefill, a second workload beside the ICL layer
 * ("Pipeline long ragged GQA4 KV loads", oxide-infer PR #114, performance
 * contract: 2 sequences, query lengths 32/64, key/value lengths 256/1024, 16
 * query heads, 4 key/value heads, head dim 128, bf16).  Sequence b owns query
 * tokens [qo_indptr[b], qo_indptr[b+1]) and key/value tokens [kv_indptr[b],
 * kv_indptr[b+1]); query head h reads key/value head h / (q_heads / kv_heads);
 * out = softmax(q k^T / sqrt(128)) v with fp32 softmax and accumulation.
 * causal = 1: the queries are the last q_len of the kv_len tokens, query i
 * sees keys j <= kv_len - q_len + i (needs kv_len >= q_len); causal = 0: every
 * key of the sequence.
 *   q    [total_q][q_heads][128] bf16;  k, v [total_kv][kv_heads][128] bf16
 *   qo_indptr, kv_indptr  HOST arrays of batch + 1 int64 offsets, starting at 0
 *   out  [total_q][q_heads][128] bf16
 *   q_heads / kv_heads in {1, 2, 4, 8, 16}; head_dim 128 (else SDM_ERR_UNSUPPORTED)
 *   ws   >= sdm_gqa_prefill_workspace_size(...) bytes (the error word; its first
 *        256 bytes zero before first use).  A query tile's keys are split over
 *        a cluster of 4 CTAs that combine their shares in shared memory, in
 *        rank order, so the result does not depend on timing.
 * This entry point has no counterpart on the pages that define the ICL layer.
 */
size_t sdm_gqa_prefill_workspace_size(const int64_t* qo_indptr, const int64_t* kv_indptr, int32_t batch,
                                      int32_t q_heads, int32_t kv_heads, int32_t head_dim, int32_t causal);

sdm_status sdm_gqa_prefill(const void* q, const void* k, const void* v, const int64_t* qo_indptr,
                           const int64_t* kv_indptr, int32_t batch, int32_t q_heads, int32_t kv_heads,
                           int32_t head_dim, int32_t causal, void* out, void* ws, size_t ws_bytes, void* stream);

/*
 * Step 2 without a workspace.  This entry point has no counterpart in the
 * pages: it exists for callers that cannot allocate device memory for the
 * library -- code that must not call cudaMalloc on its path (cudaMalloc can
 * synchronise the device), plugins whose framework owns all device memory, and
 * hooks with no allocation API at hand.  Same arguments, layouts, results and
 * errors as sdm_fp8_quantize_context, minus ws/ws_bytes.
 *   - Its scratch (the amax accumulators, 3*B*H words) is a fixed array inside
 *     the library image, sized for B*H <= SDM_NOALLOC_MAX_BATCH_HEADS (48 KiB);
 *     every GPU that loads the library holds it until the process exits.
 *     Larger B*H returns SDM_ERR_UNSUPPORTED before any work is enqueued.
 *   - The first call on a device looks up the array's device address (with
 *     that device current), and so does the first call in a new CUDA context
 *     of the device (after cudaDeviceReset, for instance); make that first
 *     call before any stream capture.
 *   - The call allocates nothing and clears the scratch it uses on `stream`.
 *   - All calls share the one array: calls that overlap on the GPU (another
 *     stream, another thread) race on it and may produce wrong scales.  Order
 *     them on one stream or synchronise between them.
 */
#define SDM_NOALLOC_MAX_BATCH_HEADS 4096
sdm_status sdm_fp8_quantize_context_noalloc(const void* q_scaled, const void* k, const void* v, int32_t batch,
                                            int64_t n_ctx, int64_t n_query, int32_t heads, int32_t head_dim,
                                            uint8_t* q8, sdm_fp8_cache* cache, void* stream);

/*
 * Step 2 split over ranks (one process per GPU), each holding a slice of the
 * context rows.  The scales are derived from ALL context rows ("[FP8 3/4]
 * Integrate FP8 attention and caching into TabICLv2", opening section:
 * context-derived per-head scales); the maximum is exact and associative, so
 * per-slice maxima combined by an all-reduce(MAX) give the one-process scales
 * bit for bit.  The pages describe no multi-GPU scheme; this split is the
 * library's.  A sharded layer call is:
 *   1. sdm_context_amax on each rank's context slice;
 *   2. all-reduce(MAX) of the [3][B][H] fp32 words over the ranks (NCCL);
 *   3. sdm_quantize_with_scales of each rank's rows with the reduced words;
 *   4. all-gather of the K8 rows and V8^T columns; sdm_cache_put_rows places
 *      each rank's slice into a full cache on every rank;
 *   5. sdm_fp8_attention of each rank's quantised rows against that cache.
 * Each row's result equals the one-process layer's bit for bit.
 */

/*
 * Per-(tensor, batch, head) maxima of |Q'|, |K|, |V| over context rows
 * [0, n_ctx) of this slice.
 *   q      [B][q_rows][H][d] fp16, q_rows >= n_ctx: raw q (query scaling with the
 *          global context length n_len, coefficients c_h and optional gate
 *          [B][q_rows][H] fused, as in sdm_icl_attention) or, with c_h == NULL,
 *          already-scaled q' (n_len and gate are then ignored)
 *   k, v   [B][n_ctx][H][d] fp16 (may be NULL when n_ctx == 0)
 *   amax   out, [3][B][H] fp32 device (values >= 0: Q', K, V); overwritten.
 *          n_ctx == 0 gives zeros (the identity of the MAX reduction).
 * No workspace.  Errors: SDM_ERR_INVALID_ARG (null/misaligned pointer,
 * q_rows < n_ctx, n_len < 1 with c_h), SDM_ERR_UNSUPPORTED (d != 64, heads
 * outside 1..128), SDM_ERR_DEVICE_MISMATCH; all before any work is enqueued.
 */
sdm_status sdm_context_amax(const void* q, const void* k, const void* v, int32_t batch, int64_t n_ctx,
                            int64_t q_rows, int32_t heads, int32_t head_dim, int64_t n_len, const float* c_h,
                            const void* gate, float* amax, void* stream);

/*
 * Scales from the (reduced) maxima and e4m3 codes of this slice's rows:
 *   scales[t][b][h] = amax[t][b][h] / 448 (IEEE fp32 division; 1 where the
 *   maximum is 0), the same words sdm_fp8_quantize_context writes;
 *   q8  [B][H][n_ctx + n_query][d]  e4m3 of the slice's rows of Q' (context rows
 *       first, then its query rows; query rows above the context maximum
 *       saturate to +-448)
 *   k8  [B][H][ld_k][d]             e4m3 of K in rows [0, n_ctx) of each (b, h)
 *                                   plane, ld_k >= n_ctx (rows past n_ctx are not
 *                                   written); may be NULL when n_ctx == 0
 *   v8t [B][H][d][ld_v]             e4m3 of V transposed; ld_v a multiple of 128,
 *                                   >= n_ctx; columns [n_ctx, ld_v) written zero
 *   q, k, v, n_len, c_h, gate as for sdm_context_amax, with q holding
 *   n_ctx + n_query rows.  amax and scales are fp32 [3][B][H] device arrays.
 * No workspace.  Errors as sdm_context_amax, plus SDM_ERR_INVALID_ARG for a bad
 * ld_k or ld_v.
 */
sdm_status sdm_quantize_with_scales(const void* q, const void* k, const void* v, int32_t batch, int64_t n_ctx,
                                    int64_t n_query, int32_t heads, int32_t head_dim, int64_t n_len,
                                    const float* c_h, const void* gate, const float* amax, float* scales,
                                    uint8_t* q8, uint8_t* k8, int64_t ld_k, uint8_t* v8t, int64_t ld_v,
                                    void* stream);

/*
 * Copies a slice of n context rows into a cache at global row `row0`:
 *   k8_rows  [B][H][ld_k][d] e4m3, rows [0, n) of each plane
 *            -> cache->k8 rows [row0, row0 + n) of every (b, h)
 *   v8t_cols [B][H][d][ld_v] e4m3, columns [0, n) of each row
 *            -> cache->v8t columns [row0, row0 + n)
 * (device memory of the cache's device; ld_k, ld_v >= n).  The cache's scales
 * block is not touched, and `filled` is not set: the caller writes the scales
 * (sdm_quantize_with_scales) and sets filled = 1 once every slice is in.
 * Columns [N, ld_v) of cache->v8t must be zero (the caller zero-fills the
 * buffer once).  Two strided device-to-device copies on `stream`.
 * Errors: SDM_ERR_INVALID_ARG (row range outside [0, N), ld_k or ld_v < n,
 * null or misaligned pointers), SDM_ERR_CACHE_MISMATCH (cache on another
 * device), SDM_ERR_CUDA.
 */
sdm_status sdm_cache_put_rows(sdm_fp8_cache* cache, const uint8_t* k8_rows, int64_t ld_k, const uint8_t* v8t_cols,
                              int64_t ld_v, int64_t row0, int64_t n, void* stream);

/*
 * Step 4 with the cache's keys split over ranks by split-KV chunk.  Cached
 * prediction cuts the N keys into S = ceil(N / L) chunks of L =
 * sdm_split_keys(N) keys, computes a partial (m2, l, acc) per chunk, and
 * combines the partials in chunk order ("[FP8 3/4] ...", opening section:
 * "Cache chunking ... supported"; the split over ranks is the library's).
 * Chunks are independent until the combine, so a rank holding only the keys
 * of chunks [c0, c1) computes their partials alone; an all-gather brings all S
 * partials to every rank, and sdm_cached_combine gives the one-GPU
 * sdm_cached_attention result bit for bit.
 *
 * sdm_cached_partials: the partials of chunks [c0, c1), 0 <= c0 < c1 <= S.
 *   cache      the full cache's descriptor (n_ctx = N, batch, heads, device,
 *              ragged, filled, the scales block on this device); its k8 and
 *              v8t are not read
 *   k8_slice   [B][H][n][d] e4m3: keys [c0 L, c0 L + n) of every (b, h),
 *              n = min(c1 L, N) - c0 L
 *   v8t_slice  [B][H][d][ld_slice] e4m3: the same keys of V8^T; ld_slice a
 *              multiple of 128, >= n; columns [n, ld_slice) zero
 *   q, c_h, gate  as for sdm_cached_attention (M query rows)
 *   part_acc   [S][B][H][M][d] fp32 and part_ml [S][B][H][M][2] fp32 (m2, l):
 *              the rows of chunks [c0, c1) are written, the others untouched
 *   ws         >= sdm_workspace_size(SDM_OP_CACHED_PARTIALS, B, N, M, H, d, 0)
 * sdm_cached_combine: out [B][M][H][d] fp16 from the partials of all S chunks.
 * Errors: SDM_ERR_INVALID_ARG (chunk range, slice sizes, null or misaligned
 * pointers), SDM_ERR_CACHE_MISMATCH (descriptor), SDM_ERR_WORKSPACE,
 * SDM_ERR_DEVICE_MISMATCH, SDM_ERR_UNSUPPORTED; before any work is enqueued.
 */
sdm_status sdm_cached_partials(const void* q, int32_t batch, int64_t n_query, int32_t heads, int32_t head_dim,
                               const sdm_fp8_cache* cache, const uint8_t* k8_slice, const uint8_t* v8t_slice,
                               int64_t ld_slice, int64_t c0, int64_t c1, const float* c_h, const void* gate,
                               float* part_acc, float* part_ml, void* ws, size_t ws_bytes, void* stream);
sdm_status sdm_cached_combine(const float* part_acc, const float* part_ml, int32_t batch, int64_t n_query,
                              int32_t heads, int32_t head_dim, const sdm_fp8_cache* cache, void* out,
                              void* stream);

/*
 * Wait for `stream`, then read and clear the device error word at the head of
 * a workspace used by the calls above.  Returns SDM_OK, SDM_ERR_TIMEOUT (an
 * in-kernel wait gave up; `*flags` gets the raw bits if flags != NULL) or
 * SDM_ERR_CUDA (an asynchronous CUDA error surfaced).
 */
sdm_status sdm_sync_status(void* ws, void* stream, uint32_t* flags);

/*
 * Self-test of the failure path shared by every in-kernel wait: launches one
 * warp that waits, with the same bounded mbarrier wait the attention kernel
 * uses, on a barrier that nothing ever arrives at.  After `limit_cycles` SM
 * clock cycles (1000 .. 2^31) the wait gives up, the kernel sets bit 7 of the
 * error word at the head of `ws` and returns; sdm_sync_status() then reports
 * SDM_ERR_TIMEOUT and the CUDA context stays usable.  Nothing faults or hangs.
 */
sdm_status sdm_selftest_wait_timeout(void* ws, int64_t limit_cycles, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SDM_FP8_H */
