// api.cu -- the C ABI declared in include/sdm_fp8.h: argument validation,
// workspace carving, and the launch sequences of the four layer operations.
// Every argument error is reported before any work is enqueued; nothing here
// allocates device memory.
#include <math.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "../../include/sdm_fp8.h"
#include "kernels.cuh"

using namespace sdm;

namespace {

constexpr size_t kAlign = 1024;
constexpr size_t kErrBytes = 256;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  return dev;
}

// True if p is device (or managed) memory on device `dev`.
bool on_device(const void* p, int dev) {
  if (p == nullptr) return false;
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) && at.device == dev;
}

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// True if p is page-locked host memory (or device memory of `dev`): what an
// asynchronous copy can read without staging through the driver.
bool pinned_or_device(const void* p, int dev) {
  if (p == nullptr) return false;
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (at.type == cudaMemoryTypeHost) return true;
  return (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) && at.device == dev;
}

sdm_status check_shape(int32_t B, int64_t rows_a, int64_t rows_b, int32_t H, int32_t d) {
  if (B < 1 || H < 1 || rows_a < 0 || rows_b < 0) return SDM_ERR_INVALID_ARG;
  if (d != kHeadDim) return SDM_ERR_UNSUPPORTED;
  if (H > 128) return SDM_ERR_UNSUPPORTED;
  // TMA coordinates and grid sizes are 32-bit: keep every row count and B*H in range
  if (rows_a > (int64_t)1 << 30 || rows_b > (int64_t)1 << 30 || (int64_t)B * H > 65535) return SDM_ERR_UNSUPPORTED;
  return SDM_OK;
}

// Checks a tensor pointer: non-null, 16-byte aligned, device memory of `dev`.
sdm_status check_tensor(const void* p, int dev) {
  if (p == nullptr || !aligned(p, 16)) return SDM_ERR_INVALID_ARG;
  if (!on_device(p, dev)) return SDM_ERR_DEVICE_MISMATCH;
  return SDM_OK;
}

#define SDM_TRY(expr)                       \
  do {                                      \
    const sdm_status _st = (expr);          \
    if (_st != SDM_OK) return _st;          \
  } while (0)

#define SDM_CUDA(expr)                      \
  do {                                      \
    if ((expr) != cudaSuccess) {            \
      cudaGetLastError();                   \
      return SDM_ERR_CUDA;                  \
    }                                       \
  } while (0)

// Workspace carve-up.  Offsets are 1 KB aligned; the error word sits at 0.
struct WsLayout {
  size_t amax = 0, gate_w = 0, q8 = 0, k8 = 0, v8t = 0, scales = 0, part_acc = 0, part_ml = 0, total = 0;
  size_t q16 = 0, vt16 = 0, meta = 0;  // normal-precision path: q', V^T in fp16, ragged meta
  size_t stage = 0, stage_bytes = 0;    // offloaded cache: two staging slots of one chunk each
};

int64_t n_splits_for(int64_t n_ctx) {
  const int64_t len = split_keys_for(n_ctx);
  return (n_ctx + len - 1) / len;
}

WsLayout ws_layout(sdm_op op, int32_t B, int64_t N, int64_t M, int32_t H, int32_t keep_cache) {
  WsLayout w;
  const size_t BH = (size_t)B * H;
  size_t off = kErrBytes;
  if (op == SDM_OP_ICL_ATTENTION_F16) {
    const int64_t ld = round_up(N, kKvTile);
    w.q16 = off;
    off = align_up(off + BH * (size_t)(N + M) * kHeadDim * sizeof(uint16_t), kAlign);
    w.vt16 = off;
    off = align_up(off + BH * kHeadDim * (size_t)ld * sizeof(uint16_t), kAlign);
    w.meta = off;  // ragged contexts: n_b int32 [B], lam_b fp32 [B]
    off = align_up(off + 2 * (size_t)B * sizeof(float), kAlign);
    w.total = off;
    return w;
  }
  w.amax = off;
  off = align_up(off + 3 * BH * sizeof(uint32_t), kAlign);
  if (op == SDM_OP_QUANTIZE_CONTEXT) {
    w.total = off;
    return w;
  }
  const int64_t rows = (op == SDM_OP_ICL_ATTENTION) ? N + M : M;  // cached ops: the M query rows
  // (SDM_OP_CACHED_PARTIALS: error word, gate factors and Q8 only -- the caller owns the partials)
  w.gate_w = off;  // GatedLogScale factors, one fp16 per (row, head)
  off = align_up(off + BH * (size_t)rows * sizeof(uint16_t), kAlign);
  w.q8 = off;
  off = align_up(off + BH * (size_t)rows * kHeadDim, kAlign);
  if (op == SDM_OP_ICL_ATTENTION && !keep_cache) {
    const int64_t ld = round_up(N, kKvTile);
    w.k8 = off;
    off = align_up(off + BH * (size_t)N * kHeadDim, kAlign);
    w.v8t = off;
    off = align_up(off + BH * kHeadDim * (size_t)ld, kAlign);
    w.scales = off;  // scales block: [3][B][H] scales, then the ragged meta words
    off = align_up(off + scales_block_words(B, H, true) * sizeof(float), kAlign);
  }
  if (op == SDM_OP_CACHED_ATTENTION || op == SDM_OP_CACHED_ATTENTION_OFFLOAD) {
    const size_t S = (size_t)n_splits_for(N);
    w.part_acc = off;
    off = align_up(off + S * BH * (size_t)M * kHeadDim * sizeof(float), kAlign);
    w.part_ml = off;
    off = align_up(off + S * BH * (size_t)M * 2 * sizeof(float), kAlign);
  }
  if (op == SDM_OP_CACHED_ATTENTION_OFFLOAD) {
    // one chunk of split_keys_for(N) keys per slot: K8 [B][H][L][64] + V8^T [B][H][64][L]
    const size_t L = (size_t)split_keys_for(N);
    w.stage_bytes = align_up(2 * BH * L * kHeadDim, kAlign);
    w.stage = off;
    off += 2 * w.stage_bytes;
  }
  w.total = off;
  return w;
}

sdm_status check_ws(void* ws, size_t ws_bytes, size_t need, int dev) {
  if (ws == nullptr || ws_bytes < need) return SDM_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return SDM_ERR_INVALID_ARG;
  if (!on_device(ws, dev)) return SDM_ERR_DEVICE_MISMATCH;
  return SDM_OK;
}

// Validates the cache descriptor against a call's B/H/d and the device.
sdm_status check_cache(const sdm_fp8_cache* c, int32_t B, int32_t H, int32_t d, int dev, bool need_filled) {
  if (c == nullptr) return SDM_ERR_INVALID_ARG;
  if (c->batch != B || c->heads != H || c->head_dim != d || c->device != dev || c->n_ctx < 1 ||
      c->ld_v != round_up(c->n_ctx, kKvTile) || (c->ragged != 0 && c->ragged != 1))
    return SDM_ERR_CACHE_MISMATCH;
  if (need_filled && c->filled != 1) return SDM_ERR_CACHE_MISMATCH;
  if (c->k8 == nullptr || c->v8t == nullptr || c->scales == nullptr) return SDM_ERR_INVALID_ARG;
  if (!aligned(c->k8, 16) || !aligned(c->v8t, 16) || !aligned(c->scales, 16)) return SDM_ERR_INVALID_ARG;
  if (!on_device(c->k8, dev) || !on_device(c->v8t, dev) || !on_device(c->scales, dev))
    return SDM_ERR_CACHE_MISMATCH;
  return SDM_OK;
}

QScale make_qscale(int64_t n_len, const float* c_h, const void* gate) {
  QScale qs;
  qs.enabled = true;
  // fp32 natural log of the shared integer length, clamped at 1, on the host
  qs.lam = logf(static_cast<float>(n_len < 1 ? 1 : n_len));
  qs.c_h = c_h;
  qs.gate = reinterpret_cast<const __half*>(gate);
  qs.gate_w = nullptr;
  qs.lam_b = nullptr;
  return qs;
}

QScale no_qscale() {
  QScale qs;
  qs.enabled = false;
  qs.lam = 0.0f;
  qs.c_h = nullptr;
  qs.gate = nullptr;
  qs.gate_w = nullptr;
  qs.lam_b = nullptr;
  return qs;
}

// With a gate, evaluate the gate factors once per (row, head) into the
// workspace so the row kernels do not repeat the double-precision tanh per lane.
cudaError_t prepare_gate(QScale& qs, int64_t n, uint8_t* ws_base, const WsLayout& w, cudaStream_t st) {
  if (!qs.enabled || qs.gate == nullptr) return cudaSuccess;
  __half* gw = reinterpret_cast<__half*>(ws_base + w.gate_w);
  cudaError_t e = launch_gate_factors(qs.gate, n, gw, st);
  qs.gate_w = gw;
  return e;
}

// Ragged contexts: checks the host array ctx_len[B] (1 <= n_b <= N) and
// enqueues the writes of n_b and lam_b = fp32 ln(n_b) (the host evaluation the
// uniform path uses) into the meta words at `meta` (n_b int32 [B], lam_b fp32 [B]).
sdm_status check_ctx_len(const int64_t* ctx_len, int32_t B, int64_t N) {
  if (ctx_len == nullptr) return SDM_ERR_INVALID_ARG;
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, ctx_len) == cudaSuccess) {
    if (at.type == cudaMemoryTypeDevice) return SDM_ERR_INVALID_ARG;  // must be host memory
  } else {
    cudaGetLastError();
  }
  for (int32_t b = 0; b < B; ++b)
    if (ctx_len[b] < 1 || ctx_len[b] > N) return SDM_ERR_INVALID_ARG;
  return SDM_OK;
}

cudaError_t put_meta(const int64_t* ctx_len, int32_t B, float* meta, cudaStream_t st) {
  int32_t* n_dst = reinterpret_cast<int32_t*>(meta);
  float* lam_dst = meta + B;
  for (int32_t b0 = 0; b0 < B; b0 += kMetaChunk) {
    MetaChunk c;
    memset(&c, 0, sizeof(c));
    c.b0 = b0;
    c.count = B - b0 < kMetaChunk ? B - b0 : kMetaChunk;
    for (int i = 0; i < c.count; ++i) {
      c.n[i] = static_cast<int32_t>(ctx_len[b0 + i]);
      c.lam[i] = logf(static_cast<float>(ctx_len[b0 + i]));
    }
    const cudaError_t e = launch_write_meta(c, n_dst, lam_dst, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// amax -> scales -> Q8 / K8 / V8^T.  `qs` is applied to Q (enabled: raw q in).
// n_valid (device, nullable): per-batch context rows; padding rows get zero codes.
sdm_status run_quantize(const __half* q, const __half* k, const __half* v, int32_t B, int64_t N, int64_t M,
                        int32_t H, QScale qs, uint8_t* q8, uint8_t* k8, uint8_t* v8t, int64_t ld, float* scales,
                        const int32_t* n_valid, uint8_t* ws_base, const WsLayout& w, cudaStream_t st) {
  const int64_t T = N + M;
  uint32_t* amax = reinterpret_cast<uint32_t*>(ws_base + w.amax);
  SDM_CUDA(cudaMemsetAsync(amax, 0, 3 * (size_t)B * H * sizeof(uint32_t), st));
  SDM_CUDA(prepare_gate(qs, (int64_t)B * T * H, ws_base, w, st));
  RowsDesc dq{q, B, H, T}, dk{k, B, H, N}, dv{v, B, H, N};
  SDM_CUDA(launch_context_amax(dq, qs, dk, dv, N, n_valid, amax, st));
  SDM_CUDA(launch_scales_from_amax(amax, B * H, scales, st));
  const int64_t BH = (int64_t)B * H;
  SDM_CUDA(launch_quantize_rows(dq, qs, T, scales, q8, T, n_valid, N, st));
  SDM_CUDA(launch_quantize_rows(dk, no_qscale(), N, scales + BH, k8, N, n_valid, N, st));
  SDM_CUDA(launch_quantize_vt(dv, N, n_valid, scales + 2 * BH, v8t, ld, st));
  return SDM_OK;
}

}  // namespace

extern "C" {

const char* sdm_status_string(sdm_status s) {
  switch (s) {
    case SDM_OK: return "SDM_OK";
    case SDM_ERR_INVALID_ARG: return "SDM_ERR_INVALID_ARG: null, misaligned or out-of-range argument";
    case SDM_ERR_UNSUPPORTED: return "SDM_ERR_UNSUPPORTED: head_dim must be 64, heads 1..128, rows <= 2^30";
    case SDM_ERR_WORKSPACE: return "SDM_ERR_WORKSPACE: workspace missing or too small";
    case SDM_ERR_DEVICE_MISMATCH: return "SDM_ERR_DEVICE_MISMATCH: pointer is not device memory of the current device";
    case SDM_ERR_CACHE_MISMATCH: return "SDM_ERR_CACHE_MISMATCH: FP8 cache shape, device or state disagrees with the call";
    case SDM_ERR_TIMEOUT: return "SDM_ERR_TIMEOUT: an in-kernel bounded wait gave up";
    case SDM_ERR_CUDA: return "SDM_ERR_CUDA: a CUDA runtime call or kernel launch failed";
  }
  return "SDM_ERR_UNKNOWN";
}

int32_t sdm_version(void) { return 101; }

int64_t sdm_split_keys(int64_t n_ctx) { return n_ctx < 1 ? 0 : split_keys_for(n_ctx); }

sdm_status sdm_cache_layout(int32_t B, int64_t N, int32_t H, int32_t d, size_t* k8_bytes, size_t* v8t_bytes,
                            size_t* scales_bytes, int64_t* ld_v) {
  SDM_TRY(check_shape(B, N, 0, H, d));
  if (N < 1) return SDM_ERR_INVALID_ARG;
  const int64_t ld = round_up(N, kKvTile);
  if (k8_bytes) *k8_bytes = (size_t)B * H * N * kHeadDim;
  if (v8t_bytes) *v8t_bytes = (size_t)B * H * kHeadDim * ld;
  if (scales_bytes) *scales_bytes = scales_block_words(B, H, true) * sizeof(float);
  if (ld_v) *ld_v = ld;
  return SDM_OK;
}

size_t sdm_workspace_size(sdm_op op, int32_t B, int64_t N, int64_t M, int32_t H, int32_t d, int32_t keep_cache) {
  if (op != SDM_OP_QUANTIZE_CONTEXT && op != SDM_OP_ICL_ATTENTION && op != SDM_OP_CACHED_ATTENTION &&
      op != SDM_OP_ICL_ATTENTION_F16 && op != SDM_OP_CACHED_ATTENTION_OFFLOAD && op != SDM_OP_CACHED_PARTIALS)
    return 0;
  if (check_shape(B, N, M, H, d) != SDM_OK || N < 1) return 0;
  return ws_layout(op, B, N, M, H, keep_cache).total;
}

sdm_status sdm_qscale_fused(const void* q, void* q_out, int32_t B, int64_t rows, int32_t H, int32_t d,
                            int64_t n_len, const float* c_h, const void* gate, void* stream) {
  SDM_TRY(check_shape(B, rows, 0, H, d));
  if (n_len < 1) return SDM_ERR_INVALID_ARG;
  const int dev = current_device();
  if (dev < 0) return SDM_ERR_CUDA;
  SDM_TRY(check_tensor(q, dev));
  SDM_TRY(check_tensor(q_out, dev));
  if (c_h == nullptr || !aligned(c_h, 4)) return SDM_ERR_INVALID_ARG;
  if (!on_device(c_h, dev)) return SDM_ERR_DEVICE_MISMATCH;
  if (gate != nullptr) {
    if (!aligned(gate, 2)) return SDM_ERR_INVALID_ARG;
    if (!on_device(gate, dev)) return SDM_ERR_DEVICE_MISMATCH;
  }
  if (rows == 0) return SDM_OK;
  SDM_CUDA(launch_qscale(reinterpret_cast<const __half*>(q), reinterpret_cast<__half*>(q_out), B, rows, H,
                         make_qscale(n_len, c_h, gate), as_stream(stream)));
  return SDM_OK;
}

sdm_status sdm_fp8_quantize_context(const void* q_scaled, const void* k, const void* v, int32_t B, int64_t N,
                                    int64_t M, int32_t H, int32_t d, uint8_t* q8, sdm_fp8_cache* cache, void* ws,
                                    size_t ws_bytes, void* stream) {
  SDM_TRY(check_shape(B, N, M, H, d));
  if (N < 1) return SDM_ERR_INVALID_ARG;
  const int dev = current_device();
  if (dev < 0) return SDM_ERR_CUDA;
  SDM_TRY(check_tensor(q_scaled, dev));
  SDM_TRY(check_tensor(k, dev));
  SDM_TRY(check_tensor(v, dev));
  SDM_TRY(check_tensor(q8, dev));
  SDM_TRY(check_cache(cache, B, H, d, dev, false));
  if (cache->n_ctx != N) return SDM_ERR_CACHE_MISMATCH;
  const WsLayout w = ws_layout(SDM_OP_QUANTIZE_CONTEXT, B, N, M, H, 1);
  SDM_TRY(check_ws(ws, ws_bytes, w.total, dev));
  cudaStream_t st = as_stream(stream);
  SDM_TRY(run_quantize(reinterpret_cast<const __half*>(q_scaled), reinterpret_cast<const __half*>(k),
                       reinterpret_cast<const __half*>(v), B, N, M, H, no_qscale(), q8, cache->k8, cache->v8t,
                       cache->ld_v, cache->scales, nullptr, reinterpret_cast<uint8_t*>(ws), w, st));
  cache->filled = 1;
  cache->ragged = 0;
  return SDM_OK;
}

sdm_status sdm_fp8_attention(const uint8_t* q8, int32_t B, int64_t rows, const sdm_fp8_cache* cache, void* out,
                             int32_t split, void* ws, size_t ws_bytes, void* stream) {
  if (cache == nullptr) return SDM_ERR_INVALID_ARG;
  SDM_TRY(check_shape(B, cache->n_ctx, rows, cache->heads, cache->head_dim));
  if (split != 0 && split != 1) return SDM_ERR_INVALID_ARG;
  const int dev = current_device();
  if (dev < 0) return SDM_ERR_CUDA;
  SDM_TRY(check_cache(cache, B, cache->heads, cache->head_dim, dev, true));
  if (rows == 0) return SDM_OK;
  SDM_TRY(check_tensor(q8, dev));
  SDM_TRY(check_tensor(out, dev));
  const int32_t H = cache->heads;
  const WsLayout w = ws_layout(SDM_OP_CACHED_ATTENTION, B, cache->n_ctx, rows, H, 1);
  SDM_TRY(check_ws(ws, ws_bytes, split ? w.total : kErrBytes, dev));
  cudaStream_t st = as_stream(stream);
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  AttnArgs a;
  a.B = B;
  a.H = H;
  a.T = rows;
  a.N = cache->n_ctx;
  a.ld_v = cache->ld_v;
  a.scales = cache->scales;
  a.partial = split != 0;
  a.n_splits = split ? n_splits_for(cache->n_ctx) : 1;
  a.split_keys = split_keys_for(cache->n_ctx);
  a.out = reinterpret_cast<__half*>(out);
  a.part_acc = split ? reinterpret_cast<float*>(base + w.part_acc) : nullptr;
  a.part_ml = split ? reinterpret_cast<float*>(base + w.part_ml) : nullptr;
  a.err = reinterpret_cast<uint32_t*>(base);
  a.n_keys = cache->ragged ? reinterpret_cast<const int32_t*>(cache->scales + 3 * (int64_t)B * H) : nullptr;
  a.pad_rows = false;
  SDM_CUDA(launch_attention(q8, cache->k8, cache->v8t, a, st));
  if (split) SDM_CUDA(launch_splitkv_reduce(a, st));
  return SDM_OK;
}

static sdm_status icl_attention_impl(const void* q, const void* k, const void* v, int32_t B, int64_t N, int64_t M,
                                     int32_t H, int32_t d, const int64_t* ctx_len, const float* c_h,
                                     const void* gate, void* out, sdm_fp8_cache* cache, void* ws, size_t ws_bytes,
                                     void* stream) {
  SDM_TRY(check_shape(B, N, M, H, d));
  if (N < 1) return SDM_ERR_INVALID_ARG;
  if (ctx_len != nullptr) SDM_TRY(check_ctx_len(ctx_len, B, N));
  const int dev = current_device();
  if (dev < 0) return SDM_ERR_CUDA;
  SDM_TRY(check_tensor(q, dev));
  SDM_TRY(check_tensor(k, dev));
  SDM_TRY(check_tensor(v, dev));
  SDM_TRY(check_tensor(out, dev));
  if (c_h == nullptr || !aligned(c_h, 4)) return SDM_ERR_INVALID_ARG;
  if (!on_device(c_h, dev)) return SDM_ERR_DEVICE_MISMATCH;
  if (gate != nullptr) {
    if (!aligned(gate, 2)) return SDM_ERR_INVALID_ARG;
    if (!on_device(gate, dev)) return SDM_ERR_DEVICE_MISMATCH;
  }
  if (cache != nullptr) {
    SDM_TRY(check_cache(cache, B, H, d, dev, false));
    if (cache->n_ctx != N) return SDM_ERR_CACHE_MISMATCH;
  }
  const WsLayout w = ws_layout(SDM_OP_ICL_ATTENTION, B, N, M, H, cache != nullptr);
  SDM_TRY(check_ws(ws, ws_bytes, w.total, dev));
  cudaStream_t st = as_stream(stream);
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  sdm_fp8_cache local;
  sdm_fp8_cache* c = cache;
  if (c == nullptr) {
    memset(&local, 0, sizeof(local));
    local.k8 = base + w.k8;
    local.v8t = base + w.v8t;
    local.scales = reinterpret_cast<float*>(base + w.scales);
    local.n_ctx = N;
    local.ld_v = round_up(N, kKvTile);
    local.batch = B;
    local.heads = H;
    local.head_dim = d;
    local.device = dev;
    local.ragged = 0;
    c = &local;
  }
  uint8_t* q8 = base + w.q8;
  QScale qs = make_qscale(N, c_h, gate);
  const int32_t* n_valid = nullptr;
  if (ctx_len != nullptr) {
    float* meta = c->scales + 3 * (int64_t)B * H;
    SDM_CUDA(put_meta(ctx_len, B, meta, st));
    n_valid = reinterpret_cast<const int32_t*>(meta);
    qs.lam_b = meta + B;
  }
  SDM_TRY(run_quantize(reinterpret_cast<const __half*>(q), reinterpret_cast<const __half*>(k),
                       reinterpret_cast<const __half*>(v), B, N, M, H, qs, q8, c->k8, c->v8t, c->ld_v, c->scales,
                       n_valid, base, w, st));
  c->filled = 1;
  c->ragged = ctx_len != nullptr ? 1 : 0;
  AttnArgs a;
  a.B = B;
  a.H = H;
  a.T = N + M;
  a.N = N;
  a.ld_v = c->ld_v;
  a.scales = c->scales;
  a.partial = false;
  a.n_splits = 1;
  a.split_keys = split_keys_for(N);
  a.out = reinterpret_cast<__half*>(out);
  a.part_acc = nullptr;
  a.part_ml = nullptr;
  a.err = reinterpret_cast<uint32_t*>(base);
  a.n_keys = n_valid;
  a.pad_rows = n_valid != nullptr;
  SDM_CUDA(launch_attention(q8, c->k8, c->v8t, a, st));
  return SDM_OK;
}

sdm_status sdm_icl_attention(const void* q, const void* k, const void* v, int32_t B, int64_t N, int64_t M,
                             int32_t H, int32_t d, const float* c_h, const void* gate, void* out,
                             sdm_fp8_cache* cache, void* ws, size_t ws_bytes, void* stream) {
  return icl_attention_impl(q, k, v, B, N, M, H, d, nullptr, c_h, gate, out, cache, ws, ws_bytes, stream);
}

sdm_status sdm_icl_attention_ragged(const void* q, const void* k, const void* v, int32_t B, int64_t N, int64_t M,
                                    int32_t H, int32_t d, const int64_t* ctx_len, const float* c_h,
                                    const void* gate, void* out, sdm_fp8_cache* cache, void* ws, size_t ws_bytes,
                                    void* stream) {
  if (ctx_len == nullptr) return SDM_ERR_INVALID_ARG;
  return icl_attention_impl(q, k, v, B, N, M, H, d, ctx_len, c_h, gate, out, cache, ws, ws_bytes, stream);
}



sdm_status sdm_cached_attention(const void* q, int32_t B, int64_t M, int32_t H, int32_t d,
                                const sdm_fp8_cache* cache, const float* c_h, const void* gate, void* out, void* ws,
                                size_t ws_bytes, void* stream) {
  if (cache == nullptr) return SDM_ERR_INVALID_ARG;
  SDM_TRY(check_shape(B, cache->n_ctx, M, H, d));
  const int dev = current_device();
  if (dev < 0) return SDM_ERR_CUDA;
  SDM_TRY(check_cache(cache, B, H, d, dev, true));
  if (c_h == nullptr || !aligned(c_h, 4)) return SDM_ERR_INVALID_ARG;
  if (!on_device(c_h, dev)) return SDM_ERR_DEVICE_MISMATCH;
  if (M == 0) return SDM_OK;
  SDM_TRY(check_tensor(q, dev));
  SDM_TRY(check_tensor(out, dev));
  if (gate != nullptr) {
    if (!aligned(gate, 2)) return SDM_ERR_INVALID_ARG;
    if (!on_device(gate, dev)) return SDM_ERR_DEVICE_MISMATCH;
  }
  const int64_t N = cache->n_ctx;
  const WsLayout w = ws_layout(SDM_OP_CACHED_ATTENTION, B, N, M, H, 1);
  SDM_TRY(check_ws(ws, ws_bytes, w.total, dev));
  cudaStream_t st = as_stream(stream);
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  uint8_t* q8 = base + w.q8;
  // query scaling with the shared key length n = N, quantised with the context s_q
  // (ragged cache: with the batch's own n_b and keys [0, n_b))
  RowsDesc dq{reinterpret_cast<const __half*>(q), B, H, M};
  QScale qs = make_qscale(N, c_h, gate);
  const float* meta = cache->scales + 3 * (int64_t)B * H;
  if (cache->ragged) qs.lam_b = meta + B;
  SDM_CUDA(prepare_gate(qs, (int64_t)B * M * H, base, w, st));
  SDM_CUDA(launch_quantize_rows(dq, qs, M, cache->scales, q8, M, nullptr, 0, st));
  AttnArgs a;
  a.B = B;
  a.H = H;
  a.T = M;
  a.N = N;
  a.ld_v = cache->ld_v;
  a.scales = cache->scales;
  a.partial = true;
  a.n_splits = n_splits_for(N);
  a.split_keys = split_keys_for(N);
  a.out = reinterpret_cast<__half*>(out);
  a.part_acc = reinterpret_cast<float*>(base + w.part_acc);
  a.part_ml = reinterpret_cast<float*>(base + w.part_ml);
  a.err = reinterpret_cast<uint32_t*>(base);
  a.n_keys = cache->ragged ? reinterpret_cast<const int32_t*>(meta) : nullptr;
  a.pad_rows = false;
  SDM_CUDA(launch_attention(q8, cache->k8, cache->v8t, a, st));
  SDM_CUDA(launch_splitkv_reduce(a, st));
  return SDM_OK;
}

int32_t sdm_fp8_eligible(int64_t n_unmasked_ctx, int32_t final_layer) {
  return (final_layer == 0 && n_unmasked_ctx > SDM_FP8_MIN_CONTEXT) ? 1 : 0;
}

static sdm_status icl_attention_f16_impl(const void* q, const void* k, const void* v, int32_t B, int64_t N,
                                         int64_t M, int32_t H, int32_t d, const int64_t* ctx_len, const float* c_h,
                                         const void* gate, void* out, void* ws, size_t ws_bytes, void* stream) {
  SDM_TRY(check_shape(B, N, M, H, d));
  if (N < 1) return SDM_ERR_INVALID_ARG;
  if (ctx_len != nullptr) SDM_TRY(check_ctx_len(ctx_len, B, N));
  const int dev = current_device();
  if (dev < 0) return SDM_ERR_CUDA;
  SDM_TRY(check_tensor(q, dev));
  SDM_TRY(check_tensor(k, dev));
  SDM_TRY(check_tensor(v, dev));
  SDM_TRY(check_tensor(out, dev));
  if (c_h != nullptr) {
    if (!aligned(c_h, 4)) return SDM_ERR_INVALID_ARG;
    if (!on_device(c_h, dev)) return SDM_ERR_DEVICE_MISMATCH;
  }
  if (gate != nullptr) {
    if (c_h == nullptr || !aligned(gate, 2)) return SDM_ERR_INVALID_ARG;
    if (!on_device(gate, dev)) return SDM_ERR_DEVICE_MISMATCH;
  }
  const WsLayout w = ws_layout(SDM_OP_ICL_ATTENTION_F16, B, N, M, H, 0);
  SDM_TRY(check_ws(ws, ws_bytes, w.total, dev));
  cudaStream_t st = as_stream(stream);
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  const int64_t T = N + M;
  const int64_t ld = round_up(N, kKvTile);
  const int32_t* n_valid = nullptr;
  const float* lam_b = nullptr;
  if (ctx_len != nullptr) {
    float* meta = reinterpret_cast<float*>(base + w.meta);
    SDM_CUDA(put_meta(ctx_len, B, meta, st));
    n_valid = reinterpret_cast<const int32_t*>(meta);
    lam_b = meta + B;
  }
  const __half* qs = reinterpret_cast<const __half*>(q);
  if (c_h != nullptr) {
    __half* q16 = reinterpret_cast<__half*>(base + w.q16);
    QScale sc = make_qscale(N, c_h, gate);
    sc.lam_b = lam_b;
    SDM_CUDA(launch_qscale(qs, q16, B, T, H, sc, st));
    qs = q16;
  }
  __half* vt16 = reinterpret_cast<__half*>(base + w.vt16);
  RowsDesc dv{reinterpret_cast<const __half*>(v), B, H, N};
  SDM_CUDA(launch_transpose_vt_f16(dv, N, n_valid, vt16, ld, st));
  SDM_CUDA(launch_attention_f16(qs, reinterpret_cast<const __half*>(k), vt16, B, T, N, H, ld, n_valid,
                                reinterpret_cast<__half*>(out), reinterpret_cast<uint32_t*>(base), st));
  return SDM_OK;
}

sdm_status sdm_icl_attention_f16(const void* q, const void* k, const void* v, int32_t B, int64_t N, int64_t M,
                                 int32_t H, int32_t d, const float* c_h, const void* gate, void* out, void* ws,
                                 size_t ws_bytes, void* stream) {
  return icl_attention_f16_impl(q, k, v, B, N, M, H, d, nullptr, c_h, gate, out, ws, ws_bytes, stream);
}

sdm_status sdm_icl_attention_f16_ragged(const void* q, const void* k, const void* v, int32_t B, int64_t N,
                                        int64_t M, int32_t H, int32_t d, const int64_t* ctx_len, const float* c_h,
                                        const void* gate, void* out, void* ws, size_t ws_bytes, void* stream) {
  if (ctx_len == nullptr) return SDM_ERR_INVALID_ARG;
  return icl_attention_f16_impl(q, k, v, B, N, M, H, d, ctx_len, c_h, gate, out, ws, ws_bytes, stream);
}



sdm_status sdm_cached_attention_offload(const void* q, int32_t B, int64_t M, int32_t H, int32_t d,
                                        const sdm_fp8_cache* cache, const float* c_h, const void* gate, void* out,
                                        void* ws, size_t ws_bytes, void* stream, void* copy_stream) {
  if (cache == nullptr) return SDM_ERR_INVALID_ARG;
  SDM_TRY(check_shape(B, cache->n_ctx, M, H, d));
  const int dev = current_device();
  if (dev < 0) return SDM_ERR_CUDA;
  // the cache: K8 / V8^T in page-locked host memory (or on this device), scales block here
  if (cache->batch != B || cache->heads != H || cache->head_dim != d || cache->device != dev || cache->n_ctx < 1 ||
      cache->ld_v != round_up(cache->n_ctx, kKvTile) || (cache->ragged != 0 && cache->ragged != 1) ||
      cache->filled != 1)
    return SDM_ERR_CACHE_MISMATCH;
  if (cache->k8 == nullptr || cache->v8t == nullptr || cache->scales == nullptr) return SDM_ERR_INVALID_ARG;
  if (!aligned(cache->k8, 16) || !aligned(cache->v8t, 16) || !aligned(cache->scales, 16)) return SDM_ERR_INVALID_ARG;
  if (!pinned_or_device(cache->k8, dev) || !pinned_or_device(cache->v8t, dev) || !on_device(cache->scales, dev))
    return SDM_ERR_CACHE_MISMATCH;
  if (c_h == nullptr || !aligned(c_h, 4)) return SDM_ERR_INVALID_ARG;
  if (!on_device(c_h, dev)) return SDM_ERR_DEVICE_MISMATCH;
  if (M == 0) return SDM_OK;
  SDM_TRY(check_tensor(q, dev));
  SDM_TRY(check_tensor(out, dev));
  if (gate != nullptr) {
    if (!aligned(gate, 2)) return SDM_ERR_INVALID_ARG;
    if (!on_device(gate, dev)) return SDM_ERR_DEVICE_MISMATCH;
  }
  const int64_t N = cache->n_ctx;
  const WsLayout w = ws_layout(SDM_OP_CACHED_ATTENTION_OFFLOAD, B, N, M, H, 1);
  SDM_TRY(check_ws(ws, ws_bytes, w.total, dev));
  cudaStream_t st = as_stream(stream);
  cudaStream_t cs = copy_stream != nullptr ? as_stream(copy_stream) : st;
  const bool overlap = cs != st;
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  const int64_t BH = (int64_t)B * H;
  const int64_t L = split_keys_for(N);
  const int64_t C = n_splits_for(N);
  // events ordering the two streams: copies into a slot wait for the attention
  // that last read it; an attention waits for its slot's copies
  cudaEvent_t ev[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
  auto destroy = [&]() {
    for (cudaEvent_t& e : ev)
      if (e != nullptr) cudaEventDestroy(e);  // released once pending work completes
  };
  if (overlap) {
    for (cudaEvent_t& e : ev)
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
        cudaGetLastError();
        destroy();
        return SDM_ERR_CUDA;
      }
  }
  cudaEvent_t start = ev[0], copied[2] = {ev[1], ev[2]}, used[2] = {ev[3], ev[4]};
  sdm_status status = SDM_OK;
  do {
    if (overlap) {
      // the slots may still be read by work enqueued on `stream` before this call
      if (cudaEventRecord(start, st) != cudaSuccess || cudaStreamWaitEvent(cs, start, 0) != cudaSuccess) {
        status = SDM_ERR_CUDA;
        break;
      }
    }
    // queries: scaled with the cache's n (n_b if ragged), quantised with its s_q
    const float* meta = cache->scales + 3 * BH;
    RowsDesc dq{reinterpret_cast<const __half*>(q), B, H, M};
    QScale qs = make_qscale(N, c_h, gate);
    if (cache->ragged) qs.lam_b = meta + B;
    uint8_t* q8 = base + w.q8;
    if (prepare_gate(qs, (int64_t)B * M * H, base, w, st) != cudaSuccess ||
        launch_quantize_rows(dq, qs, M, cache->scales, q8, M, nullptr, 0, st) != cudaSuccess) {
      status = SDM_ERR_CUDA;
      break;
    }
    AttnArgs a;
    a.B = B;
    a.H = H;
    a.T = M;
    a.N = N;
    a.ld_v = L;
    a.kv_rows = L;
    a.scales = cache->scales;
    a.partial = true;
    a.n_splits = 1;
    a.split_keys = L;
    a.out = reinterpret_cast<__half*>(out);
    a.part_acc = reinterpret_cast<float*>(base + w.part_acc);
    a.part_ml = reinterpret_cast<float*>(base + w.part_ml);
    a.err = reinterpret_cast<uint32_t*>(base);
    a.n_keys = cache->ragged ? reinterpret_cast<const int32_t*>(meta) : nullptr;
    for (int64_t c = 0; c < C && status == SDM_OK; ++c) {
      const int r = static_cast<int>(c & 1);
      uint8_t* k_slot = base + w.stage + r * w.stage_bytes;
      uint8_t* v_slot = k_slot + BH * L * kHeadDim;
      const int64_t len = (N - c * L) < L ? (N - c * L) : L;      // keys of this chunk
      const int64_t vlen = (cache->ld_v - c * L) < L ? (cache->ld_v - c * L) : L;  // with V's zero padding
      if (overlap && c >= 2 && cudaStreamWaitEvent(cs, used[r], 0) != cudaSuccess) status = SDM_ERR_CUDA;
      // K8 rows [cL, cL + len) of every (b, h); V8^T columns [cL, cL + vlen) of every (b, h, e)
      if (status == SDM_OK &&
          (cudaMemcpy2DAsync(k_slot, L * kHeadDim, cache->k8 + c * L * kHeadDim, N * kHeadDim, len * kHeadDim, BH,
                             cudaMemcpyDefault, cs) != cudaSuccess ||
           cudaMemcpy2DAsync(v_slot, L, cache->v8t + c * L, cache->ld_v, vlen, BH * kHeadDim, cudaMemcpyDefault,
                             cs) != cudaSuccess))
        status = SDM_ERR_CUDA;
      if (status == SDM_OK && overlap &&
          (cudaEventRecord(copied[r], cs) != cudaSuccess || cudaStreamWaitEvent(st, copied[r], 0) != cudaSuccess))
        status = SDM_ERR_CUDA;
      a.key_base = c * L;
      a.split_base = c;
      if (status == SDM_OK && launch_attention(q8, k_slot, v_slot, a, st) != cudaSuccess) status = SDM_ERR_CUDA;
      if (status == SDM_OK && overlap && cudaEventRecord(used[r], st) != cudaSuccess) status = SDM_ERR_CUDA;
    }
    if (status != SDM_OK) break;
    a.n_splits = C;
    if (launch_splitkv_reduce(a, st) != cudaSuccess) status = SDM_ERR_CUDA;
  } while (false);
  if (status != SDM_OK) cudaGetLastError();
  destroy();
  return status;
}

// Host-side checks of a prefill batch; fills seqs on success.
static sdm_status prefill_batch(const int64_t* qo_indptr, const int64_t* kv_indptr, int32_t batch, int32_t q_heads,
                                int32_t kv_heads, int32_t head_dim, int32_t causal, std::vector<PrefillSeq>& seqs) {
  if (batch < 0 || qo_indptr == nullptr || kv_indptr == nullptr) return SDM_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SDM_ERR_INVALID_ARG;
  if (head_dim != 128) return SDM_ERR_UNSUPPORTED;
  if (q_heads < 1 || kv_heads < 1 || q_heads % kv_heads != 0) return SDM_ERR_INVALID_ARG;
  const int32_t G = q_heads / kv_heads;
  if (G > 16 || (G & (G - 1)) != 0 || q_heads > 256 || kv_heads > 256) return SDM_ERR_UNSUPPORTED;
  for (const int64_t* ip : {qo_indptr, kv_indptr}) {  // host arrays of batch + 1 offsets
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, ip) == cudaSuccess) {
      if (at.type == cudaMemoryTypeDevice) return SDM_ERR_INVALID_ARG;
    } else {
      cudaGetLastError();
    }
  }
  if (qo_indptr[0] != 0 || kv_indptr[0] != 0) return SDM_ERR_INVALID_ARG;
  seqs.resize(static_cast<size_t>(batch));
  for (int32_t b = 0; b < batch; ++b) {
    const int64_t ql = qo_indptr[b + 1] - qo_indptr[b], kl = kv_indptr[b + 1] - kv_indptr[b];
    if (ql < 0 || kl < 0 || (ql > 0 && kl < 1) || (causal && kl < ql)) return SDM_ERR_INVALID_ARG;
    seqs[b] = PrefillSeq{qo_indptr[b], ql, kv_indptr[b], kl};
  }
  // TMA coordinates and the kernel's offsets are 32-bit
  if (qo_indptr[batch] > ((int64_t)1 << 30) || kv_indptr[batch] > ((int64_t)1 << 30)) return SDM_ERR_UNSUPPORTED;
  return SDM_OK;
}

size_t sdm_gqa_prefill_workspace_size(const int64_t* qo_indptr, const int64_t* kv_indptr, int32_t batch,
                                      int32_t q_heads, int32_t kv_heads, int32_t head_dim, int32_t causal) {
  std::vector<PrefillSeq> seqs;
  if (prefill_batch(qo_indptr, kv_indptr, batch, q_heads, kv_heads, head_dim, causal, seqs) != SDM_OK) return 0;
  return gqa_prefill_ws_bytes(seqs.data(), batch, q_heads, kv_heads, causal);
}

sdm_status sdm_gqa_prefill(const void* q, const void* k, const void* v, const int64_t* qo_indptr,
                           const int64_t* kv_indptr, int32_t batch, int32_t q_heads, int32_t kv_heads,
                           int32_t head_dim, int32_t causal, void* out, void* ws, size_t ws_bytes, void* stream) {
  std::vector<PrefillSeq> seqs;
  SDM_TRY(prefill_batch(qo_indptr, kv_indptr, batch, q_heads, kv_heads, head_dim, causal, seqs));
  const int64_t total_q = qo_indptr[batch], total_kv = kv_indptr[batch];
  if (total_q == 0) return SDM_OK;
  const int dev = current_device();
  if (dev < 0) return SDM_ERR_CUDA;
  SDM_TRY(check_tensor(q, dev));
  SDM_TRY(check_tensor(k, dev));
  SDM_TRY(check_tensor(v, dev));
  SDM_TRY(check_tensor(out, dev));
  SDM_TRY(check_ws(ws, ws_bytes, gqa_prefill_ws_bytes(seqs.data(), batch, q_heads, kv_heads, causal), dev));
  SDM_CUDA(launch_gqa_prefill(q, k, v, total_q, total_kv, seqs.data(), batch, q_heads, kv_heads, causal, out,
                              reinterpret_cast<uint8_t*>(ws), as_stream(stream)));
  return SDM_OK;
}

// ---------------------------------------------------------------- step 4 by chunk ranges
// The cache descriptor without its K8 / V8^T buffers: shape, state, device and
// the scales block.
static sdm_status check_cache_meta(const sdm_fp8_cache* c, int32_t B, int32_t H, int32_t d, int dev) {
  if (c == nullptr) return SDM_ERR_INVALID_ARG;
  if (c->batch != B || c->heads != H || c->head_dim != d || c->device != dev || c->n_ctx < 1 ||
      c->ld_v != round_up(c->n_ctx, kKvTile) || (c->ragged != 0 && c->ragged != 1) || c->filled != 1)
    return SDM_ERR_CACHE_MISMATCH;
  if (c->scales == nullptr || !aligned(c->scales, 16)) return SDM_ERR_INVALID_ARG;
  if (!on_device(c->scales, dev)) return SDM_ERR_CACHE_MISMATCH;
  return SDM_OK;
}

sdm_status sdm_cached_partials(const void* q, int32_t B, int64_t M, int32_t H, int32_t d, const sdm_fp8_cache* cache,
                               const uint8_t* k8_slice, const uint8_t* v8t_slice, int64_t ld_slice, int64_t c0,
                               int64_t c1, const float* c_h, const void* gate, float* part_acc, float* part_ml,
                               void* ws, size_t ws_bytes, void* stream) {
  if (cache == nullptr) return SDM_ERR_INVALID_ARG;
  SDM_TRY(check_shape(B, cache->n_ctx, M, H, d));
  const int dev = current_device();
  if (dev < 0) return SDM_ERR_CUDA;
  SDM_TRY(check_cache_meta(cache, B, H, d, dev));
  const int64_t N = cache->n_ctx;
  const int64_t L = split_keys_for(N);
  const int64_t S = n_splits_for(N);
  if (c0 < 0 || c1 <= c0 || c1 > S) return SDM_ERR_INVALID_ARG;
  const int64_t n = (c1 * L < N ? c1 * L : N) - c0 * L;  // keys of the slice
  if (ld_slice < n || ld_slice % kKvTile != 0 || ld_slice > ((int64_t)1 << 30)) return SDM_ERR_INVALID_ARG;
  if (c_h == nullptr || !aligned(c_h, 4)) return SDM_ERR_INVALID_ARG;
  if (!on_device(c_h, dev)) return SDM_ERR_DEVICE_MISMATCH;
  if (M == 0) return SDM_OK;
  SDM_TRY(check_tensor(q, dev));
  SDM_TRY(check_tensor(k8_slice, dev));
  SDM_TRY(check_tensor(v8t_slice, dev));
  SDM_TRY(check_tensor(part_acc, dev));
  SDM_TRY(check_tensor(part_ml, dev));
  if (gate != nullptr) {
    if (!aligned(gate, 2)) return SDM_ERR_INVALID_ARG;
    if (!on_device(gate, dev)) return SDM_ERR_DEVICE_MISMATCH;
  }
  const WsLayout w = ws_layout(SDM_OP_CACHED_PARTIALS, B, N, M, H, 1);
  SDM_TRY(check_ws(ws, ws_bytes, w.total, dev));
  cudaStream_t st = as_stream(stream);
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  uint8_t* q8 = base + w.q8;
  // queries: scaled with the cache's n (n_b if ragged), quantised with its s_q
  const float* meta = cache->scales + 3 * (int64_t)B * H;
  RowsDesc dq{reinterpret_cast<const __half*>(q), B, H, M};
  QScale qs = make_qscale(N, c_h, gate);
  if (cache->ragged) qs.lam_b = meta + B;
  SDM_CUDA(prepare_gate(qs, (int64_t)B * M * H, base, w, st));
  SDM_CUDA(launch_quantize_rows(dq, qs, M, cache->scales, q8, M, nullptr, 0, st));
  AttnArgs a;
  a.B = B;
  a.H = H;
  a.T = M;
  a.N = N;
  a.ld_v = ld_slice;
  a.kv_rows = n;
  a.key_base = c0 * L;
  a.split_base = c0;
  a.scales = cache->scales;
  a.partial = true;
  a.n_splits = c1 - c0;
  a.split_keys = L;
  a.out = nullptr;
  a.part_acc = part_acc;
  a.part_ml = part_ml;
  a.err = reinterpret_cast<uint32_t*>(base);
  a.n_keys = cache->ragged ? reinterpret_cast<const int32_t*>(meta) : nullptr;
  a.pad_rows = false;
  SDM_CUDA(launch_attention(q8, k8_slice, v8t_slice, a, st));
  return SDM_OK;
}

sdm_status sdm_cached_combine(const float* part_acc, const float* part_ml, int32_t B, int64_t M, int32_t H, int32_t d,
                              const sdm_fp8_cache* cache, void* out, void* stream) {
  if (cache == nullptr) return SDM_ERR_INVALID_ARG;
  SDM_TRY(check_shape(B, cache->n_ctx, M, H, d));
  const int dev = current_device();
  if (dev < 0) return SDM_ERR_CUDA;
  SDM_TRY(check_cache_meta(cache, B, H, d, dev));
  if (M == 0) return SDM_OK;
  SDM_TRY(check_tensor(part_acc, dev));
  SDM_TRY(check_tensor(part_ml, dev));
  SDM_TRY(check_tensor(out, dev));
  AttnArgs a;
  a.B = B;
  a.H = H;
  a.T = M;
  a.N = cache->n_ctx;
  a.ld_v = cache->ld_v;
  a.scales = cache->scales;
  a.partial = true;
  a.n_splits = n_splits_for(cache->n_ctx);
  a.split_keys = split_keys_for(cache->n_ctx);
  a.out = reinterpret_cast<__half*>(out);
  a.part_acc = const_cast<float*>(part_acc);
  a.part_ml = const_cast<float*>(part_ml);
  a.err = nullptr;
  SDM_CUDA(launch_splitkv_reduce(a, as_stream(stream)));
  return SDM_OK;
}

// ---------------------------------------------------------------- sharded step 2
// Argument checks shared by sdm_context_amax and sdm_quantize_with_scales: the
// query-scaling inputs (c_h == NULL: q is already scaled) and the slice tensors.
static sdm_status check_slice(const void* q, const void* k, const void* v, int64_t n_ctx, int64_t n_len,
                              const float* c_h, const void* gate, int dev) {
  SDM_TRY(check_tensor(q, dev));
  if (n_ctx > 0) {
    SDM_TRY(check_tensor(k, dev));
    SDM_TRY(check_tensor(v, dev));
  }
  if (c_h != nullptr) {
    if (n_len < 1 || !aligned(c_h, 4)) return SDM_ERR_INVALID_ARG;
    if (!on_device(c_h, dev)) return SDM_ERR_DEVICE_MISMATCH;
    if (gate != nullptr) {
      if (!aligned(gate, 2)) return SDM_ERR_INVALID_ARG;
      if (!on_device(gate, dev)) return SDM_ERR_DEVICE_MISMATCH;
    }
  }
  return SDM_OK;
}

static QScale slice_qscale(int64_t n_len, const float* c_h, const void* gate) {
  // the gate factors are evaluated in place (no workspace to hold them)
  return c_h != nullptr ? make_qscale(n_len, c_h, gate) : no_qscale();
}

sdm_status sdm_context_amax(const void* q, const void* k, const void* v, int32_t B, int64_t n_ctx, int64_t q_rows,
                            int32_t H, int32_t d, int64_t n_len, const float* c_h, const void* gate, float* amax,
                            void* stream) {
  SDM_TRY(check_shape(B, n_ctx, q_rows, H, d));
  if (q_rows < n_ctx) return SDM_ERR_INVALID_ARG;
  const int dev = current_device();
  if (dev < 0) return SDM_ERR_CUDA;
  if (n_ctx > 0) SDM_TRY(check_slice(q, k, v, n_ctx, n_len, c_h, gate, dev));
  SDM_TRY(check_tensor(amax, dev));
  cudaStream_t st = as_stream(stream);
  uint32_t* words = reinterpret_cast<uint32_t*>(amax);  // fp32 bits of values >= 0: integer max = float max
  SDM_CUDA(cudaMemsetAsync(words, 0, 3 * (size_t)B * H * sizeof(uint32_t), st));
  if (n_ctx == 0) return SDM_OK;
  RowsDesc dq{reinterpret_cast<const __half*>(q), B, H, q_rows};
  RowsDesc dk{reinterpret_cast<const __half*>(k), B, H, n_ctx};
  RowsDesc dv{reinterpret_cast<const __half*>(v), B, H, n_ctx};
  SDM_CUDA(launch_context_amax(dq, slice_qscale(n_len, c_h, gate), dk, dv, n_ctx, nullptr, words, st));
  return SDM_OK;
}

sdm_status sdm_quantize_with_scales(const void* q, const void* k, const void* v, int32_t B, int64_t n_ctx,
                                    int64_t n_query, int32_t H, int32_t d, int64_t n_len, const float* c_h,
                                    const void* gate, const float* amax, float* scales, uint8_t* q8, uint8_t* k8,
                                    int64_t ld_k, uint8_t* v8t, int64_t ld_v, void* stream) {
  SDM_TRY(check_shape(B, n_ctx, n_query, H, d));
  const int64_t T = n_ctx + n_query;
  if (n_ctx > 0 && (ld_k < n_ctx || ld_k > ((int64_t)1 << 30) || ld_v < n_ctx || ld_v % kKvTile != 0))
    return SDM_ERR_INVALID_ARG;
  const int dev = current_device();
  if (dev < 0) return SDM_ERR_CUDA;
  if (T > 0) {
    SDM_TRY(check_slice(q, k, v, n_ctx, n_len, c_h, gate, dev));
    SDM_TRY(check_tensor(q8, dev));
  }
  SDM_TRY(check_tensor(amax, dev));
  SDM_TRY(check_tensor(scales, dev));
  if (n_ctx > 0) {
    SDM_TRY(check_tensor(k8, dev));
    SDM_TRY(check_tensor(v8t, dev));
  }
  cudaStream_t st = as_stream(stream);
  const int64_t BH = (int64_t)B * H;
  SDM_CUDA(launch_scales_from_amax(reinterpret_cast<const uint32_t*>(amax), B * H, scales, st));
  if (T == 0) return SDM_OK;
  RowsDesc dq{reinterpret_cast<const __half*>(q), B, H, T};
  SDM_CUDA(launch_quantize_rows(dq, slice_qscale(n_len, c_h, gate), T, scales, q8, T, nullptr, 0, st));
  if (n_ctx > 0) {
    RowsDesc dk{reinterpret_cast<const __half*>(k), B, H, n_ctx};
    RowsDesc dv{reinterpret_cast<const __half*>(v), B, H, n_ctx};
    SDM_CUDA(launch_quantize_rows(dk, no_qscale(), n_ctx, scales + BH, k8, ld_k, nullptr, 0, st));
    SDM_CUDA(launch_quantize_vt(dv, n_ctx, nullptr, scales + 2 * BH, v8t, ld_v, st));
  }
  return SDM_OK;
}

sdm_status sdm_cache_put_rows(sdm_fp8_cache* cache, const uint8_t* k8_rows, int64_t ld_k, const uint8_t* v8t_cols,
                              int64_t ld_v, int64_t row0, int64_t n, void* stream) {
  if (cache == nullptr) return SDM_ERR_INVALID_ARG;
  const int dev = current_device();
  if (dev < 0) return SDM_ERR_CUDA;
  SDM_TRY(check_cache(cache, cache->batch, cache->heads, cache->head_dim, dev, false));
  if (n < 0 || row0 < 0 || row0 + n > cache->n_ctx || ld_k < n || ld_v < n) return SDM_ERR_INVALID_ARG;
  if (n == 0) return SDM_OK;
  SDM_TRY(check_tensor(k8_rows, dev));
  SDM_TRY(check_tensor(v8t_cols, dev));
  cudaStream_t st = as_stream(stream);
  const int64_t BH = (int64_t)cache->batch * cache->heads;
  const int64_t N = cache->n_ctx;
  // K8: one block of n rows (n*64 bytes) per (b, h) plane
  SDM_CUDA(cudaMemcpy2DAsync(cache->k8 + row0 * kHeadDim, (size_t)N * kHeadDim, k8_rows, (size_t)ld_k * kHeadDim,
                             (size_t)n * kHeadDim, (size_t)BH, cudaMemcpyDeviceToDevice, st));
  // V8^T: n columns of each of the B*H*64 rows
  SDM_CUDA(cudaMemcpy2DAsync(cache->v8t + row0, (size_t)cache->ld_v, v8t_cols, (size_t)ld_v, (size_t)n,
                             (size_t)BH * kHeadDim, cudaMemcpyDeviceToDevice, st));
  return SDM_OK;
}

sdm_status sdm_selftest_wait_timeout(void* ws, int64_t limit_cycles, void* stream) {
  if (ws == nullptr || !aligned(ws, 256)) return SDM_ERR_INVALID_ARG;
  if (limit_cycles < 1000 || limit_cycles > ((int64_t)1 << 31)) return SDM_ERR_INVALID_ARG;
  const int dev = current_device();
  if (dev < 0) return SDM_ERR_CUDA;
  if (!on_device(ws, dev)) return SDM_ERR_DEVICE_MISMATCH;
  SDM_CUDA(launch_wait_selftest(reinterpret_cast<uint32_t*>(ws), limit_cycles, as_stream(stream)));
  return SDM_OK;
}

sdm_status sdm_sync_status(void* ws, void* stream, uint32_t* flags) {
  if (ws == nullptr) return SDM_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess) {
    cudaGetLastError();
    return SDM_ERR_CUDA;
  }
  if (flags) *flags = word;
  if (word != 0) {
    if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), st) != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess) {
      cudaGetLastError();
      return SDM_ERR_CUDA;
    }
    return SDM_ERR_TIMEOUT;
  }
  return SDM_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Context quantisation for callers that cannot provide a workspace.
//
// Some callers of this library cannot allocate device memory for it: code on a
// latency-critical path that must not call cudaMalloc (which can synchronise
// the whole device), plugins whose host framework owns all device memory
// behind its own allocator, and hooks that run where no allocation API is
// reachable.  The only scratch the quantisation step needs is its per-(tensor,
// batch, head) amax accumulator, so this variant keeps it in a fixed
// file-scope device array instead of the caller's workspace.  The array is
// part of the library image: every GPU that loads the library holds it
// (48 KiB) until the process exits.
namespace {

constexpr int kNoAllocMaxBatchHeads = SDM_NOALLOC_MAX_BATCH_HEADS;
static __device__ __align__(256) uint32_t g_noalloc_amax[3 * kNoAllocMaxBatchHeads];

// In host code `g_noalloc_amax` names a host-side stand-in, not device memory,
// so kernels must be given the address the runtime reports for it -- looked up
// with the device current, once per device and CUDA context: the address is
// taken again when the device's current context is not the one it was taken in
// (after cudaDeviceReset, or a primary context released and created anew), so
// no call uses an address of a context that is gone.
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
struct NoAllocSlot {
  CUcontext ctx;
  uint32_t* addr;
};
NoAllocSlot g_noalloc_slot[kNoAllocMaxDevices] = {};

// cuCtxGetCurrent through the runtime's driver entry point (the library does
// not link libcuda); looked up once per process.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current() {
  static const CtxGetCurrentFn fn = []() -> CtxGetCurrentFn {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<CtxGetCurrentFn>(ptr);
    return nullptr;
  }();
  return fn;
}

sdm_status noalloc_scratch(int dev, uint32_t** out) {
  if (dev < 0 || dev >= kNoAllocMaxDevices) return SDM_ERR_UNSUPPORTED;
  const CtxGetCurrentFn get_ctx = ctx_get_current();
  CUcontext ctx = nullptr;  // null if no runtime call has made the primary context current yet
  if (get_ctx == nullptr || get_ctx(&ctx) != CUDA_SUCCESS) return SDM_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocSlot& slot = g_noalloc_slot[dev];
  if (slot.addr == nullptr || ctx == nullptr || slot.ctx != ctx) {
    void* p = nullptr;
    // also makes the device's primary context current if it was not yet
    if (cudaGetSymbolAddress(&p, g_noalloc_amax) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      slot.addr = nullptr;
      return SDM_ERR_CUDA;
    }
    if (ctx == nullptr && (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr)) {
      slot.addr = nullptr;
      return SDM_ERR_CUDA;
    }
    slot.ctx = ctx;
    slot.addr = static_cast<uint32_t*>(p);
  }
  *out = slot.addr;
  return SDM_OK;
}

}  // namespace

extern "C" sdm_status sdm_fp8_quantize_context_noalloc(const void* q_scaled, const void* k, const void* v,
                                                       int32_t B, int64_t N, int64_t M, int32_t H, int32_t d,
                                                       uint8_t* q8, sdm_fp8_cache* cache, void* stream) {
  SDM_TRY(check_shape(B, N, M, H, d));
  if (N < 1) return SDM_ERR_INVALID_ARG;
  if ((int64_t)B * H > kNoAllocMaxBatchHeads) return SDM_ERR_UNSUPPORTED;
  const int dev = current_device();
  if (dev < 0) return SDM_ERR_CUDA;
  SDM_TRY(check_tensor(q_scaled, dev));
  SDM_TRY(check_tensor(k, dev));
  SDM_TRY(check_tensor(v, dev));
  SDM_TRY(check_tensor(q8, dev));
  SDM_TRY(check_cache(cache, B, H, d, dev, false));
  if (cache->n_ctx != N) return SDM_ERR_CACHE_MISMATCH;
  uint32_t* amax = nullptr;
  SDM_TRY(noalloc_scratch(dev, &amax));
  cudaStream_t st = as_stream(stream);
  const int64_t T = N + M;
  const int64_t BH = (int64_t)B * H;
  // the array keeps whatever the previous call left: the max accumulators restart at zero
  SDM_CUDA(cudaMemsetAsync(amax, 0, 3 * (size_t)BH * sizeof(uint32_t), st));
  RowsDesc dq{reinterpret_cast<const __half*>(q_scaled), B, H, T};
  RowsDesc dk{reinterpret_cast<const __half*>(k), B, H, N};
  RowsDesc dv{reinterpret_cast<const __half*>(v), B, H, N};
  SDM_CUDA(launch_context_amax(dq, no_qscale(), dk, dv, N, nullptr, amax, st));
  SDM_CUDA(launch_scales_from_amax(amax, B * H, cache->scales, st));
  SDM_CUDA(launch_quantize_rows(dq, no_qscale(), T, cache->scales, q8, T, nullptr, 0, st));
  SDM_CUDA(launch_quantize_rows(dk, no_qscale(), N, cache->scales + BH, cache->k8, N, nullptr, 0, st));
  SDM_CUDA(launch_quantize_vt(dv, N, nullptr, cache->scales + 2 * BH, cache->v8t, cache->ld_v, st));
  cache->filled = 1;
  cache->ragged = 0;
  return SDM_OK;
}
