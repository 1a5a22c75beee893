// kernels.cuh -- launch wrappers shared by the C-ABI layer (api.cu) and the
// kernel files.  Internal to the library; the public interface is sdm_fp8.h.
#pragma once
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sdm {
// cuTensorMapEncodeTiled, reached through the runtime's driver entry point (the
// library does not link libcuda).  Looked up once per process; C++ makes the
// initialisation of the local static thread-safe.  nullptr if unavailable.
using TensorMapEncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                       const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                       CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                       CUtensorMapFloatOOBfill);
inline TensorMapEncodeFn tensor_map_encoder() {
  static const TensorMapEncodeFn fn = []() -> TensorMapEncodeFn {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<TensorMapEncodeFn>(ptr);
    return nullptr;
  }();
  return fn;
}
}  // namespace sdm

namespace sdm {

constexpr int kHeadDim = 64;   // the only head dimension the kernels are built for
constexpr int kKvTile = 128;   // keys per online-softmax block (one tcgen05 N=128 tile)
constexpr int kQTile = 128;    // query rows per tensor-core tile (M=128)
// Cached prediction: keys per split-KV chunk, a function of the context length
// alone (so a query's result never depends on the batch it came in): about 32
// chunks, each a multiple of 128 keys, between 1024 and 16384 keys.
constexpr int64_t kSplitMin = 1024, kSplitMax = 16384, kSplitTarget = 32;
inline int64_t split_keys_for(int64_t n_ctx) {
  const int64_t per = (n_ctx + kSplitTarget * kKvTile - 1) / (kSplitTarget * kKvTile) * kKvTile;
  return per < kSplitMin ? kSplitMin : (per > kSplitMax ? kSplitMax : per);
}

// Query-scaling parameters shared by the elementwise kernels.
struct QScale {
  bool enabled;        // false: the input already is q' (or is K / V)
  float lam;           // fp32 ln(max(n,1)), evaluated on the host from the integer length
  const float* c_h;    // [H] per-head coefficients (device)
  const __half* gate;  // [B][rows][H] or nullptr (LogScale)
  const __half* gate_w;  // [B][rows][H] precomputed fp16(1 + fp16(tanh g)), or nullptr: evaluate in place
  const float* lam_b;  // [B] per-batch lam (device; ragged contexts), or nullptr: lam for every batch
};

// Ragged contexts: batch b has n_b = n_valid[b] unmasked context rows (rows
// [n_b, N) are padding).  The per-batch lengths and their lam live in device
// memory right after the [3][B][H] scales ("scales block"): n_b as int32 [B],
// then lam_b as fp32 [B].
inline size_t scales_block_words(int64_t B, int64_t H, bool ragged) { return 3 * B * H + (ragged ? 2 * B : 0); }
constexpr int kMetaChunk = 256;  // batches per meta-writing launch (kernel-parameter payload)
struct MetaChunk {
  int32_t b0, count;
  int32_t n[kMetaChunk];
  float lam[kMetaChunk];
};
// Writes n_b and lam_b of batches [b0, b0 + count) into the scales block's meta words.
cudaError_t launch_write_meta(const MetaChunk& c, int32_t* n_dst, float* lam_dst, cudaStream_t st);

// Tensor-wide problem description for the elementwise kernels.
struct RowsDesc {
  const __half* x;     // [B][rows][H][64]
  int32_t B, H;
  int64_t rows;        // rows per batch in x's layout
};

cudaError_t launch_qscale(const __half* q, __half* out, int32_t B, int64_t rows, int32_t H, QScale qs,
                          cudaStream_t st);  // qs.lam_b, if set, is indexed by b

// w[i] = fp16(1 + fp16(tanh(gate[i]))) for i < n: the GatedLogScale factor, once per (row, head).
cudaError_t launch_gate_factors(const __half* gate, int64_t n, __half* w, cudaStream_t st);

// amax words: [3][B][H] uint32 (float bits, values >= 0).  Must be zeroed first.
// Context rows [0, n_valid ? n_valid[b] : n_ctx) of each batch.
cudaError_t launch_context_amax(RowsDesc q, QScale qs, RowsDesc k, RowsDesc v, int64_t n_ctx,
                                const int32_t* n_valid, uint32_t* amax, cudaStream_t st);

// scales[3][B][H] = amax/448 (1 where amax == 0); from the amax words.
cudaError_t launch_scales_from_amax(const uint32_t* amax, int32_t BH, float* scales, cudaStream_t st);

// Row-major quantisation: dst[b][h][r][64] = e4m3(qscale?(x[b][r][h][:]) / scale[b*H+h]),
// rows [0, n_rows) of x; dst has dst_rows rows per (b, h).  With n_valid, rows
// [n_valid[b], pad_end) are padding and get zero codes.
cudaError_t launch_quantize_rows(RowsDesc x, QScale qs, int64_t n_rows, const float* scale, uint8_t* dst,
                                 int64_t dst_rows, const int32_t* n_valid, int64_t pad_end, cudaStream_t st);

// Transposed quantisation for V: dst[b][h][e][ld] for keys [0, n_b), zeros in
// [n_b, round_up(n_ctx, 128)); n_b = n_valid ? n_valid[b] : n_ctx.
cudaError_t launch_quantize_vt(RowsDesc v, int64_t n_ctx, const int32_t* n_valid, const float* scale, uint8_t* dst,
                               int64_t ld, cudaStream_t st);

// fp16 transpose of V for the normal-precision attention: dst[b][h][e][ld] =
// v[b][key][h][e] for keys [0, n_b), zeros in [n_b, round_up(n_ctx, 128));
// n_b = n_valid ? n_valid[b] : n_ctx.
cudaError_t launch_transpose_vt_f16(RowsDesc v, int64_t n_ctx, const int32_t* n_valid, __half* dst, int64_t ld,
                                    cudaStream_t st);

// fp16 attention of rows [0, T) of q_scaled [B][T][H][64] to keys [0, n_b) of
// k [B][N][H][64] and vt [B][H][64][ld]; out [B][T][H][64] fp16.  With
// n_keys, n_b = n_keys[b] and rows [n_b, N) (padding) are written as zeros.
cudaError_t launch_attention_f16(const __half* q_scaled, const __half* k, const __half* vt, int32_t B, int64_t T,
                                 int64_t N, int32_t H, int64_t ld_v, const int32_t* n_keys, __half* out,
                                 uint32_t* err, cudaStream_t st);

// Ragged grouped-query prefill (bf16, head dim 128): one sequence's token ranges
// in the packed q and k/v tensors.  Sequences are launched 64 at a time.
constexpr int kPrefillMaxSeqs = 64;
struct PrefillSeq {
  int64_t q_off, q_len, kv_off, kv_len;
};
// out [total_q][q_heads][128] = attention of q [total_q][q_heads][128] to k, v
// [total_kv][kv_heads][128] (bf16), query head h reading key/value head
// h / (q_heads / kv_heads); causal: the queries are the last q_len keys.
// ws: the error word.  Each query tile is one cluster of 4 CTAs, each with a
// quarter of the tile's keys; the cluster combines them in shared memory.
cudaError_t launch_gqa_prefill(const void* q, const void* k, const void* v, int64_t total_q, int64_t total_kv,
                               const PrefillSeq* seqs, int32_t n_seqs, int32_t q_heads, int32_t kv_heads,
                               int32_t causal, void* out, uint8_t* ws, cudaStream_t st);
size_t gqa_prefill_ws_bytes(const PrefillSeq* seqs, int32_t n_seqs, int32_t q_heads, int32_t kv_heads,
                            int32_t causal);

// ---------------------------------------------------------------- attention
struct AttnArgs {
  int32_t B, H;
  int64_t T;           // query rows per (b, h) in the Q8 layout
  int64_t N;           // context keys
  int64_t ld_v;        // V8 transposed row length (keys), multiple of 128
  const float* scales; // [3][B][H]: s_q, s_k, s_v
  bool partial;        // false: one pass, normalised fp16 output; true: split-KV partials
  int64_t n_splits;    // number of key chunks (1 when !partial)
  int64_t split_keys;  // keys per chunk (multiple of kKvTile) when partial
  __half* out;         // final: [B][T][H][64] fp16
  float* part_acc;     // split: [S][B*H][T][64]
  float* part_ml;      // split: [S][B*H][T][2] (m2, l)
  uint32_t* err;       // device error word
  const int32_t* n_keys = nullptr;  // [B] keys per batch (ragged contexts), or nullptr: N for every batch
  bool pad_rows = false;  // rows [n_keys[b], N) are padding context rows: written as zeros
  // A staged chunk of a cache held elsewhere: the K8 / V8^T buffers hold keys
  // [key_base, key_base + kv_rows) of the N; the launch (partial, one split of
  // split_keys keys) writes its partials at split index split_base.
  int64_t kv_rows = 0;     // rows of the K8 buffer (0: N)
  int64_t key_base = 0;
  int64_t split_base = 0;
};

// Builds the tensor maps and launches the tcgen05 attention kernel.
cudaError_t launch_attention(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8t, const AttnArgs& a,
                             cudaStream_t st);
// Combines split-KV partials in split order into the fp16 output.
cudaError_t launch_splitkv_reduce(const AttnArgs& a, cudaStream_t st);

// Device error word bits.
constexpr uint32_t kErrTimeoutQ = 1u << 0;
constexpr uint32_t kErrTimeoutKV = 1u << 1;
constexpr uint32_t kErrTimeoutS = 1u << 2;
constexpr uint32_t kErrTimeoutP = 1u << 3;
constexpr uint32_t kErrTimeoutO = 1u << 4;
constexpr uint32_t kErrTimeoutEmpty = 1u << 5;
constexpr uint32_t kErrTimeoutDrain = 1u << 6;
constexpr uint32_t kErrTimeoutSelfTest = 1u << 7;

// One warp waits, with the kernels' bounded wait, on an mbarrier that nothing
// arrives at; when `limit` cycles pass it ORs kErrTimeoutSelfTest into *err.
cudaError_t launch_wait_selftest(uint32_t* err, long long limit, cudaStream_t st);

}  // namespace sdm
