// quant.cu -- HBM-bound elementwise kernels of the layer:
//   * fused LogScale / GatedLogScale query scaling ("Fuse shared-length query
//     scaling during inference", section "Solution": length preparation,
//     per-head conversion, query multiply and optional gate in one kernel,
//     float32 length arithmetic, every eager fp16 rounding boundary kept);
//   * per-head amax over the context rows of Q', K and V, and the
//     scale = amax / 448 ("[FP8 3/4] Integrate FP8 attention and caching into
//     TabICLv2", opening section: Q scales are derived from context rows only);
//   * e4m3 quantisation (round to nearest even, saturating) into the
//     head-major layouts the attention kernel loads with TMA.
// Each thread moves one 16-byte vector (8 fp16) per step; a (row, head)
// segment of 64 elements is 8 consecutive lanes, so warps read whole rows.
#include "kernels.cuh"
#include "ptx.cuh"

namespace sdm {
namespace {

constexpr int kUnroll = 4;  // 16-byte loads in flight per thread

__device__ __forceinline__ float head_scale(const QScale& qs, int h, int64_t b) {
  // s_h = fp16(c_h * lam): fp32 product, one rounding to the query dtype;
  // lam is the batch's own with ragged contexts.
  const float lam = qs.lam_b != nullptr ? __ldg(qs.lam_b + b) : qs.lam;
  return __half2float(__float2half_rn(__fmul_rn(__ldg(qs.c_h + h), lam)));
}

// w = fp16(1 + fp16(tanh g)); tanh evaluated in double and rounded once to fp16.
__device__ __forceinline__ __half gate_factor_of(__half g) {
  const __half u = __double2half(tanh(static_cast<double>(__half2float(g))));
  return __float2half_rn(__fadd_rn(1.0f, __half2float(u)));
}

__device__ __forceinline__ float gate_factor(const QScale& qs, int64_t br, int H, int h) {
  if (qs.gate_w != nullptr) return __half2float(qs.gate_w[br * H + h]);
  return __half2float(gate_factor_of(qs.gate[br * H + h]));
}

// One fp16 element through the eager chain: q1 = fp16(q*s), gated: fp16(q1*w).
__device__ __forceinline__ float qscale1(float q, float s, bool gated, float w) {
  float q1 = __half2float(__float2half_rn(__fmul_rn(q, s)));
  if (gated) q1 = __half2float(__float2half_rn(__fmul_rn(q1, w)));
  return q1;
}

// x / s correctly rounded, for a divisor s > 0 that stays fixed over many x:
// with y = RN(1/s) and q = RN(x*y), the remainder r = x - q*s is exact in one
// fma and RN(q + r*y) equals RN(x/s) (Markstein's correction step, IEEE
// binary32, valid while nothing under- or overflows: here |x/s| <= 448 and
// s >= 2^-33).  The one case it gets wrong is the sign of a zero (x = -0 gives
// +0 + -0 = +0), so the result takes x's sign, which is the sign of x/s for
// every x because s > 0.  Three FMA-pipe operations per pair of elements plus a
// sign copy each, instead of a division each.
struct Divider {
  float y, neg_s;
};
__device__ __forceinline__ Divider make_divider(float s) { return {__frcp_rn(s), -s}; }
__device__ __forceinline__ void divide8(float (&f)[8], const Divider& d) {
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    float q0, q1, r0, r1, d0, d1;
    mul2(q0, q1, f[i], f[i + 1], d.y, d.y);
    fma2(r0, r1, q0, q1, d.neg_s, d.neg_s, f[i], f[i + 1]);
    fma2(d0, d1, r0, r1, d.y, d.y, q0, q1);
    f[i] = copysignf(d0, f[i]);
    f[i + 1] = copysignf(d1, f[i + 1]);
  }
}

__device__ __forceinline__ void unpack8(const uint4& raw, float (&f)[8]) {
  const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 p = __half22float2(h2[i]);
    f[2 * i] = p.x;
    f[2 * i + 1] = p.y;
  }
}

// Threads per CTA for the row kernels: a multiple of 8*H (so a thread keeps
// one head for its whole life), about 256.
inline int row_threads(int H) {
  const int seg = 8 * H;
  const int k = seg >= 256 ? 1 : 256 / seg;
  return seg * k;
}

// SMs of the current device (a cheap attribute query: no caching, so several
// devices and several host threads need no coordination).
inline int num_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    sms = 148;
  return sms;
}

// ---------------------------------------------------------------- qscale
__global__ void __launch_bounds__(256) qscale_kernel(const __half* __restrict__ q, __half* __restrict__ out,
                                                     int64_t n_vec, int H, int64_t rows, QScale qs) {
  const bool gated = qs.gate != nullptr;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i0 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i0 < n_vec; i0 += kUnroll * stride) {
    uint4 raw[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)  // all loads first: kUnroll 16-byte requests in flight
      if (i0 + u * stride < n_vec) raw[u] = __ldcs(reinterpret_cast<const uint4*>(q) + i0 + u * stride);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = i0 + u * stride;
      if (i >= n_vec) break;
      const int64_t seg = i >> 3;  // (b*rows + r)*H + h
      const int h = static_cast<int>(seg % H);
      const int64_t br = seg / H;
      const float s = head_scale(qs, h, qs.lam_b != nullptr ? br / rows : 0);
      const float w = gated ? gate_factor(qs, br, H, h) : 1.0f;
      float f[8];
      unpack8(raw[u], f);
      uint4 res;
      __half2* r2 = reinterpret_cast<__half2*>(&res);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        r2[k] = __halves2half2(__float2half_rn(qscale1(f[2 * k], s, gated, w)),
                               __float2half_rn(qscale1(f[2 * k + 1], s, gated, w)));
      __stcs(reinterpret_cast<uint4*>(out) + i, res);
    }
  }
}

__global__ void __launch_bounds__(256) gate_factor_kernel(const __half* __restrict__ gate, int64_t n,
                                                          __half* __restrict__ w) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    w[i] = gate_factor_of(gate[i]);
}

// ------------------------------------------------------------ context amax
// grid: (B * chunks, 3); blockIdx.y selects Q' (query scaling applied), K, V.
__global__ void context_amax_kernel(RowsDesc q, QScale qs, RowsDesc k, RowsDesc v, int64_t n_ctx,
                                    const int32_t* __restrict__ n_valid, int64_t rows_per_cta, int chunks,
                                    uint32_t* __restrict__ amax) {
  __shared__ uint32_t s_max[128];
  const int tensor = blockIdx.y;
  const RowsDesc X = tensor == 0 ? q : (tensor == 1 ? k : v);
  const bool do_q = tensor == 0 && qs.enabled;
  const bool gated = do_q && qs.gate != nullptr;
  const int H = X.H;
  const int t = threadIdx.x;
  const int vecs_per_row = 8 * H;
  const int vrow = t % vecs_per_row;
  const int h = vrow >> 3;
  const int row_step = blockDim.x / vecs_per_row;
  const int b = blockIdx.x / chunks;
  const int64_t r0 = (blockIdx.x % chunks) * rows_per_cta;
  const int64_t n_b = n_valid != nullptr ? (int64_t)__ldg(n_valid + b) : n_ctx;
  const int64_t r1 = min(n_b, r0 + rows_per_cta);
  if (t < H) s_max[t] = 0u;
  __syncthreads();

  const float s = do_q ? head_scale(qs, h, b) : 1.0f;
  float m = 0.0f;
  for (int64_t r = r0 + t / vecs_per_row; r < r1; r += kUnroll * row_step) {
    uint4 raw[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)  // all loads first: kUnroll 16-byte requests in flight
      if (r + u * row_step < r1)
        raw[u] = __ldg(reinterpret_cast<const uint4*>(X.x + ((int64_t)b * X.rows + r + u * row_step) * H * kHeadDim) +
                       vrow);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (r + u * row_step >= r1) break;
      const int64_t br = (int64_t)b * X.rows + r + u * row_step;
      const float w = gated ? gate_factor(qs, br, H, h) : 1.0f;
      float f[8];
      unpack8(raw[u], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(do_q ? qscale1(f[e], s, gated, w) : f[e]));
    }
  }
  // reduce over the 8 lanes of the (row, head) segment, then per head in smem
  const unsigned group = 0xFFu << (threadIdx.x & 24);
  m = fmaxf(m, __shfl_xor_sync(group, m, 1));
  m = fmaxf(m, __shfl_xor_sync(group, m, 2));
  m = fmaxf(m, __shfl_xor_sync(group, m, 4));
  if ((t & 7) == 0) atomicMax(&s_max[h], __float_as_uint(m));
  __syncthreads();
  if (t < H) atomicMax(&amax[((int64_t)tensor * X.B + b) * H + t], s_max[t]);
}

__global__ void scales_kernel(const uint32_t* __restrict__ amax, int n, float* __restrict__ scales) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    const float a = __uint_as_float(amax[i]);
    scales[i] = a > 0.0f ? __fdiv_rn(a, 448.0f) : 1.0f;
  }
}

// ----------------------------------------------------- row-major quantise
__global__ void quantize_rows_kernel(RowsDesc X, QScale qs, int64_t n_rows, const float* __restrict__ scale,
                                     uint8_t* __restrict__ dst, int64_t dst_rows, const int32_t* __restrict__ n_valid,
                                     int64_t pad_end, int64_t rows_per_cta, int chunks) {
  const bool do_q = qs.enabled;
  const bool gated = do_q && qs.gate != nullptr;
  const int H = X.H;
  const int t = threadIdx.x;
  const int vecs_per_row = 8 * H;
  const int vrow = t % vecs_per_row;
  const int h = vrow >> 3;
  const int j = vrow & 7;
  const int row_step = blockDim.x / vecs_per_row;
  const int b = blockIdx.x / chunks;
  const int64_t r0 = (blockIdx.x % chunks) * rows_per_cta;
  const int64_t r1 = min(n_rows, r0 + rows_per_cta);
  const float s = do_q ? head_scale(qs, h, b) : 1.0f;
  const Divider dv = make_divider(__ldg(scale + b * H + h));
  const int64_t pad0 = n_valid != nullptr ? (int64_t)__ldg(n_valid + b) : pad_end;  // padding rows [pad0, pad_end)
  uint8_t* dbase = dst + ((int64_t)b * H + h) * dst_rows * kHeadDim + j * 8;
  for (int64_t r = r0 + t / vecs_per_row; r < r1; r += kUnroll * row_step) {
    uint4 raw[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)  // all loads first: kUnroll 16-byte requests in flight
      if (r + u * row_step < r1)
        raw[u] = __ldcs(reinterpret_cast<const uint4*>(X.x + ((int64_t)b * X.rows + r + u * row_step) * H * kHeadDim) +
                        vrow);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t rr = r + u * row_step;
      if (rr >= r1) break;
      const float w = gated ? gate_factor(qs, (int64_t)b * X.rows + rr, H, h) : 1.0f;
      float f[8];
      unpack8(raw[u], f);
      if (do_q) {
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = qscale1(f[e], s, gated, w);
      }
      divide8(f, dv);
      uint2 codes;
      codes.x = e4m3x2(f[0], f[1]) | (e4m3x2(f[2], f[3]) << 16);
      codes.y = e4m3x2(f[4], f[5]) | (e4m3x2(f[6], f[7]) << 16);
      if (rr >= pad0 && rr < pad_end) codes = make_uint2(0u, 0u);
      *reinterpret_cast<uint2*>(dbase + rr * kHeadDim) = codes;
    }
  }
}

// --------------------------------------------------- transposed V quantise
// grid: (ld / 128, B*H), 256 threads.  Reads 128 keys x 64 of one head,
// writes 64 rows of 128 keys (one 128-byte line each) via a padded smem tile.
__global__ void __launch_bounds__(256) quantize_vt_kernel(RowsDesc V, int64_t n_ctx, const int32_t* __restrict__ n_valid,
                                                          const float* __restrict__ scale, uint8_t* __restrict__ dst,
                                                          int64_t ld) {
  __shared__ uint32_t tile[kHeadDim][33];  // [e][key/4], 132-byte rows: conflict-free
  const int H = V.H;
  const int64_t bh = blockIdx.y;
  const int b = static_cast<int>(bh / H), h = static_cast<int>(bh % H);
  const int64_t r0 = (int64_t)blockIdx.x * kKvTile;
  const Divider dv = make_divider(__ldg(scale + bh));
  const int64_t n_b = n_valid != nullptr ? (int64_t)__ldg(n_valid + b) : n_ctx;
  const int t = threadIdx.x;
  const int j = t & 7;  // elements 8j..8j+7
  uint8_t* tb = reinterpret_cast<uint8_t*>(&tile[0][0]);
  uint4 raws[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {  // all loads first: four 16-byte requests in flight
    const int64_t r = r0 + (t >> 3) + 32 * i;
    if (r < n_b)
      raws[i] = __ldcs(reinterpret_cast<const uint4*>(V.x + (((int64_t)b * V.rows + r) * H + h) * kHeadDim) + j);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rl = (t >> 3) + 32 * i;
    const int64_t r = r0 + rl;
    uint32_t lo = 0, hi = 0;
    if (r < n_b) {
      float f[8];
      unpack8(raws[i], f);
      divide8(f, dv);
      lo = e4m3x2(f[0], f[1]) | (e4m3x2(f[2], f[3]) << 16);
      hi = e4m3x2(f[4], f[5]) | (e4m3x2(f[6], f[7]) << 16);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      tb[(8 * j + e) * 132 + rl] = static_cast<uint8_t>(lo >> (8 * e));
      tb[(8 * j + 4 + e) * 132 + rl] = static_cast<uint8_t>(hi >> (8 * e));
    }
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int c = t + 256 * i;
    const int e = c >> 3, part = c & 7;
    uint4 w;
    w.x = tile[e][4 * part + 0];
    w.y = tile[e][4 * part + 1];
    w.z = tile[e][4 * part + 2];
    w.w = tile[e][4 * part + 3];
    *reinterpret_cast<uint4*>(dst + (bh * kHeadDim + e) * ld + r0 + 16 * part) = w;
  }
}

// One (b, h) and 128 keys per block: 16-byte row loads of V, a shared-memory
// transpose, 32-bit stores of 64 rows (one per head element) of 128 keys.
__global__ void __launch_bounds__(256) transpose_vt_f16_kernel(RowsDesc V, int64_t n_ctx,
                                                               const int32_t* __restrict__ n_valid,
                                                               __half* __restrict__ dst, int64_t ld) {
  __shared__ uint16_t tile[kHeadDim][kKvTile + 2];  // [e][key]; 65-word rows
  const int H = V.H;
  const int64_t bh = blockIdx.y;
  const int b = static_cast<int>(bh / H), h = static_cast<int>(bh % H);
  const int64_t r0 = (int64_t)blockIdx.x * kKvTile;
  const int64_t n_b = n_valid != nullptr ? (int64_t)__ldg(n_valid + b) : n_ctx;
  const int t = threadIdx.x;
  const int j = t & 7;  // elements 8j..8j+7
  uint4 raws[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t r = r0 + (t >> 3) + 32 * i;
    raws[i] = make_uint4(0u, 0u, 0u, 0u);
    if (r < n_b)
      raws[i] = __ldcs(reinterpret_cast<const uint4*>(V.x + (((int64_t)b * V.rows + r) * H + h) * kHeadDim) + j);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rl = (t >> 3) + 32 * i;
    const uint32_t w[4] = {raws[i].x, raws[i].y, raws[i].z, raws[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      tile[8 * j + 2 * e][rl] = static_cast<uint16_t>(w[e] & 0xFFFFu);
      tile[8 * j + 2 * e + 1][rl] = static_cast<uint16_t>(w[e] >> 16);
    }
  }
  __syncthreads();
  uint32_t* out = reinterpret_cast<uint32_t*>(dst + bh * kHeadDim * ld + r0);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int c = t + 256 * i;  // 64 rows x 64 words
    const int e = c >> 6, wd = c & 63;
    const uint32_t lo = tile[e][2 * wd], hi = tile[e][2 * wd + 1];
    out[(int64_t)e * (ld / 2) + wd] = lo | (hi << 16);
  }
}

__global__ void write_meta_kernel(MetaChunk c, int32_t* __restrict__ n_dst, float* __restrict__ lam_dst) {
  const int i = threadIdx.x;
  if (i < c.count) {
    n_dst[c.b0 + i] = c.n[i];
    lam_dst[c.b0 + i] = c.lam[i];
  }
}

}  // namespace

cudaError_t launch_transpose_vt_f16(RowsDesc v, int64_t n_ctx, const int32_t* n_valid, __half* dst, int64_t ld,
                                    cudaStream_t st) {
  dim3 grid(static_cast<unsigned>((n_ctx + kKvTile - 1) / kKvTile), static_cast<unsigned>(v.B * v.H));
  if (grid.x == 0) return cudaSuccess;
  transpose_vt_f16_kernel<<<grid, 256, 0, st>>>(v, n_ctx, n_valid, dst, ld);
  return cudaGetLastError();
}

cudaError_t launch_write_meta(const MetaChunk& c, int32_t* n_dst, float* lam_dst, cudaStream_t st) {
  write_meta_kernel<<<1, kMetaChunk, 0, st>>>(c, n_dst, lam_dst);
  return cudaGetLastError();
}

cudaError_t launch_qscale(const __half* q, __half* out, int32_t B, int64_t rows, int32_t H, QScale qs,
                          cudaStream_t st) {
  const int64_t n_vec = (int64_t)B * rows * H * (kHeadDim / 8);
  if (n_vec == 0) return cudaSuccess;
  const int64_t want = (n_vec + 256 * kUnroll - 1) / (256 * kUnroll);
  const int grid = static_cast<int>(want < (int64_t)num_sms() * 8 ? want : (int64_t)num_sms() * 8);
  qscale_kernel<<<grid, 256, 0, st>>>(q, out, n_vec, H, rows, qs);
  return cudaGetLastError();
}

cudaError_t launch_gate_factors(const __half* gate, int64_t n, __half* w, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int64_t want = (n + 255) / 256;
  const int grid = static_cast<int>(want < (int64_t)num_sms() * 8 ? want : (int64_t)num_sms() * 8);
  gate_factor_kernel<<<grid, 256, 0, st>>>(gate, n, w);
  return cudaGetLastError();
}

cudaError_t launch_context_amax(RowsDesc q, QScale qs, RowsDesc k, RowsDesc v, int64_t n_ctx,
                                const int32_t* n_valid, uint32_t* amax, cudaStream_t st) {
  const int threads = row_threads(q.H);
  const int rows_per_pass = threads / (8 * q.H);
  // about 8 CTAs per SM over the three tensors
  int64_t chunks = ((int64_t)num_sms() * 8 + 3 * q.B - 1) / (3 * q.B);
  int64_t rows_per_cta = (n_ctx + chunks - 1) / chunks;
  rows_per_cta = ((rows_per_cta + rows_per_pass - 1) / rows_per_pass) * rows_per_pass;
  chunks = (n_ctx + rows_per_cta - 1) / rows_per_cta;
  dim3 grid(static_cast<unsigned>(q.B * chunks), 3);
  context_amax_kernel<<<grid, threads, 0, st>>>(q, qs, k, v, n_ctx, n_valid, rows_per_cta, static_cast<int>(chunks),
                                                amax);
  return cudaGetLastError();
}

cudaError_t launch_scales_from_amax(const uint32_t* amax, int32_t BH, float* scales, cudaStream_t st) {
  const int n = 3 * BH;
  scales_kernel<<<(n + 127) / 128, 128, 0, st>>>(amax, n, scales);
  return cudaGetLastError();
}

cudaError_t launch_quantize_rows(RowsDesc x, QScale qs, int64_t n_rows, const float* scale, uint8_t* dst,
                                 int64_t dst_rows, const int32_t* n_valid, int64_t pad_end, cudaStream_t st) {
  if (n_rows == 0) return cudaSuccess;
  const int threads = row_threads(x.H);
  const int rows_per_pass = threads / (8 * x.H);
  int64_t chunks = ((int64_t)num_sms() * 8 + x.B - 1) / x.B;
  int64_t rows_per_cta = (n_rows + chunks - 1) / chunks;
  rows_per_cta = ((rows_per_cta + rows_per_pass - 1) / rows_per_pass) * rows_per_pass;
  chunks = (n_rows + rows_per_cta - 1) / rows_per_cta;
  quantize_rows_kernel<<<static_cast<unsigned>(x.B * chunks), threads, 0, st>>>(
      x, qs, n_rows, scale, dst, dst_rows, n_valid, pad_end, rows_per_cta, static_cast<int>(chunks));
  return cudaGetLastError();
}

cudaError_t launch_quantize_vt(RowsDesc v, int64_t n_ctx, const int32_t* n_valid, const float* scale, uint8_t* dst,
                               int64_t ld, cudaStream_t st) {
  dim3 grid(static_cast<unsigned>(ld / kKvTile), static_cast<unsigned>(v.B * v.H));
  quantize_vt_kernel<<<grid, 256, 0, st>>>(v, n_ctx, n_valid, scale, dst, ld);
  return cudaGetLastError();
}

}  // namespace sdm
