// attention_f16.cu -- normal-precision (fp16) ICL attention on the sm_100a
// tensor cores.
//
// "[FP8 3/4] Integrate FP8 attention and caching into TabICLv2" (opening
// section): FP8 attention is used only on intermediate ICL layers above 8,192
// unmasked context rows; the final attention and shorter contexts keep normal
// precision (the pages fall back to SDPA).  This kernel is that path:
// softmax(q' k^T / sqrt(64)) v with fp16 operands, fp32 logits and
// accumulation, fp16 probabilities fed to the P.V product, fp16 output.
//
// Same organisation as the FP8 kernel in attention.cu -- two 128-row query
// tiles per CTA, one TMA producer warp, one MMA-issuing thread, two softmax
// warpgroups -- with tcgen05.mma kind::f16 (K = 16 per instruction):
//   Q' and K tiles come straight from the [B][rows][H][64] fp16 layout with a
//   4-D TMA box {64, 1, 128, 1} (128-byte rows, 128-byte swizzle);
//   V^T (keys contiguous, from a transpose pass) is loaded as two 64-key
//   swizzle atoms per 128-key tile;
//   P (fp16, two keys per 32-bit column) has its own TMEM columns, so the next
//   S = Q K^T is issued as soon as the softmax holds S in registers;
//   the row sum l is accumulated by the softmax in registers.
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,320) O1 [320,384)
//                     P0 [384,448) P1 [448,512).
#include <math.h>

#include "kernels.cuh"
#include "ptx.cuh"
#include "softmax.cuh"

namespace sdm {
namespace {

constexpr int kStagesH = 4;
constexpr int kTilesH = 2;
constexpr int kSoftmaxWarpsH = 4 * kTilesH;
constexpr int kProducerWarpH = kSoftmaxWarpsH;
constexpr int kMmaWarpH = kSoftmaxWarpsH + 1;
constexpr int kThreadsH = 32 * (kSoftmaxWarpsH + 2);
constexpr uint32_t kTmemColsH = 512;

constexpr int kTileBytesH = 128 * kHeadDim * 2;      // 16 KB: 128 rows x 64 fp16
constexpr int kVHalfBytesH = kHeadDim * 64 * 2;      // 8 KB: 64 rows (d) x 64 keys fp16

__device__ __forceinline__ uint32_t hs_col(int t) { return 128u * t; }
__device__ __forceinline__ uint32_t ho_col(int t) { return 256u + 64u * t; }
__device__ __forceinline__ uint32_t hp_col(int t) { return 384u + 64u * t; }

constexpr long long kWaitLimitH = 1LL << 31;
constexpr long long kDrainLimitH = 1LL << 24;

struct __align__(1024) SmemH {
  uint8_t q[kTilesH][kTileBytesH];
  uint8_t k[kStagesH][kTileBytesH];
  uint8_t v[kStagesH][2][kVHalfBytesH];
  uint64_t q_full;
  uint64_t k_full[kStagesH];
  uint64_t v_full[kStagesH];
  uint64_t kv_empty[kStagesH];
  uint64_t s_full[kTilesH];
  uint64_t s_free[kTilesH];
  uint64_t p_full[kTilesH];
  uint64_t o_ready[kTilesH];
  uint64_t drain;
  uint32_t tmem_base;
  uint32_t abort_flag;
};

struct HParams {
  int32_t B, H;
  int64_t T, N;
  int64_t n_pairs;
  __half* out;      // [B][T][H][64]
  uint32_t* err;
  const int32_t* n_keys;  // [B] keys per batch (rows [n_b, N) are padding), or nullptr: N
};

__device__ __forceinline__ void raise_abort_h(SmemH& s, uint32_t* err, uint32_t code) {
  atomicOr(err, code);
  *reinterpret_cast<volatile uint32_t*>(&s.abort_flag) = 1u;
}

__device__ __forceinline__ void drain_wait_h(uint64_t* bar, uint32_t parity, uint32_t* err) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kDrainLimitH) {
      atomicOr(err, kErrTimeoutDrain);
      return;
    }
  }
}

// Two logits -> one 32-bit column of two fp16 probabilities; adds them to l.
template <bool kPoly>
__device__ __forceinline__ uint32_t p_pair_f16(uint32_t z0, uint32_t z1, float c2, float nm2, float& l0, float& l1) {
  float t0, t1, p0, p1;
  fma2(t0, t1, __uint_as_float(z0), __uint_as_float(z1), c2, c2, nm2, nm2);
  if (kPoly) {
    // clamp far below fp16's smallest subnormal: the row sum l adds the
    // unrounded p, so a clamp value must not bias it
    exp2_fma2<-125>(t0, t1, p0, p1);
  } else {
    p0 = ex2_approx(t0);
    p1 = ex2_approx(t1);
  }
  add2(l0, l1, l0, l1, p0, p1);
  return f16x2(p0, p1);
}

// One 32-key chunk of S -> 16 P columns (keys 4W..4W+3 -> columns 2W, 2W + 1
// of pc, counted from `col0`); a and b accumulate the chunk's row sum.
template <int W>
__device__ __forceinline__ void p_chunk_f16(const uint32_t (&r)[32], uint32_t (&pc)[32], int col0, float c2,
                                            float nm2, float& a, float& b) {
  if constexpr (W < 8) {
    pc[col0 + 2 * W] = p_pair_f16<poly_word(W)>(r[4 * W], r[4 * W + 1], c2, nm2, a, b);
    pc[col0 + 2 * W + 1] = p_pair_f16<poly_word(W)>(r[4 * W + 2], r[4 * W + 3], c2, nm2, a, b);
    p_chunk_f16<W + 1>(r, pc, col0, c2, nm2, a, b);
  }
}

__global__ void __launch_bounds__(kThreadsH, 1)
    icl_attention_f16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const HParams p) {
  extern __shared__ uint8_t smem_raw[];
  SmemH& s = *reinterpret_cast<SmemH*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const volatile uint32_t* abort_flag = &s.abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int64_t blk = blockIdx.x;
  const int64_t pair = blk % p.n_pairs;
  const int64_t bh = blk / p.n_pairs;
  const int32_t b = static_cast<int32_t>(bh / p.H), h = static_cast<int32_t>(bh % p.H);
  const int64_t row0 = pair * (kTilesH * kQTile);
  const int64_t n_b = p.n_keys != nullptr ? (int64_t)__ldg(p.n_keys + b) : p.N;  // this batch's keys
  // a CTA whose rows are all padding context rows only writes zeros
  const bool all_pad = row0 >= n_b && row0 + kTilesH * kQTile <= p.N;
  const int n_tiles = all_pad ? 0 : static_cast<int>((n_b + kKvTile - 1) / kKvTile);

  if (threadIdx.x == 0) {
    mbar_init(&s.q_full, 1);
    for (int i = 0; i < kStagesH; ++i) {
      mbar_init(&s.k_full[i], 1);
      mbar_init(&s.v_full[i], 1);
      mbar_init(&s.kv_empty[i], 1);
    }
    for (int t = 0; t < kTilesH; ++t) {
      mbar_init(&s.s_full[t], 1);
      mbar_init(&s.s_free[t], 4);
      mbar_init(&s.p_full[t], 4);
      mbar_init(&s.o_ready[t], 1);
    }
    mbar_init(&s.drain, 1);
    s.abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == kMmaWarpH) {
    tmem_alloc(&s.tmem_base, kTmemColsH);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == kProducerWarpH) {
    // ================================================================ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(&s.q_full, kTilesH * kTileBytesH);
      for (int t = 0; t < kTilesH; ++t)
        tma_load_4d(s.q[t], &tm_q, &s.q_full, 0, h, static_cast<int32_t>(row0 + t * kQTile), b);
      int issued = 0;
      for (int it = 0; it < n_tiles; ++it) {
        const int st = it % kStagesH;
        const uint32_t ph = (it / kStagesH) & 1;
        if (!mbar_wait(&s.kv_empty[st], ph ^ 1u, abort_flag, kWaitLimitH)) {
          raise_abort_h(s, p.err, kErrTimeoutEmpty);
          break;
        }
        const int32_t key0 = it * kKvTile;
        mbar_arrive_expect_tx(&s.k_full[st], kTileBytesH);
        tma_load_4d(s.k[st], &tm_k, &s.k_full[st], 0, h, key0, b);
        mbar_arrive_expect_tx(&s.v_full[st], 2 * kVHalfBytesH);
        tma_load_3d(s.v[st][0], &tm_v, &s.v_full[st], key0, 0, static_cast<int32_t>(bh));
        tma_load_3d(s.v[st][1], &tm_v, &s.v_full[st], key0 + 64, 0, static_cast<int32_t>(bh));
        issued = it + 1;
      }
      drain_wait_h(&s.q_full, 0, p.err);
      for (int it = issued > kStagesH ? issued - kStagesH : 0; it < issued; ++it) {
        drain_wait_h(&s.k_full[it % kStagesH], (it / kStagesH) & 1, p.err);
        drain_wait_h(&s.v_full[it % kStagesH], (it / kStagesH) & 1, p.err);
      }
    }
  } else if (warp == kMmaWarpH) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_f16_f32(kQTile, kKvTile);
      const uint32_t idesc_o = idesc_f16_f32(kQTile, kHeadDim);
      auto issue_qk = [&](int t, int st) {
        const uint32_t a0 = smem_u32(s.q[t]), b0 = smem_u32(s.k[st]);
#pragma unroll
        for (int ks = 0; ks < kHeadDim / 16; ++ks)  // 16 fp16 = 32 bytes per step
          mma_f16_ss(tmem + hs_col(t), smem_desc_kmajor(a0 + 32 * ks, 1024, kSwizzle128B),
                     smem_desc_kmajor(b0 + 32 * ks, 1024, kSwizzle128B), idesc_s, ks > 0);
      };
      auto issue_pv = [&](int t, int st, bool acc) {
#pragma unroll
        for (int ks = 0; ks < kKvTile / 16; ++ks) {  // 8 steps of 16 keys; 4 per 64-key atom
          const uint32_t b0 = smem_u32(s.v[st][ks >> 2]) + 32 * (ks & 3);
          mma_f16_ts(tmem + ho_col(t), tmem + hp_col(t) + 8 * ks, smem_desc_kmajor(b0, 1024, kSwizzle128B), idesc_o,
                     (acc || ks > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(&s.q_full, 0, abort_flag, kWaitLimitH);
      if (!ok) raise_abort_h(s, p.err, kErrTimeoutQ);
      if (ok && n_tiles > 0) {
        ok = mbar_wait(&s.k_full[0], 0, abort_flag, kWaitLimitH);
        if (!ok) raise_abort_h(s, p.err, kErrTimeoutKV);
      }
      if (ok && n_tiles > 0) {
        tc_fence_after();
        for (int t = 0; t < kTilesH; ++t) {
          issue_qk(t, 0);
          mma_commit(&s.s_full[t]);
        }
      }
      for (int it = 0; ok && it < n_tiles; ++it) {
        const int st = it % kStagesH;
        const uint32_t ph = (it / kStagesH) & 1;
        const int nst = (it + 1) % kStagesH;
        const uint32_t nph = ((it + 1) / kStagesH) & 1;
        const bool more = it + 1 < n_tiles;
        if (more && !mbar_wait(&s.k_full[nst], nph, abort_flag, kWaitLimitH)) {
          raise_abort_h(s, p.err, kErrTimeoutKV);
          break;
        }
        if (!mbar_wait(&s.v_full[st], ph, abort_flag, kWaitLimitH)) {
          raise_abort_h(s, p.err, kErrTimeoutKV);
          break;
        }
#pragma unroll
        for (int t = 0; t < kTilesH; ++t) {
          if (more) {
            if (!mbar_wait(&s.s_free[t], it & 1, abort_flag, kWaitLimitH)) {
              raise_abort_h(s, p.err, kErrTimeoutS);
              ok = false;
              break;
            }
            tc_fence_after();
            issue_qk(t, nst);
            mma_commit(&s.s_full[t]);
          }
          if (!mbar_wait(&s.p_full[t], it & 1, abort_flag, kWaitLimitH)) {
            raise_abort_h(s, p.err, kErrTimeoutP);
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(t, st, it > 0);
          mma_commit(&s.o_ready[t]);
        }
        if (ok) mma_commit(&s.kv_empty[st]);
      }
      mma_commit(&s.drain);
      drain_wait_h(&s.drain, 0, p.err);
    }
  } else {
    // ================================================================ softmax
    const int t = warp >> 2;
    const int wq = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(32 * wq) << 16;
    const uint32_t t_s = tmem + lane_base + hs_col(t);
    const uint32_t t_p = tmem + lane_base + hp_col(t);
    const uint32_t t_o = tmem + lane_base + ho_col(t);
    const float c2 = 0.18033688011112042f;  // log2(e) / sqrt(64)
    float m_run = -INFINITY, m2 = -INFINITY;
    float l[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};  // row sum: 8 partial sums
    bool ok = true;
    for (int it = 0; it < n_tiles; ++it) {
      ok = mbar_wait(&s.s_full[t], it & 1, abort_flag, kWaitLimitH);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) raise_abort_h(s, p.err, kErrTimeoutS);
        break;
      }
      tc_fence_after();
      const int64_t nvalid = n_b - (int64_t)it * kKvTile;
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(t_s + 32 * c, r[c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.s_free[t]);
      if (nvalid < kKvTile) {
        mask_keys(r[0], r[1], 0, nvalid);
        mask_keys(r[2], r[3], 64, nvalid);
      }
      float mx0 = m_run, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        mx0 = max3(mx0, __uint_as_float(r[0][i]), __uint_as_float(r[1][i]));
        mx1 = max3(mx1, __uint_as_float(r[2][i]), __uint_as_float(r[3][i]));
        mx2 = max3(mx2, __uint_as_float(r[0][i + 1]), __uint_as_float(r[1][i + 1]));
        mx3 = max3(mx3, __uint_as_float(r[2][i + 1]), __uint_as_float(r[3][i + 1]));
      }
      const float mt = max3(mx0, mx1, fmaxf(mx2, mx3));
      const bool up = mt > m_run;
      const float m2_new = up ? __fmul_rn(mt, c2) : m2;
      float alpha = 1.0f;
      if (up && it > 0) alpha = ex2_approx(__fsub_rn(m2, m2_new));
#pragma unroll
      for (int i = 0; i < 8; ++i) l[i] = __fmul_rn(l[i], alpha);
      {
        // chunks 0, 1 -> P columns [0, 32); the previous P.V must have read
        // its P before the first store; then chunks 2, 3 -> [32, 64)
        uint32_t pa[32];
        p_chunk_f16<0>(r[0], pa, 0, c2, -m2_new, l[0], l[1]);
        p_chunk_f16<0>(r[1], pa, 16, c2, -m2_new, l[2], l[3]);
        if (it > 0) {
          ok = mbar_wait(&s.o_ready[t], (it - 1) & 1, abort_flag, kWaitLimitH);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) {
            if (lane == 0) raise_abort_h(s, p.err, kErrTimeoutO);
            break;
          }
          tc_fence_after();
        }
        tmem_st_32x32b_x32(t_p, pa);
        p_chunk_f16<0>(r[2], pa, 0, c2, -m2_new, l[4], l[5]);
        p_chunk_f16<0>(r[3], pa, 16, c2, -m2_new, l[6], l[7]);
        tmem_st_32x32b_x32(t_p + 32, pa);
      }
      if (it > 0 && __any_sync(0xffffffffu, up)) {
        // both halves of O in one TMEM round trip, packed multiplies
        uint32_t o0[32], o1[32];
        tmem_ld_32x32b_x32(t_o, o0);
        tmem_ld_32x32b_x32(t_o + 32, o1);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float a0, a1, b0, b1;
          mul2(a0, a1, __uint_as_float(o0[i]), __uint_as_float(o0[i + 1]), alpha, alpha);
          mul2(b0, b1, __uint_as_float(o1[i]), __uint_as_float(o1[i + 1]), alpha, alpha);
          o0[i] = __float_as_uint(a0);
          o0[i + 1] = __float_as_uint(a1);
          o1[i] = __float_as_uint(b0);
          o1[i + 1] = __float_as_uint(b1);
        }
        tmem_st_32x32b_x32(t_o, o0);
        tmem_st_32x32b_x32(t_o + 32, o1);
      }
      m_run = mt;
      m2 = m2_new;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.p_full[t]);
    }
    if (ok && n_tiles > 0) {
      ok = mbar_wait(&s.o_ready[t], (n_tiles - 1) & 1, abort_flag, kWaitLimitH);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok && lane == 0) raise_abort_h(s, p.err, kErrTimeoutO);
    }
    if (ok) {
      uint32_t o0[32], o1[32];
      if (n_tiles > 0) {
        tc_fence_after();
        tmem_ld_32x32b_x32(t_o, o0);
        tmem_ld_32x32b_x32(t_o + 32, o1);
        tmem_ld_wait();
      }
      const int64_t row = row0 + (int64_t)t * kQTile + 32 * wq + lane;
      if (row < p.T) {
        const bool zero = n_tiles == 0 || (row >= n_b && row < p.N);  // padding context row
        const float lf = ((l[0] + l[1]) + (l[2] + l[3])) + ((l[4] + l[5]) + (l[6] + l[7]));
        uint4* dst = reinterpret_cast<uint4*>(p.out + (((int64_t)b * p.T + row) * p.H + h) * kHeadDim);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          uint32_t w[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int e = 8 * v + 2 * k;
            const float x0 = __uint_as_float(e < 32 ? o0[e] : o1[e - 32]);
            const float x1 = __uint_as_float(e + 1 < 32 ? o0[e + 1] : o1[e + 1 - 32]);
            w[k] = zero ? 0u : f16x2(__fdiv_rn(x0, lf), __fdiv_rn(x1, lf));
          }
          dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarpH) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemColsH);
  }
}

// fp16 tensor map of rank `rank` (dims innermost first, strides in bytes for dims 1..rank-1).
bool make_map_f16(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
                  const cuuint32_t* box) {
  const TensorMapEncodeFn fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, rank, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_attention_f16(const __half* q_scaled, const __half* k, const __half* vt, int32_t B, int64_t T,
                                 int64_t N, int32_t H, int64_t ld_v, const int32_t* n_keys, __half* out,
                                 uint32_t* err, cudaStream_t st) {
  // Q' [B][T][H][64] and K [B][N][H][64]: 4-D {64, H, rows, B}, box {64, 1, 128, 1}
  const cuuint64_t dq[4] = {64, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t sq[3] = {128, (cuuint64_t)H * 128, (cuuint64_t)T * H * 128};
  const cuuint64_t dk[4] = {64, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  const cuuint64_t sk[3] = {128, (cuuint64_t)H * 128, (cuuint64_t)N * H * 128};
  const cuuint32_t box4[4] = {64, 1, 128, 1};
  // V^T [B*H][64][ld_v]: 3-D {ld_v, 64, B*H}, box {64 keys, 64 rows, 1}; the
  // keys in [N, ld_v) that the last tile reads are zeros from the transpose
  const cuuint64_t dv[3] = {(cuuint64_t)ld_v, 64, (cuuint64_t)B * H};
  const cuuint64_t sv[2] = {(cuuint64_t)ld_v * 2, (cuuint64_t)ld_v * 2 * 64};
  const cuuint32_t box3[3] = {64, 64, 1};
  CUtensorMap tq, tk, tv;
  if (!make_map_f16(&tq, q_scaled, 4, dq, sq, box4) || !make_map_f16(&tk, k, 4, dk, sk, box4) ||
      !make_map_f16(&tv, vt, 3, dv, sv, box3))
    return cudaErrorInvalidValue;
  HParams p;
  p.B = B;
  p.H = H;
  p.T = T;
  p.N = N;
  p.n_pairs = (T + kTilesH * kQTile - 1) / (kTilesH * kQTile);
  p.out = out;
  p.err = err;
  p.n_keys = n_keys;
  const size_t smem = sizeof(SmemH) + 1024;
  cudaError_t e = cudaFuncSetAttribute(icl_attention_f16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t grid = p.n_pairs * (int64_t)B * H;
  if (grid == 0) return cudaSuccess;
  icl_attention_f16_kernel<<<static_cast<unsigned>(grid), kThreadsH, smem, st>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace sdm
