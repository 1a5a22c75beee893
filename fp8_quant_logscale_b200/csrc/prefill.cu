// prefill.cu -- ragged grouped-query prefill attention, bf16, head dim 128, on
// the sm_100a tensor cores.
//
// "Pipeline long ragged GQA4 KV loads" (oxide-infer PR #114, walkthrough and
// performance contract): a packed batch of sequences, each with q_len query
// tokens that are the last q_len of its kv_len key/value tokens; G = Hq / Hkv
// query heads share one key/value head.  out = softmax(q k^T / sqrt(128)) v
// per query head, causal (query i sees keys j <= kv_len - q_len + i) or not.
//
// One CTA = one sequence, one key/value head, and a 128-row tile packed
// token-major from 128/G query tokens x the G query heads of that group, so
// the G heads share every K and V tile (one 3-D TMA box loads the rows).  The
// organisation follows the fp16 attention kernel -- TMA producer warp with
// separate K and V barriers per stage (the page's idea: S = Q K^T starts
// before V lands), one MMA-issuing thread, four softmax warps (one row each
// thread), P in its own TMEM columns so the next Q K^T overlaps the softmax --
// with tcgen05.mma kind::f16 on bf16: K is the K-major B operand of Q K^T, V
// the MN-major B operand of P V read in its natural [key][d] layout.
// TMEM: S [0,128), O [128,256), P [256,320) (bf16, two keys per column).
#include <cuda_bf16.h>
#include <math.h>

#include "kernels.cuh"
#include "ptx.cuh"
#include "softmax.cuh"

namespace sdm {
namespace {

constexpr int kDP = 128;          // head dim
constexpr int kStagesP = 3;
constexpr int kThreadsP = 192;    // 4 softmax warps, producer warp, MMA warp
constexpr int kProducerWarpP = 4;
constexpr int kMmaWarpP = 5;
constexpr int kHalfBytesP = 128 * 64 * 2;  // 128 rows x 64 bf16: one 128-byte-swizzled half of a tile
constexpr uint32_t kSColP = 0, kOColP = 128, kPColP = 256;

constexpr long long kWaitLimitP = 1LL << 31;
constexpr long long kDrainLimitP = 1LL << 24;

struct __align__(1024) SmemP {
  uint8_t q[2][kHalfBytesP];             // Q tile, head-dim halves
  uint8_t k[kStagesP][2][kHalfBytesP];   // [key][64] per half
  uint8_t v[kStagesP][2][kHalfBytesP];   // [key][64] per half (MN-major B of P V)
  uint64_t q_full;
  uint64_t k_full[kStagesP];
  uint64_t v_full[kStagesP];
  uint64_t kv_empty[kStagesP];
  uint64_t s_full, s_free, p_full, o_ready, drain;
  uint32_t tmem_base;
  uint32_t abort_flag;
  uint32_t last;  // this CTA is the last of its query tile's key chunks to finish
};

constexpr int kClusterP = 4;  // CTAs per query tile, each with a quarter of its keys
constexpr int kStashLd = kDP + 4;  // floats per row of the shared-memory partials (padded)
static_assert(kClusterP * 32 * kStashLd * 4 <= kStagesP * 2 * kHalfBytesP, "partials fit in the K stages");

struct PrefillParams {
  int32_t n_seqs, q_heads, kv_heads, group, tokens_per_tile, causal;
  int32_t q_off[kPrefillMaxSeqs], q_len[kPrefillMaxSeqs], kv_off[kPrefillMaxSeqs], kv_len[kPrefillMaxSeqs];
  int32_t tile_start[kPrefillMaxSeqs + 1];  // prefix sum of query tiles over the sequences
  float c2;                                 // log2(e) / sqrt(128)
  __nv_bfloat16* out;                       // [total_q][Hq][128]
  uint32_t* err;
};

__device__ __forceinline__ void raise_abort_p(SmemP& s, uint32_t* err, uint32_t code) {
  atomicOr(err, code);
  *reinterpret_cast<volatile uint32_t*>(&s.abort_flag) = 1u;
}

__device__ __forceinline__ void drain_wait_p(uint64_t* bar, uint32_t parity, uint32_t* err) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kDrainLimitP) {
      atomicOr(err, kErrTimeoutDrain);
      return;
    }
  }
}

// Keys past a row's last visible key (key0 + c > lim) get logit -inf.
__device__ __forceinline__ void mask_after(uint32_t (&r)[32], int key0, int lim) {
#pragma unroll
  for (int c = 0; c < 32; ++c)
    if (key0 + c > lim) r[c] = __float_as_uint(-INFINITY);
}

// Two logits -> one 32-bit TMEM column of two bf16 probabilities, added to l.
template <bool kPoly>
__device__ __forceinline__ uint32_t p_pair_bf16(uint32_t z0, uint32_t z1, float c2, float nm2, float& l0, float& l1) {
  float t0, t1, p0, p1;
  fma2(t0, t1, __uint_as_float(z0), __uint_as_float(z1), c2, c2, nm2, nm2);
  if (kPoly) {
    exp2_fma2<-125>(t0, t1, p0, p1);
  } else {
    p0 = ex2_approx(t0);
    p1 = ex2_approx(t1);
  }
  add2(l0, l1, l0, l1, p0, p1);
  return bf16x2(p0, p1);
}

// One 32-key chunk -> 16 P columns starting at col0 of pc.
template <int W>
__device__ __forceinline__ void p_chunk_bf16(const uint32_t (&r)[32], uint32_t (&pc)[32], int col0, float c2,
                                             float nm2, float& a, float& b) {
  if constexpr (W < 8) {
    pc[col0 + 2 * W] = p_pair_bf16<poly_word(W)>(r[4 * W], r[4 * W + 1], c2, nm2, a, b);
    pc[col0 + 2 * W + 1] = p_pair_bf16<poly_word(W)>(r[4 * W + 2], r[4 * W + 3], c2, nm2, a, b);
    p_chunk_bf16<W + 1>(r, pc, col0, c2, nm2, a, b);
  }
}

__global__ void __cluster_dims__(kClusterP, 1, 1) __launch_bounds__(kThreadsP, 1)
    gqa_prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  SmemP& s = *reinterpret_cast<SmemP*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const volatile uint32_t* abort_flag = &s.abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- which sequence, key/value head and query tile; this CTA's share of the keys
  const int rank = static_cast<int>(cluster_ctarank());       // 0..3 within the cluster
  const int tile = static_cast<int>(blockIdx.x) / kClusterP;  // query tile over all sequences
  int b = 0;
  while (b + 1 < p.n_seqs && p.tile_start[b + 1] <= tile) ++b;
  const int kvh = blockIdx.y;
  const int G = p.group, tpt = p.tokens_per_tile;
  const int q_len = p.q_len[b], kv_len = p.kv_len[b];
  const int tok0 = (tile - p.tile_start[b]) * tpt;
  const int tok_end = tok0 + tpt < q_len ? tok0 + tpt : q_len;
  const int n_keys = p.causal ? kv_len - q_len + tok_end : kv_len;  // keys any row of the tile sees
  // the cluster's CTAs take consecutive runs of whole 128-key tiles
  const int per = ((n_keys + kKvTile - 1) / kKvTile + kClusterP - 1) / kClusterP * kKvTile;
  const int kv_lo = rank * per < n_keys ? rank * per : n_keys;
  const int kv_hi = kv_lo + per < n_keys ? kv_lo + per : n_keys;
  const int n_tiles = (kv_hi - kv_lo + kKvTile - 1) / kKvTile;

  if (threadIdx.x == 0) {
    mbar_init(&s.q_full, 1);
    for (int i = 0; i < kStagesP; ++i) {
      mbar_init(&s.k_full[i], 1);
      mbar_init(&s.v_full[i], 1);
      mbar_init(&s.kv_empty[i], 1);
    }
    mbar_init(&s.s_full, 1);
    mbar_init(&s.s_free, 4);
    mbar_init(&s.p_full, 4);
    mbar_init(&s.o_ready, 1);
    mbar_init(&s.drain, 1);
    s.abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == kMmaWarpP) {
    tmem_alloc(&s.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  // what the softmax hands to the cluster's combine (one row per softmax thread)
  bool have_share = false;  // this CTA's keys were attended (and no wait gave up)
  float share_m2 = -INFINITY, share_l = 0.0f;

  if (warp == kProducerWarpP) {
    // ================================================================ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      // Q rows: tpt tokens x G heads (box {64, G, tpt}), both head-dim halves
      mbar_arrive_expect_tx(&s.q_full, 2 * kHalfBytesP);
      for (int hf = 0; hf < 2; ++hf)
        tma_load_3d(s.q[hf], &tm_q, &s.q_full, 64 * hf, kvh * G, p.q_off[b] + tok0);
      int issued = 0;
      for (int it = 0; it < n_tiles; ++it) {
        const int st = it % kStagesP;
        const uint32_t ph = (it / kStagesP) & 1;
        if (!mbar_wait(&s.kv_empty[st], ph ^ 1u, abort_flag, kWaitLimitP)) {
          raise_abort_p(s, p.err, kErrTimeoutEmpty);
          break;
        }
        const int key0 = p.kv_off[b] + kv_lo + it * kKvTile;
        mbar_arrive_expect_tx(&s.k_full[st], 2 * kHalfBytesP);
        for (int hf = 0; hf < 2; ++hf) tma_load_3d(s.k[st][hf], &tm_k, &s.k_full[st], 64 * hf, kvh, key0);
        mbar_arrive_expect_tx(&s.v_full[st], 2 * kHalfBytesP);
        for (int hf = 0; hf < 2; ++hf) tma_load_3d(s.v[st][hf], &tm_v, &s.v_full[st], 64 * hf, kvh, key0);
        issued = it + 1;
      }
      drain_wait_p(&s.q_full, 0, p.err);
      for (int it = issued > kStagesP ? issued - kStagesP : 0; it < issued; ++it) {
        drain_wait_p(&s.k_full[it % kStagesP], (it / kStagesP) & 1, p.err);
        drain_wait_p(&s.v_full[it % kStagesP], (it / kStagesP) & 1, p.err);
      }
    }
  } else if (warp == kMmaWarpP) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, kKvTile, false);
      const uint32_t idesc_o = idesc_bf16_f32(128, kDP, true);
      auto issue_qk = [&](int st) {
#pragma unroll
        for (int ks = 0; ks < kDP / 16; ++ks) {  // 16 bf16 (32 bytes) of the head dim per step
          const uint32_t a = smem_u32(s.q[ks >> 2]) + 32 * (ks & 3);
          const uint32_t bk = smem_u32(s.k[st][ks >> 2]) + 32 * (ks & 3);
          mma_f16_ss(tmem + kSColP, smem_desc_kmajor(a, 1024, kSwizzle128B), smem_desc_kmajor(bk, 1024, kSwizzle128B),
                     idesc_s, ks > 0);
        }
      };
      auto issue_pv = [&](int st, bool acc) {
#pragma unroll
        for (int ks = 0; ks < kKvTile / 16; ++ks) {  // 16 keys per step: 8 P columns, 2 KB of each V half
          const uint32_t bv = smem_u32(s.v[st][0]) + 2048 * ks;
          mma_f16_ts(tmem + kOColP, tmem + kPColP + 8 * ks, smem_desc_mnmajor_sw128(bv, kHalfBytesP, 1024), idesc_o,
                     (acc || ks > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(&s.q_full, 0, abort_flag, kWaitLimitP);
      if (!ok) raise_abort_p(s, p.err, kErrTimeoutQ);
      if (ok && n_tiles > 0) {
        ok = mbar_wait(&s.k_full[0], 0, abort_flag, kWaitLimitP);
        if (!ok) raise_abort_p(s, p.err, kErrTimeoutKV);
      }
      if (ok && n_tiles > 0) {
        tc_fence_after();
        issue_qk(0);
        mma_commit(&s.s_full);
      }
      for (int it = 0; ok && it < n_tiles; ++it) {
        const int st = it % kStagesP;
        const uint32_t ph = (it / kStagesP) & 1;
        const int nst = (it + 1) % kStagesP;
        const uint32_t nph = ((it + 1) / kStagesP) & 1;
        if (it + 1 < n_tiles) {
          if (!mbar_wait(&s.k_full[nst], nph, abort_flag, kWaitLimitP)) {
            raise_abort_p(s, p.err, kErrTimeoutKV);
            break;
          }
          if (!mbar_wait(&s.s_free, it & 1, abort_flag, kWaitLimitP)) {
            raise_abort_p(s, p.err, kErrTimeoutS);
            break;
          }
          tc_fence_after();
          issue_qk(nst);
          mma_commit(&s.s_full);
        }
        if (!mbar_wait(&s.v_full[st], ph, abort_flag, kWaitLimitP)) {
          raise_abort_p(s, p.err, kErrTimeoutKV);
          break;
        }
        if (!mbar_wait(&s.p_full, it & 1, abort_flag, kWaitLimitP)) {
          raise_abort_p(s, p.err, kErrTimeoutP);
          break;
        }
        tc_fence_after();
        issue_pv(st, it > 0);
        mma_commit(&s.o_ready);
        mma_commit(&s.kv_empty[st]);
      }
      mma_commit(&s.drain);
      drain_wait_p(&s.drain, 0, p.err);
    }
  } else {
    // ================================================================ softmax
    const int wq = warp;  // TMEM lane quadrant = rows 32wq..32wq+31
    const uint32_t lane_base = static_cast<uint32_t>(32 * wq) << 16;
    const uint32_t t_s = tmem + lane_base + kSColP;
    const uint32_t t_p = tmem + lane_base + kPColP;
    const uint32_t t_o = tmem + lane_base + kOColP;
    const int r = 32 * wq + lane;             // row: token tok0 + r / G, query head kvh * G + r % G
    const int tok = tok0 + r / G;
    const bool valid = tok < q_len;
    // last key this row sees (rows of tokens past the sequence use the last one: never stored)
    const int lim = p.causal ? kv_len - q_len + (valid ? tok : q_len - 1) : kv_len - 1;
    const float c2 = p.c2;
    float m_run = -INFINITY, m2 = -INFINITY;
    float l[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
    bool ok = true;
    for (int it = 0; it < n_tiles; ++it) {
      ok = mbar_wait(&s.s_full, it & 1, abort_flag, kWaitLimitP);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) raise_abort_p(s, p.err, kErrTimeoutS);
        break;
      }
      tc_fence_after();
      uint32_t rr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(t_s + 32 * c, rr[c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.s_free);
      const int key0 = kv_lo + it * kKvTile;
      if (key0 + kKvTile - 1 > lim) {  // the tile reaches past this row's last key
#pragma unroll
        for (int c = 0; c < 4; ++c) mask_after(rr[c], key0 + 32 * c, lim);
      }
      float mx[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        mx[j] = max3(j == 0 ? m_run : -INFINITY, __uint_as_float(rr[j >> 1][16 * (j & 1)]),
                     __uint_as_float(rr[j >> 1][16 * (j & 1) + 1]));
#pragma unroll
      for (int i = 2; i < 16; i += 2) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          mx[j] = max3(mx[j], __uint_as_float(rr[j >> 1][16 * (j & 1) + i]),
                       __uint_as_float(rr[j >> 1][16 * (j & 1) + i + 1]));
      }
      const float mt = max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
      const bool up = mt > m_run;
      const float m2_new = up ? __fmul_rn(mt, c2) : m2;
      // a row that has seen no key of its chunk yet (all -inf) keeps m2 = -inf:
      // shift by 0 instead, so its probabilities come out 0 rather than NaN
      const float nm2 = m2_new == -INFINITY ? 0.0f : -m2_new;
      float alpha = 1.0f;
      if (up && it > 0) alpha = ex2_approx(__fsub_rn(m2, m2_new));
#pragma unroll
      for (int i = 0; i < 8; ++i) l[i] = __fmul_rn(l[i], alpha);
      {
        uint32_t pa[32];
        p_chunk_bf16<0>(rr[0], pa, 0, c2, nm2, l[0], l[1]);
        p_chunk_bf16<0>(rr[1], pa, 16, c2, nm2, l[2], l[3]);
        if (it > 0) {  // the previous P V must have read P before it is overwritten
          ok = mbar_wait(&s.o_ready, (it - 1) & 1, abort_flag, kWaitLimitP);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) {
            if (lane == 0) raise_abort_p(s, p.err, kErrTimeoutO);
            break;
          }
          tc_fence_after();
        }
        tmem_st_32x32b_x32(t_p, pa);
        p_chunk_bf16<0>(rr[2], pa, 0, c2, nm2, l[4], l[5]);
        p_chunk_bf16<0>(rr[3], pa, 16, c2, nm2, l[6], l[7]);
        tmem_st_32x32b_x32(t_p + 32, pa);
      }
      if (it > 0 && __any_sync(0xffffffffu, up)) {
        uint32_t o[32];
#pragma unroll
        for (int c = 0; c < kDP / 32; ++c) {
          tmem_ld_32x32b_x32(t_o + 32 * c, o);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__fmul_rn(__uint_as_float(o[i]), alpha));
          tmem_st_32x32b_x32(t_o + 32 * c, o);
        }
      }
      m_run = mt;
      m2 = m2_new;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.p_full);
    }
    if (ok && n_tiles > 0) {
      ok = mbar_wait(&s.o_ready, (n_tiles - 1) & 1, abort_flag, kWaitLimitP);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok && lane == 0) raise_abort_p(s, p.err, kErrTimeoutO);
    }
    if (ok && n_tiles > 0) {
      have_share = true;
      share_m2 = m2;
      share_l = ((l[0] + l[1]) + (l[2] + l[3])) + ((l[4] + l[5]) + (l[6] + l[7]));
    }
  }

  // ---- every CTA of the cluster is done with its keys (its K stages are free):
  // the unnormalised O, m2 and l of row r go straight into the shared memory of
  // the cluster CTA that finishes row r (rank r / 32), into the slot of this
  // CTA's rank -- remote stores, no round trip -- so that after the next barrier
  // every combine reads local memory.  Slots live in the K stages; rows padded
  // to 132 floats so that a warp's 32 rows fall in different banks.
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp < 4) {
    tc_fence_after();
    const int r = 32 * warp + lane;
    const uint32_t owner = static_cast<uint32_t>(r >> 5);
    const uint32_t o_dst =
        mapa_shared(smem_u32(&s.k[0][0][0]) + 4u * ((rank * 32 + (r & 31)) * kStashLd), owner);
    const uint32_t ml_dst = mapa_shared(smem_u32(&s.v[0][0][0]) + 8u * (rank * 32 + (r & 31)), owner);
    const uint32_t t_o = tmem + (static_cast<uint32_t>(32 * warp) << 16) + kOColP;
    if (__all_sync(0xffffffffu, have_share)) {
#pragma unroll
      for (int c = 0; c < kDP / 32; ++c) {
        uint32_t o[32];
        tmem_ld_32x32b_x32(t_o + 32 * c, o);
        tmem_ld_wait();
#pragma unroll
        for (int v = 0; v < 8; ++v)
          st_cluster_f4(o_dst + 4u * (32 * c + 4 * v),
                        make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                    __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3])));
      }
      st_cluster_f2(ml_dst, make_float2(share_m2, share_l));
    } else {
      // no keys in this share (or a wait gave up): weight 0 in the combine
#pragma unroll
      for (int v = 0; v < kDP / 4; ++v) st_cluster_f4(o_dst + 16u * v, make_float4(0.0f, 0.0f, 0.0f, 0.0f));
      st_cluster_f2(ml_dst, make_float2(-INFINITY, 0.0f));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarpP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  // ---- the cluster's combine: after the barrier this CTA holds, for its rows
  // [32 rank, 32 rank + 32), the four shares in rank order:
  // M2 = max m2, w = 2^(m2 - M2), O = sum w acc / sum w l
  cluster_sync();
  if (warp < 4) {
    const int row = 32 * rank + lane;  // a warp's lanes take the 32 rows, the warp a quarter of the head dim
    const int d0 = 32 * warp;
    const int tok = tok0 + row / G;
    const float* slots = reinterpret_cast<const float*>(&s.k[0][0][0]);
    const float2* slot_ml = reinterpret_cast<const float2*>(&s.v[0][0][0]);
    float2 e[kClusterP];
#pragma unroll
    for (int c = 0; c < kClusterP; ++c) e[c] = slot_ml[c * 32 + lane];
    float M2 = -INFINITY;
#pragma unroll
    for (int c = 0; c < kClusterP; ++c) M2 = fmaxf(M2, e[c].x);
    float a[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) a[i] = 0.0f;
    float Ls = 0.0f;
#pragma unroll
    for (int c = 0; c < kClusterP; ++c) {
      const float w = ex2_approx(__fsub_rn(e[c].x, M2));  // 0 for a share with no keys
      Ls = __fmaf_rn(w, e[c].y, Ls);
      const float4* src = reinterpret_cast<const float4*>(slots + (c * 32 + lane) * kStashLd + d0);
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        const float4 x = src[v];
        a[4 * v] = __fmaf_rn(w, x.x, a[4 * v]);
        a[4 * v + 1] = __fmaf_rn(w, x.y, a[4 * v + 1]);
        a[4 * v + 2] = __fmaf_rn(w, x.z, a[4 * v + 2]);
        a[4 * v + 3] = __fmaf_rn(w, x.w, a[4 * v + 3]);
      }
    }
    if (tok < q_len) {
      // one reciprocal per row: x * RN(1/l) is within 1.5 fp32 ulp of x / l, far
      // below the bf16 rounding that follows
      const float rl = __frcp_rn(Ls);
      uint4* d4 = reinterpret_cast<uint4*>(p.out + ((int64_t)(p.q_off[b] + tok) * p.q_heads + kvh * G + row % G) * kDP +
                                           d0);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        uint32_t w4[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
          w4[k] = bf16x2(__fmul_rn(a[8 * v + 2 * k], rl), __fmul_rn(a[8 * v + 2 * k + 1], rl));
        d4[v] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
    }
  }
}

// bf16 [rows][heads][128] tensor, box {64, box_heads, box_rows}, 128-byte swizzle.
bool make_map_rows(CUtensorMap* m, const void* base, int64_t rows, int heads, int box_heads, int box_rows) {
  const TensorMapEncodeFn fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kDP, (cuuint64_t)heads, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {(cuuint64_t)kDP * 2, (cuuint64_t)heads * kDP * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)box_heads, (cuuint32_t)box_rows};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t gqa_prefill_ws_bytes(const PrefillSeq*, int32_t, int32_t, int32_t, int32_t) {
  return 256;  // the error word: the split of a tile's keys is combined on chip
}

cudaError_t launch_gqa_prefill(const void* q, const void* k, const void* v, int64_t total_q, int64_t total_kv,
                               const PrefillSeq* seqs, int32_t n_seqs, int32_t q_heads, int32_t kv_heads,
                               int32_t causal, void* out, uint8_t* ws, cudaStream_t st) {
  const int G = q_heads / kv_heads;
  const int tpt = kQTile / G;
  CUtensorMap tq, tk, tv;
  if (!make_map_rows(&tq, q, total_q, q_heads, G, tpt) || !make_map_rows(&tk, k, total_kv, kv_heads, 1, kKvTile) ||
      !make_map_rows(&tv, v, total_kv, kv_heads, 1, kKvTile))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(SmemP) + 1024;
  cudaError_t e = cudaFuncSetAttribute(gqa_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  for (int32_t s0 = 0; s0 < n_seqs; s0 += kPrefillMaxSeqs) {
    PrefillParams p;
    p.n_seqs = n_seqs - s0 < kPrefillMaxSeqs ? n_seqs - s0 : kPrefillMaxSeqs;
    p.q_heads = q_heads;
    p.kv_heads = kv_heads;
    p.group = G;
    p.tokens_per_tile = tpt;
    p.causal = causal;
    p.c2 = 0.12751743074419465f;  // log2(e) / sqrt(128)
    p.out = reinterpret_cast<__nv_bfloat16*>(out);
    p.err = reinterpret_cast<uint32_t*>(ws);
    int tiles = 0;
    for (int i = 0; i < p.n_seqs; ++i) {
      const PrefillSeq& sq = seqs[s0 + i];
      p.q_off[i] = static_cast<int32_t>(sq.q_off);
      p.q_len[i] = static_cast<int32_t>(sq.q_len);
      p.kv_off[i] = static_cast<int32_t>(sq.kv_off);
      p.kv_len[i] = static_cast<int32_t>(sq.kv_len);
      p.tile_start[i] = tiles;
      tiles += static_cast<int>((sq.q_len + tpt - 1) / tpt);
    }
    p.tile_start[p.n_seqs] = tiles;
    if (tiles == 0) continue;
    // one cluster of kClusterP CTAs per (query tile, key/value head)
    dim3 grid(static_cast<unsigned>(tiles * kClusterP), static_cast<unsigned>(kv_heads));
    gqa_prefill_kernel<<<grid, kThreadsP, smem, st>>>(tq, tk, tv, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace sdm
