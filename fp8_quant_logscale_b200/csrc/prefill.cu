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

#include <vector>

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

struct PrefillParams {
  int32_t n_seqs, q_heads, kv_heads, group, tokens_per_tile, causal, split_keys;
  int32_t q_off[kPrefillMaxSeqs], q_len[kPrefillMaxSeqs], kv_off[kPrefillMaxSeqs], kv_len[kPrefillMaxSeqs];
  int32_t tile_start[kPrefillMaxSeqs + 1];  // prefix sum of query tiles over the sequences
  int32_t item_start[kPrefillMaxSeqs + 1];  // prefix sum of (query tile, key chunk) work items
  float c2;                                 // log2(e) / sqrt(128)
  __nv_bfloat16* out;                       // [total_q][Hq][128]
  uint32_t* err;
  uint32_t* tickets;                        // [tiles][kv_heads], zero between launches
  float* part_ml;                           // [items][kv_heads][128][2]: m2, l
  float* part_acc;                          // [items][kv_heads][128][128]
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

__global__ void __launch_bounds__(kThreadsP, 1)
    gqa_prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  SmemP& s = *reinterpret_cast<SmemP*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const volatile uint32_t* abort_flag = &s.abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- which sequence, key/value head, query tile and key chunk
  int b = 0;
  while (b + 1 < p.n_seqs && p.item_start[b + 1] <= static_cast<int>(blockIdx.x)) ++b;
  const int kvh = blockIdx.y;
  const int G = p.group, tpt = p.tokens_per_tile, L = p.split_keys;
  const int q_len = p.q_len[b], kv_len = p.kv_len[b];
  // keys the rows of query tile t see: the causal limit of its last token
  auto tile_keys = [&](int t) {
    const int te = (t + 1) * tpt < q_len ? (t + 1) * tpt : q_len;
    return p.causal ? kv_len - q_len + te : kv_len;
  };
  int qt = 0, chunk = static_cast<int>(blockIdx.x) - p.item_start[b], item0 = p.item_start[b];
  while (true) {  // walk the tiles of sequence b to this item's (tile, chunk)
    const int nc = (tile_keys(qt) + L - 1) / L;
    if (chunk < nc) break;
    chunk -= nc;
    item0 += nc;
    ++qt;
  }
  const int n_chunks = (tile_keys(qt) + L - 1) / L;
  const int tok0 = qt * tpt;
  const int kv_lo = chunk * L;
  const int kv_hi = kv_lo + L < tile_keys(qt) ? kv_lo + L : tile_keys(qt);
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
      tc_fence_after();
      const float lf = ((l[0] + l[1]) + (l[2] + l[3])) + ((l[4] + l[5]) + (l[6] + l[7]));
      if (n_chunks == 1) {
        // one reciprocal per row: x * RN(1/l) is within 1.5 fp32 ulp of x / l, far
        // below the bf16 rounding that follows
        const float rl = __frcp_rn(lf);
        __nv_bfloat16* dst = p.out + ((int64_t)(p.q_off[b] + tok) * p.q_heads + kvh * G + r % G) * kDP;
#pragma unroll
        for (int c = 0; c < kDP / 32; ++c) {
          uint32_t o[32];
          tmem_ld_32x32b_x32(t_o + 32 * c, o);
          tmem_ld_wait();
          if (valid) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint32_t w[4];
#pragma unroll
              for (int k = 0; k < 4; ++k)
                w[k] = bf16x2(__fmul_rn(__uint_as_float(o[8 * v + 2 * k]), rl),
                              __fmul_rn(__uint_as_float(o[8 * v + 2 * k + 1]), rl));
              d4[v] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      } else {
        // one chunk of the keys: the unnormalised O, m2 and l for the combine
        const int64_t prow = ((int64_t)(item0 + chunk) * p.kv_heads + kvh) * kQTile + r;
        float4* acc = reinterpret_cast<float4*>(p.part_acc + prow * kDP);
#pragma unroll
        for (int c = 0; c < kDP / 32; ++c) {
          uint32_t o[32];
          tmem_ld_32x32b_x32(t_o + 32 * c, o);
          tmem_ld_wait();
#pragma unroll
          for (int v = 0; v < 8; ++v)
            acc[8 * c + v] = make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                         __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3]));
        }
        reinterpret_cast<float2*>(p.part_ml)[prow] = make_float2(m2, lf);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarpP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (n_chunks > 1) {
    // the last CTA of this query tile to finish combines the chunks in chunk
    // order (M2 = max m2, w = 2^(m2 - M2), O = sum w acc / sum w l) and returns
    // the ticket to zero for the next launch.  The block barrier above orders
    // every thread's partial stores before thread 0's release fence and ticket.
    const int64_t tile_id = (int64_t)(p.tile_start[b] + qt) * p.kv_heads + kvh;
    if (threadIdx.x == 0) {
      __threadfence();
      s.last = atomicAdd(p.tickets + tile_id, 1u) == static_cast<uint32_t>(n_chunks - 1);
      __threadfence();
    }
    __syncthreads();
    if (s.last) {
      if (warp < 4) {
        const int r = 32 * warp + lane;
        const int tok = tok0 + r / G;
        const float2* ml = reinterpret_cast<const float2*>(p.part_ml);
        const int64_t base = ((int64_t)item0 * p.kv_heads + kvh) * kQTile + r;  // chunk 0 of this row
        const int64_t step = (int64_t)p.kv_heads * kQTile;                      // next chunk
        float M2 = -INFINITY;
        for (int c = 0; c < n_chunks; ++c) M2 = fmaxf(M2, __ldcg(&ml[base + c * step].x));
        if (tok < q_len) {
          float a[kDP];
#pragma unroll
          for (int i = 0; i < kDP; ++i) a[i] = 0.0f;
          float Ls = 0.0f;
          for (int c = 0; c < n_chunks; ++c) {
            const float2 e = __ldcg(&ml[base + c * step]);
            const float w = ex2_approx(__fsub_rn(e.x, M2));
            Ls = __fmaf_rn(w, e.y, Ls);
            const float4* src = reinterpret_cast<const float4*>(p.part_acc + (base + c * step) * kDP);
            float4 x[kDP / 4];
#pragma unroll
            for (int v = 0; v < kDP / 4; ++v) x[v] = __ldcg(src + v);  // the chunk's row: 32 loads in flight
#pragma unroll
            for (int v = 0; v < kDP / 4; ++v) {
              a[4 * v] = __fmaf_rn(w, x[v].x, a[4 * v]);
              a[4 * v + 1] = __fmaf_rn(w, x[v].y, a[4 * v + 1]);
              a[4 * v + 2] = __fmaf_rn(w, x[v].z, a[4 * v + 2]);
              a[4 * v + 3] = __fmaf_rn(w, x[v].w, a[4 * v + 3]);
            }
          }
          const float rl = __frcp_rn(Ls);
          uint4* d4 = reinterpret_cast<uint4*>(p.out + ((int64_t)(p.q_off[b] + tok) * p.q_heads + kvh * G + r % G) * kDP);
#pragma unroll
          for (int v = 0; v < kDP / 8; ++v) {
            uint32_t w4[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
              w4[k] = bf16x2(__fmul_rn(a[8 * v + 2 * k], rl), __fmul_rn(a[8 * v + 2 * k + 1], rl));
            d4[v] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
      }
      if (threadIdx.x == 0) p.tickets[tile_id] = 0u;
    }
  }
}

typedef CUresult (*EncodeTiledFnP)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFnP encode_fn_p() {
  static EncodeTiledFnP fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFnP>(ptr);
  }
  return fn;
}

// bf16 [rows][heads][128] tensor, box {64, box_heads, box_rows}, 128-byte swizzle.
bool make_map_rows(CUtensorMap* m, const void* base, int64_t rows, int heads, int box_heads, int box_rows) {
  EncodeTiledFnP fn = encode_fn_p();
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

namespace {
constexpr int kPrefillSplitKeys = 2048;  // keys per chunk: longer key ranges are split over CTAs

struct PrefillLaunch {  // one launch: sequences [s0, s0 + n)
  int32_t s0, n, tiles, items;
};

inline size_t al1k(size_t x) { return (x + 1023) / 1024 * 1024; }

// Tiles and work items of the launches covering all sequences.
std::vector<PrefillLaunch> plan_prefill(const PrefillSeq* seqs, int32_t n_seqs, int32_t tpt, int32_t causal) {
  std::vector<PrefillLaunch> out;
  for (int32_t s0 = 0; s0 < n_seqs; s0 += kPrefillMaxSeqs) {
    PrefillLaunch l{s0, n_seqs - s0 < kPrefillMaxSeqs ? n_seqs - s0 : kPrefillMaxSeqs, 0, 0};
    for (int32_t i = 0; i < l.n; ++i) {
      const PrefillSeq& q = seqs[s0 + i];
      const int64_t nt = (q.q_len + tpt - 1) / tpt;
      for (int64_t t = 0; t < nt; ++t) {
        const int64_t te = (t + 1) * tpt < q.q_len ? (t + 1) * tpt : q.q_len;
        const int64_t keys = causal ? q.kv_len - q.q_len + te : q.kv_len;
        l.items += static_cast<int32_t>((keys + kPrefillSplitKeys - 1) / kPrefillSplitKeys);
      }
      l.tiles += static_cast<int32_t>(nt);
    }
    out.push_back(l);
  }
  return out;
}

// Scratch after the 256-byte error word: tickets, then the chunk partials.
struct PrefillScratch {
  size_t tickets, ml, acc, total;
};
PrefillScratch prefill_scratch(int32_t tiles, int32_t items, int32_t kv_heads) {
  PrefillScratch w;
  w.tickets = 256;
  w.ml = al1k(w.tickets + (size_t)tiles * kv_heads * sizeof(uint32_t));
  w.acc = al1k(w.ml + (size_t)items * kv_heads * kQTile * 2 * sizeof(float));
  w.total = al1k(w.acc + (size_t)items * kv_heads * kQTile * kDP * sizeof(float));
  return w;
}
}  // namespace

size_t gqa_prefill_ws_bytes(const PrefillSeq* seqs, int32_t n_seqs, int32_t q_heads, int32_t kv_heads,
                            int32_t causal) {
  const int32_t tpt = kQTile / (q_heads / kv_heads);
  size_t need = 256;
  for (const PrefillLaunch& l : plan_prefill(seqs, n_seqs, tpt, causal)) {
    const size_t t = prefill_scratch(l.tiles, l.items, kv_heads).total;
    need = t > need ? t : need;
  }
  return need;
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
  for (const PrefillLaunch& l : plan_prefill(seqs, n_seqs, tpt, causal)) {
    if (l.items == 0) continue;
    const PrefillScratch w = prefill_scratch(l.tiles, l.items, kv_heads);
    PrefillParams p;
    p.n_seqs = l.n;
    p.q_heads = q_heads;
    p.kv_heads = kv_heads;
    p.group = G;
    p.tokens_per_tile = tpt;
    p.causal = causal;
    p.split_keys = kPrefillSplitKeys;
    p.c2 = 0.12751743074419465f;  // log2(e) / sqrt(128)
    p.out = reinterpret_cast<__nv_bfloat16*>(out);
    p.err = reinterpret_cast<uint32_t*>(ws);
    p.tickets = reinterpret_cast<uint32_t*>(ws + w.tickets);
    p.part_ml = reinterpret_cast<float*>(ws + w.ml);
    p.part_acc = reinterpret_cast<float*>(ws + w.acc);
    int tiles = 0, items = 0;
    for (int i = 0; i < l.n; ++i) {
      const PrefillSeq& sq = seqs[l.s0 + i];
      p.q_off[i] = static_cast<int32_t>(sq.q_off);
      p.q_len[i] = static_cast<int32_t>(sq.q_len);
      p.kv_off[i] = static_cast<int32_t>(sq.kv_off);
      p.kv_len[i] = static_cast<int32_t>(sq.kv_len);
      p.tile_start[i] = tiles;
      p.item_start[i] = items;
      const int nt = static_cast<int>((sq.q_len + tpt - 1) / tpt);
      for (int t = 0; t < nt; ++t) {
        const int64_t te = (int64_t)(t + 1) * tpt < sq.q_len ? (int64_t)(t + 1) * tpt : sq.q_len;
        const int64_t keys = causal ? sq.kv_len - sq.q_len + te : sq.kv_len;
        items += static_cast<int>((keys + kPrefillSplitKeys - 1) / kPrefillSplitKeys);
      }
      tiles += nt;
    }
    p.tile_start[l.n] = tiles;
    p.item_start[l.n] = items;
    dim3 grid(static_cast<unsigned>(items), static_cast<unsigned>(kv_heads));
    gqa_prefill_kernel<<<grid, kThreadsP, smem, st>>>(tq, tk, tv, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace sdm
