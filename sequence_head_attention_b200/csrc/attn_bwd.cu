// attn_bwd.cu -- gradients of exact multi-head attention on the 5th-generation tensor cores (sm_100a).
//
// What it computes (the backward pass of the attention in attn_fwd.cu, whose speed the CHARM+ pages
// report next to the forward's: "CHARM+ ...", abstract), for an upstream gradient dO of O, with
// p_ij = exp(q_i.k_j / sqrt(D) - lse_i) over the keys j that query i sees (all, or j <= i when causal):
//   delta_i = dO_i . O_i
//   dV_j = sum_i p_ij dO_i,   dp_ij = dO_i . v_j,   ds_ij = p_ij (dp_ij - delta_i)
//   dK_j = sum_i ds_ij q_i / sqrt(D),   dQ_i = sum_j ds_ij k_j / sqrt(D)
// lse is the forward's natural-log log-sum-exp, so p is recomputed exactly as the forward normalised it.
//
// How: three launches.
//   bwd_delta_kernel   delta = rowsum(dO * O), fp32 [B, H, S] (HBM-bound, 16-byte loads).
//   bwd_kernel<D, false>  one CTA per (b, h, key tile of 128): K and V stay in shared memory while the
//                      query tiles stream through a two-slot ring.  Per query tile, on the tensor cores:
//                      S^T = K Q^T and dP^T = V dO^T (both operands in shared memory, fp32 in TMEM); the
//                      eight row warps turn them into P^T and dS^T (bf16, written back over S^T and dP^T in
//                      TMEM); then dV += P^T dO and dK += dS^T Q with the left operand read from TMEM.
//   bwd_kernel<D, true>   one CTA per (b, h, query tile): Q and dO stay, key tiles stream; S = Q K^T and
//                      dP = dO V^T, then dS, then dQ += dS K.
//   Streamed tiles are taken in halves of 64 rows, alternating between two TMEM buffers, so the tensor
//   cores compute one half while the row warps work on the other.
//   Warps: 0 TMA producer, 1 MMA issuer (one elected lane), 2-3 idle, 4-11 the 128 tile rows (one row per
//   thread; the TMEM lane quadrant of warp w is w % 4, and warps w and w + 4 take 32 columns each of a
//   half).  TMEM: buffer b holds S at [128 b, 128 b + 64) and dP at [128 b + 64, 128 b + 128);
//   accumulators from 256 (dV then dK, or dQ).  The MMA issuer queues a half's S and dP right behind the
//   previous half's accumulating MMAs: tcgen05 MMAs from one thread execute in order, so a new S cannot
//   overwrite P before it has been read.
// Every barrier wait is bounded in time; on expiry the kernel records an error and returns cleanly.
#include <cuda_bf16.h>

#include <climits>
#include <cstdint>

#include "sp_internal.h"
#include "sp_ptx.cuh"

namespace spattn {
namespace {

constexpr int kBT = 128;           // tile edge
constexpr int kBwdThreads = 384;   // 12 warps
constexpr int kWarpLoad = 0, kWarpIssue = 1, kWarpRow0 = 4;
constexpr int kRowWarps = 8;       // two per TMEM lane quadrant, 32 columns of a 64-row half each

template <int D>
struct BCfg {
  static constexpr int kSub = D / 64;
  static constexpr int kTileBytes = kBT * D * 2;
  static constexpr int kStages = 2;
  // resident tiles (K, V or Q, dO) at [0, 2 tiles); then per slot: two streamed tiles and 2 x 128 floats
  static constexpr int kResOff = 0;
  static constexpr int kStageOff = 2 * kTileBytes;
  static constexpr int kStageBytes = 2 * kTileBytes + 1024;
  static constexpr int kBarOff = kStageOff + kStages * kStageBytes;
  // res_full, full[S], empty[S], st_full[2], p_full[2], acc_full, drain
  static constexpr int kNumBars = 1 + 2 * kStages + 6;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  // one CTA per SM: its TMEM allocation takes all 512 columns
  static constexpr int kRaw = kMiscOff + 16 + 1024;
  static constexpr int kSmemBytes = kRaw > 120 * 1024 ? kRaw : 120 * 1024;
  static constexpr uint32_t kIdescSq = idesc_bf16_f32(128, 64, false, false);  // S, dP of a 64-row half; K-major
  static constexpr uint32_t kIdescAcc = idesc_bf16_f32(128, D, false, true);    // B operand MN-major
};

struct BwdMaps {
  CUtensorMap q, k, v, dout;
};

struct BwdBars {
  uint32_t res_full, full0, empty0, st_full0, p_full0, acc_full, drain;
  __device__ uint32_t full(int s) const { return full0 + 8u * s; }
  __device__ uint32_t empty(int s) const { return empty0 + 8u * s; }
  __device__ uint32_t st_full(int b) const { return st_full0 + 8u * b; }  // per TMEM buffer
  __device__ uint32_t p_full(int b) const { return p_full0 + 8u * b; }
};

// TMEM: two buffers of a 64-row half of a streamed tile, each S (64 columns) then dP (64 columns): buffer b
// at columns [128 b, 128 b + 128); accumulators from 256.
__device__ __forceinline__ uint32_t tS_of(uint32_t t, int b) { return t + 128u * b; }
__device__ __forceinline__ uint32_t tdP_of(uint32_t t, int b) { return t + 128u * b + 64u; }
// The row warp of columns [32 j, 32 j + 32) of a half packs their bf16 P (dS) into the 16 columns at 32 j of
// the S (dP) region, columns it has itself just read.  K-step kk (16 rows of the half) of an accumulating
// MMA therefore starts at packed column 32 (kk / 2) + 8 (kk % 2).
__device__ __forceinline__ uint32_t packed_col(int kk) { return 32u * (kk >> 1) + 8u * (kk & 1); }

// The CTA's tile and the range of streamed tiles it walks.
struct BwdItem {
  int b, h, tile;      // resident tile index (key tile for dK/dV, query tile for dQ)
  int first, n_steps;  // streamed tiles first .. first + n_steps - 1
};

template <bool kDQ>
__device__ __forceinline__ BwdItem bwd_item(const BwdParams& p) {
  BwdItem it;
  const int w = blockIdx.x;
  if (kDQ) {  // every query tile; key tiles of the range, up to (causal) the query tile's own
    it.b = w / (p.H * p.T);
    it.h = (w / p.T) % p.H;
    it.tile = w % p.T;
    it.first = p.kt0;
    const int last = p.causal ? min(p.kt0 + p.n_kt, it.tile + 1) : p.kt0 + p.n_kt;  // exclusive
    it.n_steps = max(0, last - it.first);
  } else {    // the range's key tiles; query tiles (causal: from the key tile's own) .. T-1
    it.b = w / (p.H * p.n_kt);
    it.h = (w / p.n_kt) % p.H;
    it.tile = p.kt0 + w % p.n_kt;
    it.first = p.causal ? it.tile : 0;
    it.n_steps = p.T - it.first;
  }
  return it;
}

// ------------------------------------------------------------------------------------------------
template <int D, bool kDQ>
__device__ void bwd_load(const BwdParams& p, const BwdMaps& tm, const BwdItem& it, uint32_t sbase, uint8_t* smem,
                         const BwdBars& bars, volatile int* abort_flag) {
  using C = BCfg<D>;
  const int lane = threadIdx.x & 31;
  const uint64_t tmo = p.timeout_ns;
  const CUtensorMap* res0 = kDQ ? &tm.q : &tm.k;     // resident pair
  const CUtensorMap* res1 = kDQ ? &tm.dout : &tm.v;
  const CUtensorMap* str0 = kDQ ? &tm.k : &tm.q;     // streamed pair
  const CUtensorMap* str1 = kDQ ? &tm.v : &tm.dout;
  if (elect_one_sync()) {
    mbar_arrive_expect_tx(bars.res_full, 2 * C::kTileBytes);
#pragma unroll
    for (int c = 0; c < C::kSub; ++c) {
      tma_load_4d(sbase + C::kResOff + c * 16384, res0, bars.res_full, 64 * c, it.h, it.tile * kBT, it.b);
      tma_load_4d(sbase + C::kResOff + C::kTileBytes + c * 16384, res1, bars.res_full, 64 * c, it.h, it.tile * kBT,
                  it.b);
    }
  }
  __syncwarp();
  int issued = 0;
  bool ok = true;
  for (int n = 0; n < it.n_steps && ok; ++n) {
    const int s = n % C::kStages;
    const int lap = n / C::kStages;
    const int t = it.first + n;
    // the streamed query tile's lse (in log2 units) and delta, one per column of S^T, read before the
    // wait for the slot so that their latency hides behind it; rows past S get lse = +inf, so their
    // probabilities are exactly 0
    float l2v[kBT / 32], dlv[kBT / 32];
    if (!kDQ) {
      const size_t base = ((size_t)it.b * p.H + it.h) * p.S;
#pragma unroll
      for (int j = 0; j < kBT / 32; ++j) {
        const int row = t * kBT + lane + 32 * j;
        l2v[j] = row < p.S ? __ldg(p.lse + base + row) * 1.4426950408889634f : INFINITY;
        dlv[j] = row < p.S ? __ldg(p.delta + base + row) : 0.f;
      }
    }
    if (lap > 0) {
      ok = warp_mbar_wait(bars.empty(s), (lap - 1) & 1, tmo, ERR_TIMEOUT_KV_EMPTY, abort_flag, p.err);
      if (!ok) break;
    }
    const uint32_t stage = sbase + C::kStageOff + s * C::kStageBytes;
    if (!kDQ) {
      float* lse2 = reinterpret_cast<float*>(smem + C::kStageOff + s * C::kStageBytes + 2 * C::kTileBytes);
      float* dlt = lse2 + kBT;
#pragma unroll
      for (int j = 0; j < kBT / 32; ++j) {
        lse2[lane + 32 * j] = l2v[j];
        dlt[lane + 32 * j] = dlv[j];
      }
      __threadfence_block();
      __syncwarp();
    }
    if (elect_one_sync()) {
      mbar_arrive_expect_tx(bars.full(s), 2 * C::kTileBytes);
#pragma unroll
      for (int c = 0; c < C::kSub; ++c) {
        tma_load_4d(stage + c * 16384, str0, bars.full(s), 64 * c, it.h, t * kBT, it.b);
        tma_load_4d(stage + C::kTileBytes + c * 16384, str1, bars.full(s), 64 * c, it.h, t * kBT, it.b);
      }
    }
    __syncwarp();
    issued = n + 1;
  }
  if (*abort_flag) {  // no copy may still be landing when the CTA exits: wait (bounded) for the last ones
    warp_mbar_wait(bars.res_full, 0, tmo, ERR_TIMEOUT_Q_FULL, nullptr, p.err);
    for (int n = issued > C::kStages ? issued - C::kStages : 0; n < issued; ++n)
      warp_mbar_wait(bars.full(n % C::kStages), (n / C::kStages) & 1, tmo, ERR_TIMEOUT_KV_FULL, nullptr, p.err);
  }
}

// ------------------------------------------------------------------------------------------------
template <int D, bool kDQ>
__device__ void bwd_issue(const BwdParams& p, const BwdItem& it, uint32_t sbase, uint32_t tmem_in, const BwdBars& bars,
                          volatile int* abort_flag) {
  using C = BCfg<D>;
  const uint64_t tmo = p.timeout_ns;
  const uint32_t tmem = __shfl_sync(0xffffffffu, tmem_in, 0);
  const uint32_t tAcc0 = tmem + 256, tAcc1 = tmem + 256 + D;
  // K-major descriptors of K-step 0 (the row-major tiles as the MMAs' K-major operands), and MN-major ones
  // of the streamed tiles as the right operand of the accumulating MMAs.  Streamed tiles are taken in two
  // halves of 64 rows (sub-step m = 2 n + h, TMEM buffer h): half h starts 8192 bytes into each 64-column
  // sub-tile.  The S and dP of half m are issued before the accumulating MMAs of half m - 1, so the tensor
  // cores run one half while the row warps work on the other.
  const uint64_t res0_k = smem_desc_sw128(sbase + C::kResOff, 16, 1024);
  const uint64_t res1_k = smem_desc_sw128(sbase + C::kResOff + C::kTileBytes, 16, 1024);
  bool ok = warp_mbar_wait(bars.res_full, 0, tmo, ERR_TIMEOUT_Q_FULL, abort_flag, p.err);
  // accumulating MMAs of half hh of streamed tile nn (rows 64 hh .. 64 hh + 63), from TMEM buffer hh
  auto accumulate = [&](int nn, int hh) {
    const uint32_t stage = sbase + C::kStageOff + (nn % C::kStages) * C::kStageBytes;
    const uint64_t str0_mn = smem_desc_sw128(stage, 16384, 1024) + (uint64_t)((8192 * hh) >> 4);
    const uint64_t str1_mn = smem_desc_sw128(stage + C::kTileBytes, 16384, 1024) + (uint64_t)((8192 * hh) >> 4);
    const bool first = nn == 0 && hh == 0;
    if (kDQ) {
      // dQ += dS K
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ts(tAcc0, tdP_of(tmem, hh) + packed_col(kk), str0_mn + (uint64_t)(kk * 128), C::kIdescAcc,
               (first && kk == 0) ? 0u : 1u);
    } else {
      // dV += P^T dO, dK += dS^T Q
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ts(tAcc0, tS_of(tmem, hh) + packed_col(kk), str1_mn + (uint64_t)(kk * 128), C::kIdescAcc,
               (first && kk == 0) ? 0u : 1u);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ts(tAcc1, tdP_of(tmem, hh) + packed_col(kk), str0_mn + (uint64_t)(kk * 128), C::kIdescAcc,
               (first && kk == 0) ? 0u : 1u);
    }
    if (hh == 1) mma_commit(bars.empty(nn % C::kStages));  // both halves of the tile consumed
  };
  const int n_sub = 2 * it.n_steps;
  for (int m = 0; m < n_sub && ok; ++m) {
    const int n = m >> 1, h = m & 1;
    if (h == 0) {
      ok = warp_mbar_wait(bars.full(n % C::kStages), (n / C::kStages) & 1, tmo, ERR_TIMEOUT_KV_FULL, abort_flag, p.err);
      if (!ok) break;
      tc_fence_after();
    }
    const uint32_t stage = sbase + C::kStageOff + (n % C::kStages) * C::kStageBytes;
    const uint64_t str0_k = smem_desc_sw128(stage, 16, 1024) + (uint64_t)((8192 * h) >> 4);
    const uint64_t str1_k = smem_desc_sw128(stage + C::kTileBytes, 16, 1024) + (uint64_t)((8192 * h) >> 4);
    if (elect_one_sync()) {
      // dK/dV: S^T = K Q_h^T, dP^T = V dO_h^T.   dQ: S = Q K_h^T, dP = dO V_h^T.
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = (uint64_t)(((kk / 4) * 16384 + (kk % 4) * 32) >> 4);
        mma_ss(tS_of(tmem, h), res0_k + off, str0_k + off, C::kIdescSq, kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = (uint64_t)(((kk / 4) * 16384 + (kk % 4) * 32) >> 4);
        mma_ss(tdP_of(tmem, h), res1_k + off, str1_k + off, C::kIdescSq, kk > 0 ? 1u : 0u);
      }
      mma_commit(bars.st_full(h));
    }
    __syncwarp();
    if (m > 0) {  // the previous half: once its P and dS are in TMEM
      const int mp = m - 1, hp = mp & 1;
      ok = warp_mbar_wait(bars.p_full(hp), (mp >> 1) & 1, tmo, ERR_TIMEOUT_P_FULL, abort_flag, p.err);
      if (!ok) break;
      tc_fence_after();
      if (elect_one_sync()) accumulate(mp >> 1, hp);
      __syncwarp();
    }
  }
  if (ok && n_sub > 0) {  // the last half
    const int mp = n_sub - 1, hp = mp & 1;
    ok = warp_mbar_wait(bars.p_full(hp), (mp >> 1) & 1, tmo, ERR_TIMEOUT_P_FULL, abort_flag, p.err);
    if (ok) {
      tc_fence_after();
      if (elect_one_sync()) accumulate(mp >> 1, hp);
      __syncwarp();
    }
  }
  if (ok && elect_one_sync()) mma_commit(bars.acc_full);
  __syncwarp();
  // nothing of ours may still run on the tensor cores when TMEM is released
  if (elect_one_sync()) mma_commit(bars.drain);
  __syncwarp();
  warp_mbar_wait(bars.drain, 0, tmo, ERR_TIMEOUT_DRAIN, nullptr, p.err);
}

// ------------------------------------------------------------------------------------------------
// P and dS of 32 columns (streamed-tile rows c0 .. c0 + 31) of this thread's row, packed to bf16 pairs.
// dK/dV: per-column lse (log2 units) and delta from shared memory; column c is kept when c >= lo.
// dQ: the row's lse and delta; column c is kept when c < hi.  kMask false: every column is kept.
template <bool kDQ, bool kMask>
__device__ __forceinline__ void bwd_chunk(const uint32_t (&s)[32], const uint32_t (&dp)[32], float sl2,
                                          float lse2_row, float dlt_row, const float* lse2, const float* dlt,
                                          int c0, int lo, int hi, uint32_t (&pk_p)[16], uint32_t (&pk_ds)[16]) {
#pragma unroll
  for (int e = 0; e < 32; e += 4) {
    float l4[4], d4[4];
    if (kDQ) {
#pragma unroll
      for (int u = 0; u < 4; ++u) { l4[u] = lse2_row; d4[u] = dlt_row; }
    } else {
      const float4 lv = *reinterpret_cast<const float4*>(lse2 + c0 + e);
      const float4 dv = *reinterpret_cast<const float4*>(dlt + c0 + e);
      l4[0] = lv.x; l4[1] = lv.y; l4[2] = lv.z; l4[3] = lv.w;
      d4[0] = dv.x; d4[1] = dv.y; d4[2] = dv.z; d4[3] = dv.w;
    }
    float pr[4], ds[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float pv = ex2_approx(__uint_as_float(s[e + u]) * sl2 - l4[u]);
      if (kMask) {
        const int c = c0 + e + u;
        if (kDQ ? c >= hi : c < lo) pv = 0.f;
      }
      pr[u] = pv;
      ds[u] = pv * (__uint_as_float(dp[e + u]) - d4[u]);
    }
    pk_p[e >> 1] = pack_bf16x2(pr[0], pr[1]);
    pk_p[(e >> 1) + 1] = pack_bf16x2(pr[2], pr[3]);
    pk_ds[e >> 1] = pack_bf16x2(ds[0], ds[1]);
    pk_ds[(e >> 1) + 1] = pack_bf16x2(ds[2], ds[3]);
  }
}

template <int D, bool kDQ>
__device__ void bwd_rows(const BwdParams& p, const BwdItem& it, uint8_t* smem, uint32_t tmem, const BwdBars& bars,
                         volatile int* abort_flag) {
  using C = BCfg<D>;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quad = warp & 3;
  const int j = (warp - kWarpRow0) >> 2;                         // this warp's 32 columns of each half
  const int r = quad * 32 + lane;                                // row of the resident tile
  const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
  const uint32_t tAcc0 = trow + 256, tAcc1 = trow + 256 + D;
  const uint64_t tmo = p.timeout_ns;
  const float sl2 = p.scale_log2;
  const int row = it.tile * kBT + r;                             // global position of this thread's row
  const int kv_lim = min(p.kv_end, p.S);
  // rows this CTA writes: queries < S (dQ); keys of the range (dK, dV)
  const bool row_out = kDQ ? row < p.S : row < kv_lim;
  float lse2_row = 0.f, dlt_row = 0.f;
  if (kDQ && row < p.S) {
    const size_t i = ((size_t)it.b * p.H + it.h) * p.S + row;
    lse2_row = __ldg(p.lse + i) * 1.4426950408889634f;
    dlt_row = __ldg(p.delta + i);
  }
  bool ok = true;
  // sub-step m = 2 n + h: the 64 rows 64 h .. 64 h + 63 of streamed tile n, in TMEM buffer h
  for (int m = 0; m < 2 * it.n_steps; ++m) {
    const int n = m >> 1, h = m & 1;
    const int t = it.first + n;
    const float* lse2 = reinterpret_cast<const float*>(smem + C::kStageOff + (n % C::kStages) * C::kStageBytes +
                                                       2 * C::kTileBytes);
    const float* dlt = lse2 + kBT;
    if (!kDQ && h == 0) {
      // lse and delta of the streamed tile were stored by the producer before it released the slot's
      // full barrier: acquire them from that barrier (the slot is refilled only after both halves' P
      // arrive, so the phase cannot have moved on)
      ok = mbar_wait(bars.full(n % C::kStages), (n / C::kStages) & 1, tmo, ERR_TIMEOUT_KV_FULL, abort_flag, p.err);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
    }
    ok = mbar_wait(bars.st_full(h), n & 1, tmo, ERR_TIMEOUT_S_FULL, abort_flag, p.err);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    tc_fence_after();
    const uint32_t tS = trow + 128u * h + 32u * j, tdP = tS + 64;
    uint32_t s[32], dp[32];
    tmem_ld32(tS, s);
    tmem_ld32(tdP, dp);
    const int c0 = 64 * h + 32 * j;  // first column: the streamed tile's row
    // kept columns: dK/dV, queries t kBT + c not before the key (causal); dQ, keys t kBT + c not after the
    // query (causal) and inside the key range
    const int lo = (!kDQ && p.causal) ? row - t * kBT : INT_MIN;
    const int hi = kDQ ? min(p.causal ? row - t * kBT + 1 : INT_MAX, kv_lim - t * kBT) : INT_MAX;
    const bool edge = kDQ ? hi < c0 + 32 : lo > c0;
    uint32_t pk_p[16], pk_ds[16];
    tmem_wait_ld();
    if (edge)
      bwd_chunk<kDQ, true>(s, dp, sl2, lse2_row, dlt_row, lse2, dlt, c0, lo, hi, pk_p, pk_ds);
    else
      bwd_chunk<kDQ, false>(s, dp, sl2, lse2_row, dlt_row, lse2, dlt, c0, lo, hi, pk_p, pk_ds);
    // packed into the first 16 of the 32 columns of S and dP this warp has just read
    if (!kDQ) tmem_st16(tS, pk_p);
    tmem_st16(tdP, pk_ds);
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bars.p_full(h));
  }
  if (!ok) return;
  ok = __all_sync(0xffffffffu, mbar_wait(bars.acc_full, 0, tmo, ERR_TIMEOUT_PV_DONE, abort_flag, p.err));
  if (!ok) return;
  if (it.n_steps == 0) return;  // (dQ of a key range before this query tile) nothing accumulated
  tc_fence_after();
  const float scale = p.scale;
  const size_t out = (((size_t)it.b * p.S + row) * p.H + it.h) * D;
#pragma unroll
  for (int which = 0; which < (kDQ ? 1 : 2); ++which) {
    // dQ: tAcc0, scaled.  dK/dV: dV from tAcc0 unscaled, dK from tAcc1 scaled.
    const uint32_t tacc = which == 0 ? tAcc0 : tAcc1;
    const float f = (kDQ || which == 1) ? scale : 1.f;
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(kDQ ? p.dq : (which == 0 ? p.dv : p.dk));
#pragma unroll 1
    for (int c = j * (D / 64); c < (j + 1) * (D / 64); ++c) {  // this warp's half of the D columns
      uint32_t a[32];
      tmem_ld32(tacc + c * 32, a);
      tmem_wait_ld();
      if (kDQ && p.dq_acc) {  // add this key range's contribution to the fp32 accumulator
        if (row_out) {
          float4* d4 = reinterpret_cast<float4*>(p.dq_acc + out + c * 32);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float4 x = d4[e];
            x.x += __uint_as_float(a[4 * e]) * f;
            x.y += __uint_as_float(a[4 * e + 1]) * f;
            x.z += __uint_as_float(a[4 * e + 2]) * f;
            x.w += __uint_as_float(a[4 * e + 3]) * f;
            d4[e] = x;
          }
        }
      } else if (row_out) {
        uint4* d4 = reinterpret_cast<uint4*>(dst + out + c * 32);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          d4[e] = make_uint4(pack_bf16x2(__uint_as_float(a[8 * e]) * f, __uint_as_float(a[8 * e + 1]) * f),
                             pack_bf16x2(__uint_as_float(a[8 * e + 2]) * f, __uint_as_float(a[8 * e + 3]) * f),
                             pack_bf16x2(__uint_as_float(a[8 * e + 4]) * f, __uint_as_float(a[8 * e + 5]) * f),
                             pack_bf16x2(__uint_as_float(a[8 * e + 6]) * f, __uint_as_float(a[8 * e + 7]) * f));
      }
    }
  }
}

template <int D, bool kDQ>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_kernel(const __grid_constant__ BwdMaps tm, const __grid_constant__ BwdParams p) {
  using C = BCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::kBarOff;
  BwdBars bars;
  bars.res_full = bar0;
  bars.full0 = bar0 + 8;
  bars.empty0 = bars.full0 + 8 * C::kStages;
  bars.st_full0 = bars.empty0 + 8 * C::kStages;
  bars.p_full0 = bars.st_full0 + 16;
  bars.acc_full = bars.p_full0 + 16;
  bars.drain = bars.acc_full + 8;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(bars.res_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bars.full(s), 1);
      mbar_init(bars.empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bars.st_full(b), 1);
      mbar_init(bars.p_full(b), kRowWarps);  // one arrival per row warp
    }
    mbar_init(bars.acc_full, 1);
    mbar_init(bars.drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpLoad && (threadIdx.x & 31) == 0) {
    tma_prefetch_desc(&tm.q);
    tma_prefetch_desc(&tm.k);
    tma_prefetch_desc(&tm.v);
    tma_prefetch_desc(&tm.dout);
  }
  if (warp == kWarpIssue) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const BwdItem it = bwd_item<kDQ>(p);
  if (warp == kWarpLoad) {
    bwd_load<D, kDQ>(p, tm, it, sbase, smem, bars, abort_flag);
  } else if (warp == kWarpIssue) {
    bwd_issue<D, kDQ>(p, it, sbase, tmem, bars, abort_flag);
  } else if (warp >= kWarpRow0) {
    bwd_rows<D, kDQ>(p, it, smem, tmem, bars, abort_flag);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpIssue) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// delta[b, h, i] = sum_d dO[b, i, h, d] * O[b, i, h, d]: D/8 lanes per row, 16-byte loads.
template <int D>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const __nv_bfloat16* __restrict__ o,
                                                        const __nv_bfloat16* __restrict__ dout,
                                                        float* __restrict__ delta, int B, int S, int H) {
  constexpr int kLanes = D / 8;             // lanes per row
  constexpr int kRowsPerWarp = 32 / kLanes;
  const long long n_rows = (long long)B * S * H;
  const int lane = threadIdx.x & 31;
  const int sub = lane / kLanes, l = lane % kLanes;
  const long long warps = (long long)gridDim.x * (blockDim.x / 32);
  for (long long w = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
       w * kRowsPerWarp < n_rows; w += warps) {
    const long long rrow = w * kRowsPerWarp + sub;  // (b, s, h) in BSHD order
    float acc = 0.f;
    if (rrow < n_rows) {
      const uint4 a = __ldcs(reinterpret_cast<const uint4*>(o + rrow * D) + l);
      const uint4 g = __ldcs(reinterpret_cast<const uint4*>(dout + rrow * D) + l);
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 x = __bfloat1622float2(a2[e]), y = __bfloat1622float2(g2[e]);
        acc = fmaf(x.x, y.x, acc);
        acc = fmaf(x.y, y.y, acc);
      }
    }
#pragma unroll
    for (int off = kLanes / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (rrow < n_rows && l == 0) {
      const long long h = rrow % H, bs = rrow / H, s = bs % S, b = bs / S;
      delta[(b * H + h) * S + s] = acc;
    }
  }
}

__global__ void __launch_bounds__(256) f32_to_bf16_kernel(const float4* __restrict__ in, uint2* __restrict__ out,
                                                          long long n4) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    const float4 x = __ldcs(in + i);
    out[i] = make_uint2(pack_bf16x2(x.x, x.y), pack_bf16x2(x.z, x.w));
  }
}

template <int D, bool kDQ>
sp_status launch_bwd_one(const BwdMaps& tm, const BwdParams& p, int grid, cudaStream_t stream) {
  using C = BCfg<D>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SP_ERR_CUDA;
  static bool attr_set[kMaxDevices] = {};
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(bwd_kernel<D, kDQ>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
        cudaSuccess)
      return SP_ERR_CUDA;
    attr_set[dev] = true;
  }
  bwd_kernel<D, kDQ><<<grid, kBwdThreads, C::kSmemBytes, stream>>>(tm, p);
  return cudaGetLastError() == cudaSuccess ? SP_OK : SP_ERR_CUDA;
}

}  // namespace

sp_status launch_attn_bwd(const BwdParams& p_in, const void* q, const void* k, const void* v, const void* o,
                          const void* dout, cudaStream_t stream) {
  BwdParams p = p_in;
  BwdMaps tm;
  if (!encode_bshd_tmap(&tm.q, q, p.B, p.S, p.H, p.D) || !encode_bshd_tmap(&tm.k, k, p.B, p.S, p.H, p.D) ||
      !encode_bshd_tmap(&tm.v, v, p.B, p.S, p.H, p.D) || !encode_bshd_tmap(&tm.dout, dout, p.B, p.S, p.H, p.D))
    return SP_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SP_ERR_CUDA;
  const long long rows = (long long)p.B * p.S * p.H;
  const int rows_per_block = 8 * (32 / (p.D / 8));
  long long blocks = (rows + rows_per_block - 1) / rows_per_block;
  const long long cap = (long long)num_sms(dev) * 8;
  if (blocks > cap) blocks = cap;
  if (p.D == 128)
    bwd_delta_kernel<128><<<(int)blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(o),
                                                            static_cast<const __nv_bfloat16*>(dout), p.delta, p.B, p.S, p.H);
  else
    bwd_delta_kernel<64><<<(int)blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(o),
                                                           static_cast<const __nv_bfloat16*>(dout), p.delta, p.B, p.S, p.H);
  if (cudaGetLastError() != cudaSuccess) return SP_ERR_CUDA;
  const long long items_kv = (long long)p.B * p.H * p.n_kt;  // dK/dV: the range's key tiles
  const long long items_q = (long long)p.B * p.H * p.T;      // dQ: every query tile
  if (items_q > 0x7fffffffLL) return SP_ERR_INVALID_ARG;
  if (items_kv > 0) {
    sp_status s = p.D == 128 ? launch_bwd_one<128, false>(tm, p, (int)items_kv, stream)
                             : launch_bwd_one<64, false>(tm, p, (int)items_kv, stream);
    if (s != SP_OK) return s;
  }
  return p.D == 128 ? launch_bwd_one<128, true>(tm, p, (int)items_q, stream)
                    : launch_bwd_one<64, true>(tm, p, (int)items_q, stream);
}

sp_status launch_f32_to_bf16(const float* in, void* out, long long n, cudaStream_t stream) {
  if (n <= 0) return SP_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SP_ERR_CUDA;
  const long long n4 = n / 4;
  long long blocks = (n4 + 255) / 256;
  const long long cap = (long long)num_sms(dev) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  f32_to_bf16_kernel<<<(int)blocks, 256, 0, stream>>>(reinterpret_cast<const float4*>(in), static_cast<uint2*>(out), n4);
  return cudaGetLastError() == cudaSuccess ? SP_OK : SP_ERR_CUDA;
}

}  // namespace spattn
