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
//                      S'^T = K Q^T - lse / scale and dP'^T = V dO^T - delta (both operands in shared
//                      memory, fp32 in TMEM).  The per-query terms enter as one extra K-step of 16: a
//                      constant left operand with ones in its first three columns times a right operand
//                      holding each query's value split into three bf16 parts (hi + mid + lo carries the
//                      fp32 value to about 2^-24 of it), so the row warps need no per-column loads.
//                      The eight row warps read S' into registers (which frees it for the next tile's
//                      S', computed meanwhile), turn it into P^T = 2^(S' scale log2 e) and, once dP' is
//                      in, dS^T = P^T dP'; both go back as bf16 into the dP' region of TMEM, where
//                      dK += dS^T Q and dV += P^T dO read their left operand.  Q and dO of a ring slot
//                      are released separately (dK runs first), so the next Q copy starts early.
//   bwd_kernel<D, true>   one CTA per (b, h, query tile): the row warps copy the tile's Q and dO rows into
//                      TMEM once, as the left operands of S = Q K^T and dP = dO V^T; key tiles stream
//                      through a three-slot ring, with the same early release of S as above, and
//                      dQ += dS K reads dS from TMEM.
//   Warps: 0 TMA producer, 1 MMA issuer (one elected lane), 2-3 idle, 4-11 the 128 tile rows (one row per
//   thread; the TMEM lane quadrant of warp w is w % 4, and warps w and w + 4 take half of the columns
//   each).  TMEM: S (S') at [0,128), dP (dP') at [128,256), accumulators from 256 (dV then dK, or dQ),
//   and, dQ, the resident Q and dO after its accumulator.
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
constexpr int kRowWarps = 8;       // two per TMEM lane quadrant, 64 columns of a streamed tile each
#ifndef SP_BWD_POLY_PAIRS
#define SP_BWD_POLY_PAIRS 0            // of every 4 pairs of exponentials, this many run on the FMA pipe
#endif
constexpr int kBwdPolyPairs = SP_BWD_POLY_PAIRS;

template <int D, bool kDQ>
struct BCfg {
  static constexpr int kSub = D / 64;
  static constexpr int kTileBytes = kBT * D * 2;
  // dQ keeps its resident Q and dO in TMEM, so its shared memory holds three slots of the K/V ring
  static constexpr int kStages = kDQ ? 3 : 2;
  // dK/dV: the per-query terms of S' and dP' as the right operand of one K-step (128 rows x 16 bf16,
  // 32-byte swizzle), and the constant left operand of that step
  static constexpr int kAugBytes = kBT * 32;
  // dK/dV: resident K and V at [0, 2 tiles), then the constant operand; then per slot the two streamed
  // tiles, and (dK/dV) the lse and delta operands
  static constexpr int kResOff = 0;
  static constexpr int kResBytes = kDQ ? 0 : 2 * kTileBytes;
  static constexpr int kOnesOff = kResBytes;
  static constexpr int kStageOff = kResBytes + (kDQ ? 0 : 1024 * ((kAugBytes + 1023) / 1024));
  static constexpr int kStageBytes = 2 * kTileBytes + (kDQ ? 0 : 2 * kAugBytes);
  static constexpr int kBarOff = kStageOff + kStages * kStageBytes;
  // res_full, full[S], empty[S], st_full[2], p_full[2], acc_full, drain, full_o[S], empty_o[S]
  static constexpr int kNumBars = 1 + 4 * kStages + 6;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  // one CTA per SM: its TMEM allocation takes all 512 columns
  static constexpr int kRaw = kMiscOff + 16 + 1024;
  static constexpr int kSmemBytes = kRaw > 120 * 1024 ? kRaw : 120 * 1024;
  // S, dP over a whole streamed tile; K-major operands
  static constexpr uint32_t kIdescSq = idesc_bf16_f32(128, 128, false, false);
  static constexpr uint32_t kIdescAcc = idesc_bf16_f32(128, D, false, true);  // B operand MN-major
};

struct BwdMaps {
  CUtensorMap q, k, v, dout;
};

struct BwdBars {
  uint32_t res_full, full0, empty0, st_full0, p_full0, acc_full, drain, full_o0, empty_o0;
  // slot s of the streamed ring: dQ, its K and V; dK/dV, its Q and lse operand
  __device__ uint32_t full(int s) const { return full0 + 8u * s; }
  __device__ uint32_t empty(int s) const { return empty0 + 8u * s; }
  // dK/dV: the dO and delta operand of slot s, loaded and released on their own
  __device__ uint32_t full_o(int s) const { return full_o0 + 8u * s; }
  __device__ uint32_t empty_o(int s) const { return empty_o0 + 8u * s; }
  // S (S') computed, dP (dP') computed, S read by every row warp, dS (and P) stored
  __device__ uint32_t s_ready() const { return st_full0; }
  __device__ uint32_t dp_ready() const { return st_full0 + 8u; }
  __device__ uint32_t s_free() const { return p_full0; }
  __device__ uint32_t pds_stored() const { return p_full0 + 8u; }
};

// The row warp of columns [64 j, 64 j + 64) of a streamed tile packs their dS into the 32 columns at 64 j
// of the dP region (and, dK/dV, their P into the 32 after them); K-step kk (16 streamed rows) of the
// accumulating MMA starts at packed column 64 (kk / 4) + 8 (kk % 4) there, or 32 columns further for P.
__device__ __forceinline__ uint32_t packed_col_full(int kk) { return 64u * (kk >> 2) + 8u * (kk & 3); }

// Row r of a 32-byte-swizzled K-major operand of 16 bf16 columns: its 16-byte half holding columns 0-7.
__device__ __forceinline__ uint32_t sw32_first_half(int r) { return 32u * r + 16u * ((r >> 2) & 1); }

// x as hi + mid + lo, each rounded to bf16, packed as the first three bf16 of a 16-byte row half.
__device__ __forceinline__ uint4 bf16_split3(float x) {
  const __nv_bfloat16 hi = __float2bfloat16_rn(x);
  const float r1 = x - __bfloat162float(hi);
  const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
  const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
  return make_uint4((uint32_t)__bfloat16_as_ushort(hi) | ((uint32_t)__bfloat16_as_ushort(mid) << 16),
                    (uint32_t)__bfloat16_as_ushort(lo), 0u, 0u);
}

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
  using C = BCfg<D, kDQ>;
  const int lane = threadIdx.x & 31;
  const uint64_t tmo = p.timeout_ns;
  const CUtensorMap* res0 = kDQ ? &tm.q : &tm.k;     // resident pair
  const CUtensorMap* res1 = kDQ ? &tm.dout : &tm.v;
  const CUtensorMap* str0 = kDQ ? &tm.k : &tm.q;     // streamed pair
  const CUtensorMap* str1 = kDQ ? &tm.v : &tm.dout;
  if (!kDQ && elect_one_sync()) {
    mbar_arrive_expect_tx(bars.res_full, 2 * C::kTileBytes);
#pragma unroll
    for (int c = 0; c < C::kSub; ++c) {
      tma_load_4d(sbase + C::kResOff + c * 16384, res0, bars.res_full, 64 * c, it.h, it.tile * kBT, it.b);
      tma_load_4d(sbase + C::kResOff + C::kTileBytes + c * 16384, res1, bars.res_full, 64 * c, it.h, it.tile * kBT,
                  it.b);
    }
  }
  __syncwarp();
  int issued = 0, issued_o = 0;  // slots whose (Q / K and V) and (dO) copies were started
  bool ok = true;
  for (int n = 0; n < it.n_steps && ok; ++n) {
    const int s = n % C::kStages;
    const int lap = n / C::kStages;
    const int t = it.first + n;
    // dK/dV: the streamed query tile's -lse / scale and -delta (the per-query terms of S' and dP'), read
    // before the wait for the slot so that their latency hides behind it.  Query rows past S (zero-filled
    // Q and dO) get -1e30, so their probabilities are exactly 0, and delta 0.
    float lq[kBT / 32], dq[kBT / 32];
    if (!kDQ) {
      const size_t base = ((size_t)it.b * p.H + it.h) * p.S;
      const float inv_scale = 1.f / p.scale;
#pragma unroll
      for (int j = 0; j < kBT / 32; ++j) {
        const int row = t * kBT + lane + 32 * j;
        lq[j] = row < p.S ? -__ldg(p.lse + base + row) * inv_scale : -1e30f;
        dq[j] = row < p.S ? -__ldg(p.delta + base + row) : 0.f;
      }
    }
    const uint32_t stage = sbase + C::kStageOff + s * C::kStageBytes;
    // Part 0 of the slot (dK/dV: Q with its lse operand; dQ: K), then part 1 (dK/dV: dO with its delta
    // operand; dQ: V), each once its own reader has released it: dK (or dQ) is the last reader of part 0,
    // dV (or dP) of part 1.  dK/dV operand row q: (hi, mid, lo, 0 ...) in its first 16 bytes; the rest
    // stays zero.
    uint8_t* aug = smem + C::kStageOff + s * C::kStageBytes + 2 * C::kTileBytes;
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      const uint32_t full_b = part == 0 ? bars.full(s) : bars.full_o(s);
      if (lap > 0) {
        ok = warp_mbar_wait(part == 0 ? bars.empty(s) : bars.empty_o(s), (lap - 1) & 1, tmo, ERR_TIMEOUT_KV_EMPTY,
                            abort_flag, p.err);
        if (!ok) break;
      }
      if (!kDQ) {
#pragma unroll
        for (int j = 0; j < kBT / 32; ++j)
          *reinterpret_cast<uint4*>(aug + part * C::kAugBytes + sw32_first_half(lane + 32 * j)) =
              bf16_split3(part == 0 ? lq[j] : dq[j]);
        fence_proxy_async_smem();  // the tensor cores read them once the full barrier passes them on
        __syncwarp();
      }
      if (elect_one_sync()) {
        mbar_arrive_expect_tx(full_b, C::kTileBytes);
#pragma unroll
        for (int c = 0; c < C::kSub; ++c)
          tma_load_4d(stage + part * C::kTileBytes + c * 16384, part == 0 ? str0 : str1, full_b, 64 * c, it.h,
                      t * kBT, it.b);
      }
      __syncwarp();
      if (part == 0) issued = n + 1; else issued_o = n + 1;
    }
  }
  if (*abort_flag) {  // no copy may still be landing when the CTA exits: wait (bounded) for the last ones
    if (!kDQ) warp_mbar_wait(bars.res_full, 0, tmo, ERR_TIMEOUT_Q_FULL, nullptr, p.err);
    for (int n = issued > C::kStages ? issued - C::kStages : 0; n < issued; ++n)
      warp_mbar_wait(bars.full(n % C::kStages), (n / C::kStages) & 1, tmo, ERR_TIMEOUT_KV_FULL, nullptr, p.err);
    for (int n = issued_o > C::kStages ? issued_o - C::kStages : 0; n < issued_o; ++n)
      warp_mbar_wait(bars.full_o(n % C::kStages), (n / C::kStages) & 1, tmo, ERR_TIMEOUT_KV_FULL, nullptr, p.err);
  }
}

// ------------------------------------------------------------------------------------------------
// dQ issuer.  Order on the tensor cores: S(0) dP(0) | S(1) dQ(0) dP(1) | S(2) dQ(1) dP(2) | ...
// S = Q K^T and dP = dO V^T take their left operand (Q, dO) from TMEM.  S(n+1) is issued as soon as every
// row warp has read S(n); dQ(n) += dS(n) K(n) waits for dS(n), which the row warps pack into the dP
// region, and dP(n+1) overwrites it only behind dQ(n).  dP(n) frees the slot's V, dQ(n) its K.
template <int D>
__device__ void dq_issue(const BwdParams& p, const BwdItem& it, uint32_t sbase, uint32_t tmem_in, const BwdBars& bars,
                         volatile int* abort_flag) {
  using C = BCfg<D, true>;
  const uint64_t tmo = p.timeout_ns;
  const uint32_t tmem = __shfl_sync(0xffffffffu, tmem_in, 0);
  const uint32_t tS = tmem, tdP = tmem + 128, tAcc = tmem + 256, tQ = tmem + 256 + D, tdO = tQ + D / 2;
  auto stage_of = [&](int n) { return sbase + C::kStageOff + (n % C::kStages) * C::kStageBytes; };
  auto issue_s = [&](int n) {  // S = Q K^T, left operand from TMEM (8 columns per K-step of 16)
    const uint64_t k_k = smem_desc_sw128(stage_of(n), 16, 1024);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t off = (uint64_t)(((kk / 4) * 16384 + (kk % 4) * 32) >> 4);
      mma_ts(tS, tQ + 8 * kk, k_k + off, C::kIdescSq, kk > 0 ? 1u : 0u);
    }
    mma_commit(bars.s_ready());
  };
  auto issue_dp = [&](int n) {  // dP = dO V^T; then the slot's V is free
    const uint64_t v_k = smem_desc_sw128(stage_of(n) + C::kTileBytes, 16, 1024);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t off = (uint64_t)(((kk / 4) * 16384 + (kk % 4) * 32) >> 4);
      mma_ts(tdP, tdO + 8 * kk, v_k + off, C::kIdescSq, kk > 0 ? 1u : 0u);
    }
    mma_commit(bars.dp_ready());
    mma_commit(bars.empty_o(n % C::kStages));
  };
  // the row warps have put Q and dO (bf16 pairs) into TMEM
  bool ok = warp_mbar_wait(bars.res_full, 0, tmo, ERR_TIMEOUT_Q_FULL, abort_flag, p.err);
  const int N = it.n_steps;
  if (ok && N > 0) {
    ok = warp_mbar_wait(bars.full(0), 0, tmo, ERR_TIMEOUT_KV_FULL, abort_flag, p.err);
    if (ok) ok = warp_mbar_wait(bars.full_o(0), 0, tmo, ERR_TIMEOUT_KV_FULL, abort_flag, p.err);
    if (ok) {
      tc_fence_after();
      if (elect_one_sync()) {
        issue_s(0);
        issue_dp(0);
      }
      __syncwarp();
    }
  }
  for (int n = 0; n < N && ok; ++n) {
    if (n + 1 < N) {
      ok = warp_mbar_wait(bars.s_free(), n & 1, tmo, ERR_TIMEOUT_P_FULL, abort_flag, p.err);
      if (ok)
        ok = warp_mbar_wait(bars.full((n + 1) % C::kStages), ((n + 1) / C::kStages) & 1, tmo, ERR_TIMEOUT_KV_FULL,
                            abort_flag, p.err);
      if (!ok) break;
      tc_fence_after();
      if (elect_one_sync()) issue_s(n + 1);
      __syncwarp();
    }
    ok = warp_mbar_wait(bars.pds_stored(), n & 1, tmo, ERR_TIMEOUT_P_FULL, abort_flag, p.err);
    if (!ok) break;
    tc_fence_after();
    if (elect_one_sync()) {  // dQ += dS K (K-steps of 16 keys: MN-major K, 2048 bytes apart)
      const uint64_t k_mn = smem_desc_sw128(stage_of(n), 16384, 1024);
#pragma unroll
      for (int kk = 0; kk < kBT / 16; ++kk)
        mma_ts(tAcc, tdP + packed_col_full(kk), k_mn + (uint64_t)(kk * 128), C::kIdescAcc,
               (n == 0 && kk == 0) ? 0u : 1u);
      mma_commit(bars.empty(n % C::kStages));
    }
    __syncwarp();
    if (n + 1 < N) {
      ok = warp_mbar_wait(bars.full_o((n + 1) % C::kStages), ((n + 1) / C::kStages) & 1, tmo, ERR_TIMEOUT_KV_FULL,
                          abort_flag, p.err);
      if (!ok) break;
      tc_fence_after();
      if (elect_one_sync()) issue_dp(n + 1);
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

// dK/dV issuer.  Order on the tensor cores: S'(0) dP'(0) | S'(1) dK(0) dV(0) dP'(1) | S'(2) dK(1) ...
// S'(n+1) is issued as soon as every row warp has read S'(n) into registers, so it runs while they
// compute P(n); dK(n) and dV(n) wait for P(n) and dS(n), which the row warps pack into the dP' region;
// dP'(n+1) overwrites them only behind dV(n) (tcgen05 MMAs of one thread run in order).  dK(n) frees
// the slot's Q, then dV(n) its dO.
template <int D>
__device__ void dkdv_issue(const BwdParams& p, const BwdItem& it, uint32_t sbase, uint32_t tmem_in,
                           const BwdBars& bars, volatile int* abort_flag) {
  using C = BCfg<D, false>;
  const uint64_t tmo = p.timeout_ns;
  const uint32_t tmem = __shfl_sync(0xffffffffu, tmem_in, 0);
  const uint32_t tS = tmem, tdP = tmem + 128, tdV = tmem + 256, tdK = tmem + 256 + D;
  const uint64_t k_k = smem_desc_sw128(sbase + C::kResOff, 16, 1024);
  const uint64_t v_k = smem_desc_sw128(sbase + C::kResOff + C::kTileBytes, 16, 1024);
  const uint64_t ones = smem_desc_sw32(sbase + C::kOnesOff, 256);
  auto stage_of = [&](int n) { return sbase + C::kStageOff + (n % C::kStages) * C::kStageBytes; };
  // S'^T = K Q^T + ones lq^T (lq: -lse / scale in three parts), into TMEM [0, 128)
  auto issue_s = [&](int n) {
    const uint32_t st = stage_of(n);
    const uint64_t q_k = smem_desc_sw128(st, 16, 1024);
    mma_ss(tS, ones, smem_desc_sw32(st + 2 * C::kTileBytes, 256), C::kIdescSq, 0u);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t off = (uint64_t)(((kk / 4) * 16384 + (kk % 4) * 32) >> 4);
      mma_ss(tS, k_k + off, q_k + off, C::kIdescSq, 1u);
    }
    mma_commit(bars.s_ready());
  };
  // dP'^T = V dO^T + ones dl^T (dl: -delta in three parts), into TMEM [128, 256)
  auto issue_dp = [&](int n) {
    const uint32_t st = stage_of(n);
    const uint64_t do_k = smem_desc_sw128(st + C::kTileBytes, 16, 1024);
    mma_ss(tdP, ones, smem_desc_sw32(st + 2 * C::kTileBytes + C::kAugBytes, 256), C::kIdescSq, 0u);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t off = (uint64_t)(((kk / 4) * 16384 + (kk % 4) * 32) >> 4);
      mma_ss(tdP, v_k + off, do_k + off, C::kIdescSq, 1u);
    }
    mma_commit(bars.dp_ready());
  };
  bool ok = warp_mbar_wait(bars.res_full, 0, tmo, ERR_TIMEOUT_Q_FULL, abort_flag, p.err);
  const int N = it.n_steps;
  if (ok && N > 0) {
    ok = warp_mbar_wait(bars.full(0), 0, tmo, ERR_TIMEOUT_KV_FULL, abort_flag, p.err);
    if (ok) ok = warp_mbar_wait(bars.full_o(0), 0, tmo, ERR_TIMEOUT_KV_FULL, abort_flag, p.err);
    if (ok) {
      tc_fence_after();
      if (elect_one_sync()) {
        issue_s(0);
        issue_dp(0);
      }
      __syncwarp();
    }
  }
  for (int n = 0; n < N && ok; ++n) {
    const uint32_t st = stage_of(n);
    // K-steps of 16 queries: MN-major right operands, 2048 bytes apart
    const uint64_t q_mn = smem_desc_sw128(st, 16384, 1024);
    const uint64_t do_mn = smem_desc_sw128(st + C::kTileBytes, 16384, 1024);
    if (n + 1 < N) {
      ok = warp_mbar_wait(bars.s_free(), n & 1, tmo, ERR_TIMEOUT_P_FULL, abort_flag, p.err);
      if (ok)
        ok = warp_mbar_wait(bars.full((n + 1) % C::kStages), ((n + 1) / C::kStages) & 1, tmo, ERR_TIMEOUT_KV_FULL,
                            abort_flag, p.err);
      if (!ok) break;
      tc_fence_after();
      if (elect_one_sync()) issue_s(n + 1);
      __syncwarp();
    }
    ok = warp_mbar_wait(bars.pds_stored(), n & 1, tmo, ERR_TIMEOUT_P_FULL, abort_flag, p.err);
    if (!ok) break;
    tc_fence_after();
    if (elect_one_sync()) {
      // dK += dS^T Q, then the slot's Q is free; dV += P^T dO, then its dO
#pragma unroll
      for (int kk = 0; kk < kBT / 16; ++kk)
        mma_ts(tdK, tdP + packed_col_full(kk), q_mn + (uint64_t)(kk * 128), C::kIdescAcc, (n == 0 && kk == 0) ? 0u : 1u);
      mma_commit(bars.empty(n % C::kStages));
#pragma unroll
      for (int kk = 0; kk < kBT / 16; ++kk)
        mma_ts(tdV, tdP + 32 + packed_col_full(kk), do_mn + (uint64_t)(kk * 128), C::kIdescAcc,
               (n == 0 && kk == 0) ? 0u : 1u);
      mma_commit(bars.empty_o(n % C::kStages));
    }
    __syncwarp();
    if (n + 1 < N) {
      ok = warp_mbar_wait(bars.full_o((n + 1) % C::kStages), ((n + 1) / C::kStages) & 1, tmo, ERR_TIMEOUT_KV_FULL,
                          abort_flag, p.err);
      if (!ok) break;
      tc_fence_after();
      if (elect_one_sync()) issue_dp(n + 1);
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
// Epilogue of the accumulators: this warp's half of the D columns of each, scaled, to bf16 (or added into
// the fp32 dQ accumulator).
template <int D, bool kDQ>
__device__ __forceinline__ void bwd_epilogue(const BwdParams& p, const BwdItem& it, uint32_t trow, int j, int row,
                                             bool row_out) {
  const uint32_t tAcc0 = trow + 256, tAcc1 = trow + 256 + D;
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

// dQ rows: P = 2^(S scale log2 e - lse log2 e) of 64 keys from this query row's -lse (log2 units); keys
// c >= hi get 0 (kMask).  Of every 4 pairs of exponentials, kBwdPolyPairs run through the FMA-pipe
// polynomial, the rest through ex2.approx.
template <bool kMask>
__device__ __forceinline__ void dq_p(const uint32_t (&s)[64], float (&pf)[64], f2 sc, f2 nl, int hi) {
#pragma unroll
  for (int i = 0; i < 64; i += 2) {
    const f2 x = ffma2(f2{__uint_as_float(s[i]), __uint_as_float(s[i + 1])}, sc, nl);
    f2 pv;
    if (((i >> 1) & 3) >= 4 - kBwdPolyPairs) {
      pv = exp2_poly2(x);
    } else {
      pv.x = ex2_approx(x.x);
      pv.y = ex2_approx(x.y);
    }
    if (kMask) {
      if (i >= hi) pv.x = 0.f;
      if (i + 1 >= hi) pv.y = 0.f;
    }
    pf[i] = pv.x;
    pf[i + 1] = pv.y;
  }
}

// dQ rows: this thread is query `row`; warp j takes keys [64 j, 64 j + 64) of each key tile.
template <int D>
__device__ void dq_rows(const BwdParams& p, const BwdItem& it, uint32_t tmem, const BwdBars& bars,
                        volatile int* abort_flag) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quad = warp & 3;
  const int j = (warp - kWarpRow0) >> 2;
  const int r = quad * 32 + lane;
  const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
  const uint32_t tS = trow + 64u * j, tdP = trow + 128u + 64u * j;
  const uint64_t tmo = p.timeout_ns;
  const f2 sc = {p.scale_log2, p.scale_log2};
  const int row = it.tile * kBT + r;                             // this thread's query
  const int kv_lim = min(p.kv_end, p.S);
  const bool row_out = row < p.S;
  float nlse2_row = 0.f, ndlt_row = 0.f;  // -lse (log2 units) and -delta of this thread's query
  if (row < p.S) {
    const size_t i = ((size_t)it.b * p.H + it.h) * p.S + row;
    nlse2_row = __ldg(p.lse + i) * -1.4426950408889634f;
    ndlt_row = -__ldg(p.delta + i);
  }
  {
    // this thread's query row of Q and dO, half j of the D columns, into TMEM (zeros past S): the left
    // operands of S and dP for every key tile
    const uint32_t tQ = trow + 256 + D + (D / 4) * j, tdO = tQ + D / 2;
    const size_t src = (((size_t)it.b * p.S + row) * p.H + it.h) * D + (D / 2) * j;
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const uint4* g = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(which ? p.dout : p.q) + src);
      uint32_t v[D / 4];
#pragma unroll
      for (int e = 0; e < D / 16; ++e) {
        const uint4 x = row < p.S ? __ldg(g + e) : make_uint4(0u, 0u, 0u, 0u);
        v[4 * e] = x.x; v[4 * e + 1] = x.y; v[4 * e + 2] = x.z; v[4 * e + 3] = x.w;
      }
      if (D == 128)
        tmem_st32(which ? tdO : tQ, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
      else
        tmem_st16(which ? tdO : tQ, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bars.res_full);
  }
  const f2 nl = {nlse2_row, nlse2_row}, nd = {ndlt_row, ndlt_row};
  bool ok = true;
  for (int n = 0; n < it.n_steps; ++n) {
    const int t = it.first + n;
    ok = __all_sync(0xffffffffu, mbar_wait(bars.s_ready(), n & 1, tmo, ERR_TIMEOUT_S_FULL, abort_flag, p.err));
    if (!ok) break;
    tc_fence_after();
    float pf[64];
    {
      uint32_t s[64];
      tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.s_free());
      // kept: keys t kBT + 64 j + i not after the query (causal) and inside the key range
      const int hi = min(p.causal ? row - t * kBT + 1 : INT_MAX, kv_lim - t * kBT) - 64 * j;
      if (hi < 64)
        dq_p<true>(s, pf, sc, nl, hi);
      else
        dq_p<false>(s, pf, sc, nl, hi);
    }
    // dS = P (dP - delta) in two chunks of 32 keys, packed over columns already read
    ok = __all_sync(0xffffffffu, mbar_wait(bars.dp_ready(), n & 1, tmo, ERR_TIMEOUT_S_FULL, abort_flag, p.err));
    if (!ok) break;
    tc_fence_after();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t d[32], pk[16];
      tmem_ld32(tdP + 32 * h, d);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const f2 ds = fmul2(f2{pf[32 * h + i], pf[32 * h + i + 1]},
                            fadd2(f2{__uint_as_float(d[i]), __uint_as_float(d[i + 1])}, nd));
        pk[i >> 1] = pack_bf16x2(ds.x, ds.y);
      }
      tmem_st16(tdP + 16 * h, pk);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bars.pds_stored());
  }
  if (!ok) return;
  ok = __all_sync(0xffffffffu, mbar_wait(bars.acc_full, 0, tmo, ERR_TIMEOUT_PV_DONE, abort_flag, p.err));
  if (!ok) return;
  if (it.n_steps == 0) return;  // (a key range before this query tile) nothing accumulated
  tc_fence_after();
  bwd_epilogue<D, true>(p, it, trow, j, row, row_out);
}

// P = 2^(S' scale log2 e) of 64 queries; kMask: queries i < lo get 0.  Of every 4 pairs of exponentials,
// kBwdPolyPairs run through the FMA-pipe polynomial, the rest through ex2.approx.
template <bool kMask>
__device__ __forceinline__ void dkdv_p(const uint32_t (&s)[64], float (&pf)[64], f2 sc, int lo) {
#pragma unroll
  for (int i = 0; i < 64; i += 2) {
    const f2 x = fmul2(f2{__uint_as_float(s[i]), __uint_as_float(s[i + 1])}, sc);
    f2 pv;
    if (((i >> 1) & 3) >= 4 - kBwdPolyPairs) {
      pv = exp2_poly2(x);
    } else {
      pv.x = ex2_approx(x.x);
      pv.y = ex2_approx(x.y);
    }
    if (kMask) {
      if (i < lo) pv.x = 0.f;
      if (i + 1 < lo) pv.y = 0.f;
    }
    pf[i] = pv.x;
    pf[i + 1] = pv.y;
  }
}

// dK/dV rows: this thread is key `row`; warp j takes queries [64 j, 64 j + 64) of each query tile.
template <int D>
__device__ void dkdv_rows(const BwdParams& p, const BwdItem& it, uint32_t tmem, const BwdBars& bars,
                          volatile int* abort_flag) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quad = warp & 3;
  const int j = (warp - kWarpRow0) >> 2;
  const int r = quad * 32 + lane;
  const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
  const uint32_t tS = trow + 64u * j, tdP = trow + 128u + 64u * j;
  const uint64_t tmo = p.timeout_ns;
  const f2 sc = {p.scale_log2, p.scale_log2};
  const int row = it.tile * kBT + r;
  const bool row_out = row < min(p.kv_end, p.S);
  bool ok = true;
  for (int n = 0; n < it.n_steps; ++n) {
    const int t = it.first + n;
    ok = __all_sync(0xffffffffu, mbar_wait(bars.s_ready(), n & 1, tmo, ERR_TIMEOUT_S_FULL, abort_flag, p.err));
    if (!ok) break;
    tc_fence_after();
    // P = 2^(S' scale log2 e) over this warp's 64 queries; causal: queries before the key get 0.  S' is
    // released to the next tile's MMA as soon as it is in registers.
    float pf[64];
    {
      uint32_t s[64];
      tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.s_free());
      const int lo = p.causal ? row - t * kBT - 64 * j : INT_MIN;  // kept: this warp's query i >= lo
      if (lo > 0)
        dkdv_p<true>(s, pf, sc, lo);
      else
        dkdv_p<false>(s, pf, sc, lo);
    }
    // dS = P dP' in two chunks of 32 queries, packed over columns already read; then P after them
    ok = __all_sync(0xffffffffu, mbar_wait(bars.dp_ready(), n & 1, tmo, ERR_TIMEOUT_S_FULL, abort_flag, p.err));
    if (!ok) break;
    tc_fence_after();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t d[32], pk[16];
      tmem_ld32(tdP + 32 * h, d);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const f2 ds = fmul2(f2{pf[32 * h + i], pf[32 * h + i + 1]}, f2{__uint_as_float(d[i]), __uint_as_float(d[i + 1])});
        pk[i >> 1] = pack_bf16x2(ds.x, ds.y);
      }
      tmem_st16(tdP + 16 * h, pk);
    }
    {
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 64; i += 2) pk[i >> 1] = pack_bf16x2(pf[i], pf[i + 1]);
      tmem_st32(tdP + 32, pk);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bars.pds_stored());
  }
  if (!ok) return;
  ok = __all_sync(0xffffffffu, mbar_wait(bars.acc_full, 0, tmo, ERR_TIMEOUT_PV_DONE, abort_flag, p.err));
  if (!ok) return;
  tc_fence_after();
  bwd_epilogue<D, false>(p, it, trow, j, row, row_out);
}

template <int D, bool kDQ>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_kernel(const __grid_constant__ BwdMaps tm, const __grid_constant__ BwdParams p) {
  using C = BCfg<D, kDQ>;
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
  bars.full_o0 = bars.drain + 8;
  bars.empty_o0 = bars.full_o0 + 8 * C::kStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(bars.res_full, kDQ ? kRowWarps : 1);  // dQ: every row warp's Q and dO in TMEM
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bars.full(s), 1);
      mbar_init(bars.empty(s), 1);
      mbar_init(bars.full_o(s), 1);
      mbar_init(bars.empty_o(s), 1);
    }
    mbar_init(bars.s_ready(), 1);
    mbar_init(bars.dp_ready(), 1);
    mbar_init(bars.s_free(), kRowWarps);  // one arrival per row warp
    mbar_init(bars.pds_stored(), kRowWarps);
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
  if (!kDQ) {
    // the constant operand (rows 1, 1, 1, 0 ...), and zeros in the per-query operands of both slots (the
    // producer rewrites only the first three columns of each row)
    for (int i = threadIdx.x; i < kBT * 2; i += kBwdThreads) {
      const int r = i >> 1, half = i & 1;
      const uint32_t at = sw32_first_half(r) ^ (half ? 16u : 0u);
      *reinterpret_cast<uint4*>(smem + C::kOnesOff + at) =
          half ? make_uint4(0u, 0u, 0u, 0u) : make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u);
    }
    for (int i = threadIdx.x; i < C::kStages * 2 * C::kAugBytes / 16; i += kBwdThreads) {
      const int s = i / (2 * C::kAugBytes / 16), rem = i % (2 * C::kAugBytes / 16);
      *reinterpret_cast<uint4*>(smem + C::kStageOff + s * C::kStageBytes + 2 * C::kTileBytes + 16 * rem) =
          make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const BwdItem it = bwd_item<kDQ>(p);
  if (warp == kWarpLoad) {
    bwd_load<D, kDQ>(p, tm, it, sbase, smem, bars, abort_flag);
  } else if (warp == kWarpIssue) {
    if (kDQ)
      dq_issue<D>(p, it, sbase, tmem, bars, abort_flag);
    else
      dkdv_issue<D>(p, it, sbase, tmem, bars, abort_flag);
  } else if (warp >= kWarpRow0) {
    if (kDQ)
      dq_rows<D>(p, it, tmem, bars, abort_flag);
    else
      dkdv_rows<D>(p, it, tmem, bars, abort_flag);
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
  using C = BCfg<D, kDQ>;
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
  p.q = q;
  p.dout = dout;
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
