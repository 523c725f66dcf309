// attn_fwd.cu -- exact multi-head attention forward on the 5th-generation tensor cores (sm_100a).
//
// What it computes: for every (batch b, head h, query i), over the keys j it may see,
//   o = sum_j softmax_j(q_i . k_j / sqrt(D)) v_j,   lse = ln sum_j exp(q_i . k_j / sqrt(D))
// ("LLM Lab Notes 05: Attention Tensor Parallelism", section 2 step 4: per head q @ k^T / sqrt(d),
// softmax, @ v).  The visible keys are those in [kv_begin, kv_end) (one Ring-Attention KV block, "CHARM+:
// How Cross-Hardware Attention Breaks Through ...", Ring-Attention paragraph), j <= i when causal, and
// only 128 x 128 tiles kept by a per-head block mask when one is given ("db-SP", abstract).
//
// How (one persistent CTA per SM, each taking work items in turn):
//   work item = (b, h, pair of 128-row query tiles).  The two query tiles are the two "lanes" of the
//   CTA; they share every K/V tile that both need.
//   warp 8      TMA producer: Q tiles of both lanes, then K_j, V_j tiles into a ring of shared-memory
//               slots (128B-swizzled, the tensor cores' canonical layout).
//   warp 9      MMA issuer (one thread): S_t = Q_t K_j^T into TMEM (fp32), and O_t += P_t V_j with P_t
//               read from TMEM and V_j from shared memory; tcgen05.commit signals completions.
//   warps 0-7   softmax, 4 warps per lane: thread r owns query row r of its lane's tile, loads its row
//               of S from TMEM (so every row reduction stays inside one thread), keeps the running
//               maximum m and sum l, writes P = exp(S - m) as bf16 back into TMEM over S, rescales
//               the O row in TMEM when the maximum grows by more than 2^8, and finally writes
//               O / l and lse = (m + log2 l) ln 2.
//   TMEM (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256, 256+D), O_1 [256+D, 256+2D); P_t
//   overwrites the first 64 columns of S_t.
// Every barrier wait is bounded in time; on expiry the kernel records an error and returns cleanly.
#include <climits>
#include <cstdint>

#include "sp_internal.h"
#include "sp_ptx.cuh"

namespace spattn {

namespace {

constexpr int kTile = 128;
constexpr int kThreads = 320;
constexpr int kWarpProducer = 8;
constexpr int kWarpMma = 9;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: O and l are rescaled when m grows by > 2^8

template <int D>
struct Cfg {
  static constexpr int kSub = D / 64;                   // 64-column (128-byte) sub-tiles per row
  static constexpr int kTileBytes = kTile * D * 2;      // one 128 x D bf16 tile
  static constexpr int kStages = D == 128 ? 4 : 8;      // K/V ring slots
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  static constexpr int kBarOff = kKVOff + kStages * kTileBytes;
  // barriers: q_full, q_empty, kv_full[S], kv_empty[S], s_full[2], p_full[2], pv_done[2], drain, and
  // two 8-byte slots for the o_done counters
  static constexpr int kNumBars = 2 + 2 * kStages + 9;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscOff + 16 + 1024;  // + alignment slack
  static constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false, false);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, false, true);
  static constexpr uint32_t kColS = 0;
  static constexpr uint32_t kColO = 256;
};

struct Bars {
  uint32_t q_full, q_empty, kv_full0, kv_empty0, s_full0, p_full0, pv_done0, o_done0, drain;
  __device__ uint32_t kv_full(int s) const { return kv_full0 + 8u * s; }
  __device__ uint32_t kv_empty(int s) const { return kv_empty0 + 8u * s; }
  __device__ uint32_t s_full(int t) const { return s_full0 + 8u * t; }
  __device__ uint32_t p_full(int t) const { return p_full0 + 8u * t; }
  __device__ uint32_t pv_done(int t) const { return pv_done0 + 8u * t; }
  // o_done[t]: a counter, +1 per softmax warp of lane t per finished item (epilogue reads of O done)
  __device__ uint32_t o_done(int t) const { return o_done0 + 8u * t; }
};

struct Item {
  int b, h, qp;
  int q_start[2];
  int q_last[2];
  bool valid[2];
};

__device__ __forceinline__ Item decode_item(const AttnParams& p, int w) {
  // Items are ordered by head chunk, then batch, then head, then query-tile pair (heaviest first when
  // causal, so that the round-robin assignment to CTAs interleaves long and short items).
  int c = 0;
  while (c + 1 < p.n_chunks && w >= p.chunk_item0[c + 1]) ++c;
  const int r = w - p.chunk_item0[c];
  const int hc = p.chunk_h0[c + 1] - p.chunk_h0[c];
  const int per_b = hc * p.n_qpairs;
  Item it;
  it.b = r / per_b;
  const int r2 = r - it.b * per_b;
  it.h = p.chunk_h0[c] + r2 / p.n_qpairs;
  const int qq = r2 % p.n_qpairs;
  it.qp = p.causal ? (p.n_qpairs - 1 - qq) : qq;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    it.q_start[t] = (2 * it.qp + t) * kTile;
    it.valid[t] = it.q_start[t] < p.S;
    it.q_last[t] = min(p.S, it.q_start[t] + kTile) - 1;
  }
  return it;
}

// Walks the key tiles a work item needs, in increasing key order, with which lanes need each.
struct StepIter {
  bool sparse, causal;
  int kv_begin;
  int q_last0, q_last1;
  bool v0, v1;
  int j, n_dense;
  const int* l0;
  const int* l1;
  int i0, e0, i1, e1, c0, c1;

  __device__ __forceinline__ static int lower_bound(const int* a, int lo, int hi, int x) {
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(a + mid) < x) lo = mid + 1; else hi = mid;
    }
    return lo;
  }

  __device__ __forceinline__ void init(const AttnParams& p, const Item& it) {
    causal = p.causal != 0;
    kv_begin = p.kv_begin;
    q_last0 = it.q_last[0];
    q_last1 = it.q_last[1];
    v0 = it.valid[0];
    v1 = it.valid[1];
    sparse = p.row_ptr != nullptr;
    j = 0;
    if (!sparse) {
      n_dense = 0;
      if (v0 || v1) {
        n_dense = p.n_kv_tiles;
        if (causal) {
          const int ql = v1 ? q_last1 : q_last0;
          n_dense = ql < p.kv_begin ? 0 : min(p.n_kv_tiles, (ql - p.kv_begin) / kTile + 1);
        }
      }
      return;
    }
    // Tile range allowed by [kv_begin, kv_lim): kv_begin is a multiple of 128 here.
    const int t_lo = p.kv_begin / kTile;
    const int t_hi = (p.kv_lim + kTile - 1) / kTile;  // exclusive
    l0 = p.col_idx;
    l1 = p.col_idx;
    const int row0 = it.h * p.mask_T + 2 * it.qp;
    i0 = e0 = i1 = e1 = 0;
    if (v0) {
      i0 = __ldg(p.row_ptr + row0);
      e0 = __ldg(p.row_ptr + row0 + 1);
      const int hi0 = causal ? min(t_hi, q_last0 / kTile + 1) : t_hi;
      if (t_lo > 0) i0 = lower_bound(l0, i0, e0, t_lo);
      if (hi0 < p.mask_T) e0 = lower_bound(l0, i0, e0, hi0);
    }
    if (v1) {
      i1 = __ldg(p.row_ptr + row0 + 1);
      e1 = __ldg(p.row_ptr + row0 + 2);
      const int hi1 = causal ? min(t_hi, q_last1 / kTile + 1) : t_hi;
      if (t_lo > 0) i1 = lower_bound(l1, i1, e1, t_lo);
      if (hi1 < p.mask_T) e1 = lower_bound(l1, i1, e1, hi1);
    }
    c0 = i0 < e0 ? __ldg(l0 + i0) : INT_MAX;
    c1 = i1 < e1 ? __ldg(l1 + i1) : INT_MAX;
  }

  __device__ __forceinline__ bool next(int& kv_start, bool& k0, bool& k1) {
    if (!sparse) {
      if (j >= n_dense) return false;
      kv_start = kv_begin + j * kTile;
      ++j;
      k0 = v0 && (!causal || kv_start <= q_last0);
      k1 = v1 && (!causal || kv_start <= q_last1);
      return true;
    }
    const int t = min(c0, c1);
    if (t == INT_MAX) return false;
    k0 = c0 == t;
    k1 = c1 == t;
    if (k0) { ++i0; c0 = i0 < e0 ? __ldg(l0 + i0) : INT_MAX; }
    if (k1) { ++i1; c1 = i1 < e1 ? __ldg(l1 + i1) : INT_MAX; }
    kv_start = t * kTile;
    return true;
  }
};

// ------------------------------------------------------------------------------------------------
// Producer: one thread issues all TMA loads.
// ------------------------------------------------------------------------------------------------
template <int D>
__device__ void run_producer(const AttnParams& p, const CUtensorMap* tq, const CUtensorMap* tk,
                             const CUtensorMap* tv, uint8_t* smem, const Bars& bars,
                             volatile int* abort_flag) {
  using C = Cfg<D>;
  const uint32_t sbase = smem_u32(smem);
  uint32_t q_empty_ph = 0;
  int ring = 0;
  int n_item = 0;
  int last_q_item = -1;
  bool ok = true;
  for (int w = blockIdx.x; w < p.n_items && ok; w += gridDim.x, ++n_item) {
    const Item it = decode_item(p, w);
    if (n_item > 0) {
      ok = mbar_wait(bars.q_empty, q_empty_ph, p.timeout_ns, ERR_TIMEOUT_Q_EMPTY, abort_flag, p.err);
      q_empty_ph ^= 1;
      if (!ok) break;
    }
    mbar_arrive_expect_tx(bars.q_full, 2 * C::kTileBytes);
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int c = 0; c < C::kSub; ++c)
        tma_load_4d(sbase + C::kQOff + t * C::kTileBytes + c * 16384, tq, bars.q_full, 64 * c, it.h,
                    it.q_start[t], it.b);
    last_q_item = n_item;
    StepIter st;
    st.init(p, it);
    int kv_start;
    bool k0, k1;
    while (st.next(kv_start, k0, k1)) {
#pragma unroll
      for (int kv = 0; kv < 2; ++kv) {
        const int slot = ring % C::kStages;
        const int lap = ring / C::kStages;
        if (lap > 0) {
          ok = mbar_wait(bars.kv_empty(slot), (lap - 1) & 1, p.timeout_ns, ERR_TIMEOUT_KV_EMPTY, abort_flag, p.err);
          if (!ok) break;
        }
        mbar_arrive_expect_tx(bars.kv_full(slot), C::kTileBytes);
        const CUtensorMap* tm = kv == 0 ? tk : tv;
#pragma unroll
        for (int c = 0; c < C::kSub; ++c)
          tma_load_4d(sbase + C::kKVOff + slot * C::kTileBytes + c * 16384, tm, bars.kv_full(slot), 64 * c,
                      it.h, kv_start, it.b);
        ++ring;
      }
      if (!ok) break;
    }
  }
  if (*abort_flag) {
    // Do not leave copies in flight into shared memory: wait (bounded) for the most recent load of
    // every slot and for the last Q load.
    const uint64_t tmo = p.timeout_ns;
    for (int pos = max(0, ring - C::kStages); pos < ring; ++pos)
      mbar_wait(bars.kv_full(pos % C::kStages), (pos / C::kStages) & 1, tmo, ERR_TIMEOUT_KV_FULL, nullptr, p.err);
    if (last_q_item >= 0) mbar_wait(bars.q_full, last_q_item & 1, tmo, ERR_TIMEOUT_Q_FULL, nullptr, p.err);
  }
}

// ------------------------------------------------------------------------------------------------
// MMA issuer: one thread.
// ------------------------------------------------------------------------------------------------
template <int D>
__device__ void run_mma(const AttnParams& p, uint8_t* smem, const Bars& bars, uint32_t tmem,
                        volatile int* abort_flag) {
  using C = Cfg<D>;
  const uint32_t sbase = smem_u32(smem);
  const uint64_t tmo = p.timeout_ns;
  uint32_t q_full_ph = 0;
  uint32_t p_full_ph[2] = {0, 0}, pv_done_ph[2] = {0, 0};
  bool pv_pending[2] = {false, false};
  int ring = 0;
  int n_item = 0;
  bool ok = true;
  for (int w = blockIdx.x; w < p.n_items && ok; w += gridDim.x, ++n_item) {
    const Item it = decode_item(p, w);
    ok = mbar_wait(bars.q_full, q_full_ph, tmo, ERR_TIMEOUT_Q_FULL, abort_flag, p.err);
    q_full_ph ^= 1;
    if (!ok) break;
    tc_fence_after();
    // O_t may be overwritten by this item's first P V only after the 4 softmax warps of lane t have
    // read out the previous item's O: o_done[t] counts 4 per finished item.
    bool need_odone[2] = {n_item > 0, n_item > 0};
    bool first_pv[2] = {true, true};
    StepIter st;
    st.init(p, it);
    bool prev_has = false, prev_keep[2] = {false, false};
    int prev_v_pos = 0;
    bool prev_v_waited = false;
    for (;;) {
      int kv_start;
      bool keep[2];
      const bool has = st.next(kv_start, keep[0], keep[1]);
      const int k_pos = ring;
      bool k_waited = false;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (prev_has && prev_keep[t]) {
          if (!prev_v_waited) {
            ok = mbar_wait(bars.kv_full(prev_v_pos % C::kStages), (prev_v_pos / C::kStages) & 1, tmo,
                           ERR_TIMEOUT_KV_FULL, abort_flag, p.err);
            if (!ok) break;
            prev_v_waited = true;
          }
          if (need_odone[t]) {
            ok = counter_wait(bars.o_done(t), 4u * (uint32_t)n_item, tmo, ERR_TIMEOUT_O_FREE, abort_flag, p.err);
            need_odone[t] = false;
            if (!ok) break;
          }
          ok = mbar_wait(bars.p_full(t), p_full_ph[t], tmo, ERR_TIMEOUT_P_FULL, abort_flag, p.err);
          p_full_ph[t] ^= 1;
          if (!ok) break;
          tc_fence_after();
          const uint32_t v_addr = sbase + C::kKVOff + (prev_v_pos % C::kStages) * C::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk) {
            const uint64_t bdesc = smem_desc_sw128(v_addr + kk * 2048, 16384, 1024);
            mma_ts(tmem + C::kColO + t * D, tmem + C::kColS + t * 128 + kk * 8, bdesc, C::kIdescPV,
                   (first_pv[t] && kk == 0) ? 0u : 1u);
          }
          first_pv[t] = false;
          mma_commit(bars.pv_done(t));
          pv_pending[t] = true;
        }
        if (has && keep[t]) {
          if (!k_waited) {
            ok = mbar_wait(bars.kv_full(k_pos % C::kStages), (k_pos / C::kStages) & 1, tmo,
                           ERR_TIMEOUT_KV_FULL, abort_flag, p.err);
            if (!ok) break;
            k_waited = true;
            tc_fence_after();
          }
          if (pv_pending[t]) {
            ok = mbar_wait(bars.pv_done(t), pv_done_ph[t], tmo, ERR_TIMEOUT_PV_DONE, abort_flag, p.err);
            pv_done_ph[t] ^= 1;
            pv_pending[t] = false;
            if (!ok) break;
            tc_fence_after();
          }
          const uint32_t q_addr = sbase + C::kQOff + t * C::kTileBytes;
          const uint32_t k_addr = sbase + C::kKVOff + (k_pos % C::kStages) * C::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk / 4) * 16384 + (kk % 4) * 32;
            const uint64_t adesc = smem_desc_sw128(q_addr + off, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(k_addr + off, 16, 1024);
            mma_ss(tmem + C::kColS + t * 128, adesc, bdesc, C::kIdescS, kk > 0 ? 1u : 0u);
          }
          mma_commit(bars.s_full(t));
        }
      }
      if (!ok) break;
      if (prev_has) mma_commit(bars.kv_empty(prev_v_pos % C::kStages));
      if (!has) break;
      mma_commit(bars.kv_empty(k_pos % C::kStages));
      ring += 2;
      prev_has = true;
      prev_keep[0] = keep[0];
      prev_keep[1] = keep[1];
      prev_v_pos = k_pos + 1;
      prev_v_waited = false;
    }
    if (!ok) break;
    mma_commit(bars.q_empty);  // every S MMA that read this item's Q tiles has been issued
  }
  // Drain: nothing of ours may still run on the tensor cores when TMEM is released.
  mma_commit(bars.drain);
  mbar_wait(bars.drain, 0, tmo, ERR_TIMEOUT_DRAIN, nullptr, p.err);
}

// ------------------------------------------------------------------------------------------------
// Softmax + epilogue: 4 warps per lane, one query row per thread.
// ------------------------------------------------------------------------------------------------
template <int D>
__device__ void run_softmax(const AttnParams& p, const Bars& bars, uint32_t tmem, int lane_t,
                            volatile int* abort_flag) {
  using C = Cfg<D>;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int row = (warp & 3) * 32 + lane;                            // row within the 128-row tile
  const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16);  // this warp's TMEM lane base
  const uint32_t tS = trow + C::kColS + lane_t * 128;
  const uint32_t tO = trow + C::kColO + lane_t * D;
  const uint64_t tmo = p.timeout_ns;
  const float scale_log2 = p.scale_log2;
  uint32_t s_full_ph = 0;
  uint32_t total_pv = 0;
  bool ok = true;

  for (int w = blockIdx.x; w < p.n_items && ok; w += gridDim.x) {
    const Item it = decode_item(p, w);
    StepIter st;
    st.init(p, it);
    const int q_row = (lane_t ? it.q_start[1] : it.q_start[0]) + row;
    const bool lane_valid = lane_t ? it.valid[1] : it.valid[0];
    const int lim_row = p.causal ? min(p.kv_lim, q_row + 1) : p.kv_lim;
    float m_used = -INFINITY;  // running maximum of the scaled scores, log2 units
    float l = 0.f;             // running sum of exp2(score - m_used)
    int n_kept = 0;
    int kv_start;
    bool k0, k1;
    while (st.next(kv_start, k0, k1)) {
      if (!(lane_t == 0 ? k0 : k1)) continue;
      ok = mbar_wait(bars.s_full(lane_t), s_full_ph, tmo, ERR_TIMEOUT_S_FULL, abort_flag, p.err);
      ok = __all_sync(0xffffffffu, ok);
      s_full_ph ^= 1;
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr[c]);
      tmem_wait_ld();
      // Keys past the KV range, past S, or (causal) after this query: -inf.
      const int n_valid = lim_row - kv_start;
      if (__any_sync(0xffffffffu, n_valid < kTile)) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (c * 32 + e >= n_valid) sr[c][e] = __float_as_uint(-INFINITY);
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 32; ++e) mx = fmaxf(mx, __uint_as_float(sr[c][e]));
      const float m_tile = mx * scale_log2;
      const bool grow = m_tile > m_used + kRescaleThreshold;
      float alpha = 1.f;
      if (grow) {
        alpha = ex2_approx(m_used - m_tile);  // 0 when nothing was seen before
        l *= alpha;
        m_used = m_tile;
      }
      if (n_kept > 0 && __any_sync(0xffffffffu, grow)) {
        // O row *= alpha.  The previous O += P V of this lane has completed: S_t was only issued
        // after it, and its next one waits for this thread's P.
#pragma unroll 1
        for (int c = 0; c < D / 16; ++c) {
          uint32_t o[16];
          tmem_ld16(tO + c * 16, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st16(tO + c * 16, o);
        }
      }
      const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
      float rowsum = 0.f;
      // P (bf16, two per column) over the first 64 columns of S_t: the A operand of O += P V.  Each
      // half is stored as soon as it is packed, so its registers are free for the next half.
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2)
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int c = half * 2 + c2;
            const float p0 = ex2_approx(fmaf(__uint_as_float(sr[c][e]), scale_log2, neg_m));
            const float p1 = ex2_approx(fmaf(__uint_as_float(sr[c][e + 1]), scale_log2, neg_m));
            rowsum += p0 + p1;
            pk[c2 * 16 + (e >> 1)] = pack_bf16x2(p0, p1);
          }
        tmem_st32(tS + half * 32, pk);
      }
      l += rowsum;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.p_full(lane_t));
      ++n_kept;
      ++total_pv;
    }
    if (!ok) break;
    // Epilogue: O / l and lse for the rows of this lane.
    if (lane_valid) {
      const bool row_ok = q_row < p.S;
      const size_t o_idx = (((size_t)it.b * p.S + q_row) * p.H + it.h) * D;
      if (n_kept > 0) {
        ok = mbar_wait(bars.pv_done(lane_t), (total_pv - 1) & 1, tmo, ERR_TIMEOUT_PV_DONE, abort_flag, p.err);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld();
          if (row_ok) {
            if (p.o_f32) {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.o) + o_idx + c * 32);
#pragma unroll
              for (int e = 0; e < 8; ++e)
                dst[e] = make_float4(__uint_as_float(o[4 * e]) * inv_l, __uint_as_float(o[4 * e + 1]) * inv_l,
                                     __uint_as_float(o[4 * e + 2]) * inv_l,
                                     __uint_as_float(o[4 * e + 3]) * inv_l);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + o_idx + c * 32);
#pragma unroll
              for (int e = 0; e < 4; ++e)
                dst[e] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * e]) * inv_l, __uint_as_float(o[8 * e + 1]) * inv_l),
                                    pack_bf16x2(__uint_as_float(o[8 * e + 2]) * inv_l, __uint_as_float(o[8 * e + 3]) * inv_l),
                                    pack_bf16x2(__uint_as_float(o[8 * e + 4]) * inv_l, __uint_as_float(o[8 * e + 5]) * inv_l),
                                    pack_bf16x2(__uint_as_float(o[8 * e + 6]) * inv_l, __uint_as_float(o[8 * e + 7]) * inv_l));
            }
          }
        }
      } else if (row_ok) {
        if (p.o_f32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.o) + o_idx);
          for (int e = 0; e < D / 4; ++e) dst[e] = make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + o_idx);
          for (int e = 0; e < D / 8; ++e) dst[e] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      if (row_ok && p.lse)
        p.lse[((size_t)it.b * p.H + it.h) * p.S + q_row] =
            l > 0.f ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) smem_counter_add_release(bars.o_done(lane_t), 1u);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, const __grid_constant__ AttnParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t bar0 = smem_u32(smem + C::kBarOff);
  Bars bars;
  bars.q_full = bar0;
  bars.q_empty = bar0 + 8;
  bars.kv_full0 = bar0 + 16;
  bars.kv_empty0 = bars.kv_full0 + 8 * C::kStages;
  bars.s_full0 = bars.kv_empty0 + 8 * C::kStages;
  bars.p_full0 = bars.s_full0 + 16;
  bars.pv_done0 = bars.p_full0 + 16;
  bars.o_done0 = bars.pv_done0 + 16;
  bars.drain = bars.o_done0 + 16;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bars.q_full, 1);
    mbar_init(bars.q_empty, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bars.kv_full(s), 1);
      mbar_init(bars.kv_empty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bars.s_full(t), 1);
      mbar_init(bars.p_full(t), 4);   // one arrival per softmax warp
      mbar_init(bars.pv_done(t), 1);
    }
    *reinterpret_cast<volatile uint32_t*>(smem + C::kBarOff + (bars.o_done0 - bar0)) = 0u;
    *reinterpret_cast<volatile uint32_t*>(smem + C::kBarOff + (bars.o_done0 - bar0) + 8) = 0u;
    mbar_init(bars.drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpProducer && lane == 0) {
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp < 8) {
    run_softmax<D>(p, bars, tmem, warp >> 2, abort_flag);
  } else if (warp == kWarpProducer) {
    if (lane == 0) run_producer<D>(p, &tq, &tk, &tv, smem, bars, abort_flag);
    __syncwarp();
  } else {
    if (lane == 0) run_mma<D>(p, smem, bars, tmem, abort_flag);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

// ------------------------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------------------------
int attn_smem_bytes(int D) { return D == 128 ? Cfg<128>::kSmemBytes : Cfg<64>::kSmemBytes; }

sp_status launch_attn(const AttnParams& p_in, const void* q, const void* k, const void* v,
                      cudaStream_t stream) {
  AttnParams p = p_in;
  CUtensorMap tq, tk, tv;
  if (!encode_bshd_tmap(&tq, q, p.B, p.S, p.H, p.D) || !encode_bshd_tmap(&tk, k, p.B, p.S, p.H, p.D) ||
      !encode_bshd_tmap(&tv, v, p.B, p.S, p.H, p.D))
    return SP_ERR_CUDA;
  if (p.n_items <= 0) return SP_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SP_ERR_CUDA;
  const int grid = p.n_items < num_sms(dev) ? p.n_items : num_sms(dev);
  const int smem = attn_smem_bytes(p.D);
  cudaError_t e;
  if (p.D == 128) {
    static bool attr_set[kMaxDevices] = {};
    if (!attr_set[dev]) {
      e = cudaFuncSetAttribute(attn_fwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return SP_ERR_CUDA;
      attr_set[dev] = true;
    }
    attn_fwd_kernel<128><<<grid, kThreads, smem, stream>>>(tq, tk, tv, p);
  } else {
    static bool attr_set[kMaxDevices] = {};
    if (!attr_set[dev]) {
      e = cudaFuncSetAttribute(attn_fwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return SP_ERR_CUDA;
      attr_set[dev] = true;
    }
    attn_fwd_kernel<64><<<grid, kThreads, smem, stream>>>(tq, tk, tv, p);
  }
  return cudaGetLastError() == cudaSuccess ? SP_OK : SP_ERR_CUDA;
}

}  // namespace spattn
