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
//   warps 9,10  MMA issuers, one per lane: S_t = Q_t K_j^T into TMEM (fp32), and O_t += P_t V_j with
//               P_t read from TMEM and V_j from shared memory; tcgen05.commit signals completions.
//   warps 0-7   softmax, 4 warps per lane: thread r owns query row r of its lane's tile, loads its row
//               of S from TMEM (so every row reduction stays inside one thread), keeps the running
//               maximum m and sum l, writes P = exp(S - m) as bf16 back into TMEM over S, rescales
//               the O row in TMEM when the maximum grows by more than 2^8, and finally writes
//               O / l and lse = (m + log2 l) ln 2.  The two lanes run independently: while one
//               lane's warps compute exponentials, the tensor core runs the other lane's MMAs, and
//               when both are in their softmax phase the two warps per SMSP hide each other's latency.
//   warp 11     idle (it completes the third warpgroup, which gives its registers to the softmax).
//   TMEM (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256, 256+D), O_1 [256+D, 256+2D); P_t
//   overwrites the last 64 columns of S_t.  Each lane's issuer queues S_t(j+1) right behind
//   O_t += P_t(j) V_j: MMAs from one thread execute in issue order, so S_t(j+1) cannot overwrite P_t(j)
//   before the P V has read it.
// Every barrier wait is bounded in time; on expiry the kernel records an error and returns cleanly.
#include <atomic>
#include <climits>
#include <cstdint>
#include <cstdlib>
#include <type_traits>

#include "sp_internal.h"
#include "sp_ptx.cuh"

namespace spattn {

namespace {

constexpr int kTile = 128;
// 12 warps: 0-7 softmax (two warpgroups), 8 TMA producer, 9 and 10 MMA issuers (lanes 0 and 1),
// 11 idle.  Launched with
// kRegsLaunch registers per thread; the producer/MMA warpgroup gives registers back (kRegsControl)
// and the softmax warpgroups take them (kRegsSoftmax): 128 * 104 + 256 * 200 = 384 * 168.
constexpr int kThreads = 384;
constexpr int kWarpProducer = 8;
constexpr int kWarpMma = 9;  // MMA issuer of lane 0; kWarpMma + 1 issues for lane 1
constexpr int kRegsLaunch = 168;
constexpr uint32_t kRegsControl = 104;
constexpr uint32_t kRegsSoftmax = 200;
static_assert(128 * kRegsControl + 256 * kRegsSoftmax <= kThreads * kRegsLaunch, "register split");
constexpr int kItemRing = 8;     // work-item ids in flight between the producer and the other roles
constexpr int kSchedSlots = 64;  // launch-rotated work counters
// Per-launch work counters [next item, CTAs finished], kSchedSlots pairs handed out in rotation, so that
// up to kSchedSlots launches in flight at once (on different streams) draw different pairs.  Launches
// kSchedSlots apart draw the same pair: if two such launches overlapped on the GPU they would claim from
// one counter and skip or repeat items, so at most kSchedSlots attention launches may be in flight on a
// device (the C header states this limit).  A launch leaves its pair at zero when its last CTA ends.
__device__ unsigned int g_attn_sched[2 * kSchedSlots];
constexpr float kRescaleThreshold = 8.0f;  // log2 units: O and l are rescaled when m grows by > 2^8
constexpr uint32_t kPCol = 64;  // P_t (bf16 pairs) lives over the last 64 of S_t's 128 columns
// Of every 8 pairs of exponentials, this many run on the FMA pipe (the rest on the MUFU unit).  Measured on
// a B200: one in eight speeds split-key launches (one query tile per CTA) by 2-3%, and slows the launches with
// two query tiles per CTA (6% for CTA pairs), whose softmax warps have no registers to spare.
#ifdef SP_EXP2_POLY_PAIRS
template <bool kSplit>
constexpr int poly_pairs() { return SP_EXP2_POLY_PAIRS; }
#else
template <bool kSplit>
constexpr int poly_pairs() { return kSplit ? 1 : 0; }
#endif

// kSplit: both lanes work on ONE query tile and take alternate kept key tiles of its list (lane 0 the even
// ones, lane 1 the odd ones), each with its own running maximum, sum and O; the epilogue merges the two.
template <int D, bool kPair = false, bool kSplit = false>
struct Cfg {
  static_assert(!(kPair && kSplit), "a CTA pair never splits keys");
  static constexpr int kSub = D / 64;                   // 64-column (128-byte) sub-tiles per row
  static constexpr int kTileBytes = kTile * D * 2;      // one 128 x D bf16 tile
  static constexpr int kQTiles = kSplit ? 1 : 2;        // query tiles resident per work item
  // A K or V slot: a whole tile, or for a CTA pair this CTA's half (K: 64 of the 128 keys; V: 64 of the D
  // columns), the MMA's B operand being split by N between the two SMs.
  static constexpr int kKVBytes = kPair ? kTileBytes / 2 : kTileBytes;
  static constexpr int kKSubBytes = kPair ? 8192 : 16384;  // between the 64-column sub-tiles of a K slot
  // K/V ring slots (with one query tile resident, D = 128 has room for a fifth)
  static constexpr int kStages = kPair ? 6 : (D == 128 ? (kSplit ? 5 : 4) : 8);
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = kQTiles * kTileBytes;
  static constexpr int kBarOff = kKVOff + kStages * kKVBytes;
  // barriers: q_full, q_empty, kv_full[S], kv_empty[S], s_full[2], p_full[2], pv_done[2], drain, and
  // stg_full[8][2] (a merging epilogue's loads of the running O into each softmax warp's staging buffers)
  static constexpr int kNumBars = 2 + 2 * kStages + 7 + 16;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  // misc: TMEM base, abort flag, published-item count, per-warp item-read counts, the item ring (96
  // bytes); the O read-out progress words, 8 per lane (64 bytes); with kSplit also the lanes' exchange:
  // one 8-byte slot per query row (lane 1 posts its row maximum and sum, lane 0 answers with both lanes'
  // weights) and four hand-off counters, one per TMEM lane quadrant.
  static constexpr int kProgOff = kMiscOff + 96;
  static constexpr int kXchOff = kMiscOff + 160;
  static constexpr int kXcntOff = kXchOff + 128 * 8;
  static constexpr int kMiscBytes = kSplit ? 160 + 128 * 8 + 16 : 160;
  // then, 1024-aligned, staging for the O stores: per softmax warp two 4 KB buffers (32 rows x 128 bytes)
  // where they fit in the 227 KB a CTA may have, else one
  static constexpr int kStgOff = (kMiscOff + kMiscBytes + 1023) / 1024 * 1024;
  static constexpr int kStgBufs = kStgOff + 2 * 8 * 4096 + 1024 <= 232448 ? 2 : 1;
  static constexpr int kSmemBytes = kStgOff + kStgBufs * 8 * 4096 + 1024;  // + alignment slack
  static constexpr int kM = kPair ? 256 : 128;  // MMA rows: a pair computes both CTAs' 128 rows at once
  static constexpr uint32_t kIdescS = idesc_bf16_f32(kM, 128, false, false);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(kM, D, false, true);
  static constexpr uint32_t kRowWarps = kPair ? 8u : 4u;  // softmax warps per lane over the (pair of) CTAs
  // The softmax warps whose read-out of O_t an item's first P V into O_t waits for: lane t's (kRowWarps),
  // or with kSplit every softmax warp of the CTA, since each reads both lanes' O for its half of the columns.
  // Each has a progress word of its own, the number of items whose epilogue it has finished.
  static constexpr uint32_t kProgWords = kSplit ? 8u : kRowWarps;
  static constexpr uint32_t kColS = 0;
  static constexpr uint32_t kColO = 256;
};

// every configuration fits the 227 KB of shared memory a CTA may have
static_assert(Cfg<128, true>::kSmemBytes <= 232448 && Cfg<128, false>::kSmemBytes <= 232448 &&
                  Cfg<64, false>::kSmemBytes <= 232448 && Cfg<128, false, true>::kSmemBytes <= 232448 &&
                  Cfg<64, false, true>::kSmemBytes <= 232448,
              "shared memory");

struct Bars {
  uint32_t q_full, q_empty, kv_full0, kv_empty0, s_full0, p_full0, pv_done0, drain, stg_full0, prog0;
  // stg_full[w][b]: staging buffer b of softmax warp w holds the running O loaded for a merge
  __device__ uint32_t stg_full(int w, int b) const { return stg_full0 + 8u * (2 * w + b); }
  __device__ uint32_t kv_full(int s) const { return kv_full0 + 8u * s; }
  __device__ uint32_t kv_empty(int s) const { return kv_empty0 + 8u * s; }
  __device__ uint32_t s_full(int t) const { return s_full0 + 8u * t; }
  __device__ uint32_t p_full(int t) const { return p_full0 + 8u * t; }
  __device__ uint32_t pv_done(int t) const { return pv_done0 + 8u * t; }
  // prog(t, k): progress word k of lane t (rank 0's shared memory for a pair): the items whose epilogue,
  // and so whose read-out of O_t, softmax warp k has finished.  A word per warp, not one shared count: a
  // warp with nothing to read out may finish two items before another has finished one.
  __device__ uint32_t prog(int t, int k) const { return prog0 + 4u * (8u * t + k); }
};

struct Item {
  int b, h, qp;
  int sub;         // kSplit: which query tile of the pair (2 qp + sub) both lanes work on
  int shard;       // sequence shard holding both query tiles (0 when not sharded)
  int q_start[2];  // first row of each lane's query tile (global position)
  int q_last[2];   // last row of each lane's tile that exists (global position)
  int q_end;       // one past the last row of the shard (rows from here on belong to the next shard)
  bool valid[2];
  bool id_ok;      // false: the item list named an item that does not exist
  // What the MMAs walk: for a CTA pair, lane t covers this CTA's tile and the other CTA's tile t; the key
  // tiles are those either needs (equal to the fields above for a single CTA).
  int q_last_u[2];
  bool valid_u[2];
};

template <bool kPair = false, bool kSplit = false>
__device__ __forceinline__ Item decode_item(const AttnParams& p, int w) {
  // kSplit: the ring carries one entry per query tile, 2 * (item id) + tile within the item's pair
  const int sub = kSplit ? (w & 1) : 0;
  if (kSplit) w >>= 1;
  bool id_ok = true;
  if (p.item_list) {  // an explicit list: ids of the one-chunk layout, query-tile pair as given
    w = __ldg(p.item_list + w);
    id_ok = w >= 0 && w < p.item_space;
    if (!id_ok) w = 0;
  }
  // Items are ordered by head chunk, then batch, then head, then query-tile pair, so that the CTAs
  // running at the same time share one head's K/V in L2.  When causal, a head's pairs run longest
  // first, so that the last items of a launch, claimed by whichever CTA is free, are the short ones.
  int c = 0;
  while (c + 1 < p.n_chunks && w >= p.chunk_item0[c + 1]) ++c;
  const int r = w - p.chunk_item0[c];
  const int hc = p.chunk_h0[c + 1] - p.chunk_h0[c];
  // (a causal partial launch has no items for the leading p.qp_skip pairs, which no key reaches)
  const int n_run = p.n_qpairs - p.qp_skip;
  const int per_b = hc * n_run;
  Item it;
  it.b = r / per_b;
  const int r2 = r - it.b * per_b;
  it.h = p.chunk_h0[c] + r2 / n_run;
  const int qq = r2 % n_run;
  it.qp = (p.causal && !p.item_list) ? (p.n_qpairs - 1 - qq) : qq;
  // Query tiles are laid on each shard's own 128-row grid (one shard: the global grid); a shard's last
  // tile may be short, and items never cross shards.  An item is a pair of tiles, or for a CTA pair four:
  // rank r of the pair takes tiles 4u + 2r and 4u + 2r + 1 of its unit u.
  it.shard = it.qp / p.pairs_per_shard;
  const int lp = it.qp - it.shard * p.pairs_per_shard;
  it.q_end = min(p.S, (it.shard + 1) * p.shard_rows);
  const int rk = kPair ? (int)cluster_rank() : 0;
  it.sub = sub;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    it.valid_u[t] = false;
    it.q_last_u[t] = -1;
#pragma unroll
    for (int rr = 0; rr < (kPair ? 2 : 1); ++rr) {
      const int lt = kPair ? 4 * lp + 2 * rr + t : (kSplit ? 2 * lp + sub : 2 * lp + t);
      const int start = it.shard * p.shard_rows + lt * kTile;
      const bool valid = lt < p.tiles_per_shard && start < it.q_end;
      const int last = min(it.q_end, start + kTile) - 1;
      if (rr == rk) {
        it.q_start[t] = start;
        it.valid[t] = valid;
        it.q_last[t] = last;
      }
      if (valid) {
        it.valid_u[t] = true;
        it.q_last_u[t] = max(it.q_last_u[t], last);
      }
    }
  }
  it.id_ok = id_ok;
  if (!id_ok) it.valid[0] = it.valid[1] = it.valid_u[0] = it.valid_u[1] = false;  // nothing computed or written
  return it;
}

// Walks the key tiles a work item needs, in increasing key order, with which lanes need each.  Dense
// key tiles lie on each shard's own grid as the query tiles do (a shard's last tile may be short).
struct StepIter {
  bool sparse, causal, sharded;
  int kv_begin;
  int shard_rows, tiles_per_shard;
  int r, lt;       // shard and tile within it of the next dense tile (sharded)
  int shard;       // shard of the tile next() returned last (0 when not sharded)
  int key_end;     // one past that shard's last row (INT_MAX when not sharded)
  int q_last0, q_last1;
  bool v0, v1;
  bool split;      // both lanes on one query tile: the walked tiles go to lane 0 and lane 1 in turn
  int par;         // split: the lane that takes the next tile
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

  __device__ __forceinline__ void init(const AttnParams& p, const Item& it, bool split_keys = false) {
    split = split_keys;
    par = 0;
    causal = p.causal != 0;
    kv_begin = p.kv_begin;
    q_last0 = it.q_last_u[0];
    q_last1 = it.q_last_u[1];
    v0 = it.valid_u[0];
    v1 = it.valid_u[1];
    sparse = p.row_ptr != nullptr;
    sharded = p.n_shards > 1;
    shard_rows = p.shard_rows;
    tiles_per_shard = p.tiles_per_shard;
    j = 0;
    r = lt = 0;
    shard = 0;
    key_end = INT_MAX;
    if (!sparse) {
      n_dense = 0;
      if (v0 || v1) {
        n_dense = p.n_kv_tiles;
        if (causal) {
          const int ql = v1 ? q_last1 : q_last0;
          if (sharded) {  // the tile of key ql on its shard's grid (kv_begin is 0 here)
            const int r = ql / shard_rows;
            n_dense = min(p.n_kv_tiles, r * tiles_per_shard + (ql - r * shard_rows) / kTile + 1);
          } else {
            n_dense = ql < p.kv_begin ? 0 : min(p.n_kv_tiles, (ql - p.kv_begin) / kTile + 1);
          }
        }
      }
      return;
    }
    // Tile range allowed by [kv_begin, kv_lim): kv_begin is a multiple of 128 here.
    const int t_lo = p.kv_begin / kTile;
    const int t_hi = (p.kv_lim + kTile - 1) / kTile;  // exclusive
    l0 = p.col_idx;
    l1 = p.col_idx;
    const int row0 = it.h * p.mask_T + 2 * it.qp + (split ? it.sub : 0);
    i0 = e0 = i1 = e1 = 0;
    if (split) {  // one list (the tile's row), dealt to the lanes in turn by next()
      if (v0) {
        i0 = __ldg(p.row_ptr + row0);
        e0 = __ldg(p.row_ptr + row0 + 1);
        const int hi0 = causal ? min(t_hi, q_last0 / kTile + 1) : t_hi;
        if (t_lo > 0) i0 = lower_bound(l0, i0, e0, t_lo);
        if (hi0 < p.mask_T) e0 = lower_bound(l0, i0, e0, hi0);
      }
      c0 = c1 = INT_MAX;
      return;
    }
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
      if (sharded) {  // walk the shards' grids without dividing
        kv_start = r * shard_rows + lt * kTile;
        shard = r;
        key_end = (r + 1) * shard_rows;
        if (++lt == tiles_per_shard) {
          lt = 0;
          ++r;
        }
      } else {
        kv_start = kv_begin + j * kTile;
      }
      ++j;
      k0 = v0 && (!causal || kv_start <= q_last0);
      k1 = v1 && (!causal || kv_start <= q_last1);
      if (split) {
        k0 = k0 && par == 0;
        k1 = k1 && par == 1;
        par ^= 1;
      }
      return true;
    }
    if (split) {
      if (i0 >= e0) return false;
      kv_start = __ldg(l0 + i0) * kTile;
      ++i0;
      k0 = par == 0;
      k1 = par == 1;
      par ^= 1;
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
// Work distribution: every CTA starts with item blockIdx.x; after that the producer warp claims items
// from a per-launch counter in global memory (dynamic: a CTA that drew short items takes more), and
// publishes the claimed ids, in order, into a ring in shared memory that the other roles read.
// -1 marks the end.  The ring slot of item n is reused for item n + kItemRing only after each of the
// eight softmax warps has read it: every softmax warp counts its reads in a word of its own (a sum
// over warps would not do, since on items without keys the warps of a lane do not wait for one another
// and one may read ahead of another by more than the ring holds).  The MMA warps need no count: the
// producer loads item n's Q only after both of them are done with item n - 1.
// ------------------------------------------------------------------------------------------------
struct ItemRing {
  uint32_t pub;    // shared address: number of item ids published
  uint32_t used0;  // shared address: items read by softmax warp 0; warp k at +4k
  volatile int* ids;
};

// cluster_acquire: the ring is written by the other CTA of a pair (rank 1 reads what rank 0 publishes).
__device__ __forceinline__ bool ring_read(const ItemRing& r, int n, int& w, uint64_t tmo, volatile int* abort_flag,
                                          unsigned int* err, bool cluster_acquire = false) {
  const bool ok = cluster_acquire ? warp_counter_wait_cluster(r.pub, (uint32_t)(n + 1), tmo, ERR_TIMEOUT_ITEM, abort_flag, err)
                                  : warp_counter_wait(r.pub, (uint32_t)(n + 1), tmo, ERR_TIMEOUT_ITEM, abort_flag, err);
  if (!ok) return false;
  w = r.ids[n % kItemRing];
  return true;
}

// ------------------------------------------------------------------------------------------------
// Sequence shards: the tensor maps of every shard of Q, K and V (one shard when the tensors are not
// split).  Every tile lies on one shard's grid, so it is one TMA box of that shard; the rows of a short
// last tile past the shard's end read as zero and are masked (keys) or not written (queries).
// ------------------------------------------------------------------------------------------------
struct TMaps {
  CUtensorMap q[kMaxShards];
  CUtensorMap k[kMaxShards];
  CUtensorMap v[kMaxShards];
  CUtensorMap k64[kMaxShards];  // K with 64-row boxes: a CTA pair's halves of a key tile
  CUtensorMap o[kMaxShards];    // O as a store target (bf16 or fp32), 32-row boxes
};

// ------------------------------------------------------------------------------------------------
// Producer: one warp walks the work in lockstep (all values warp-uniform); one elected lane issues the
// TMA loads.
// ------------------------------------------------------------------------------------------------
template <int D, bool kPair, bool kSplit>
__device__ void run_producer(const AttnParams& p, const TMaps& tm, uint8_t* smem, const Bars& bars,
                             const ItemRing& ir, volatile int* abort_flag) {
  using C = Cfg<D, kPair, kSplit>;
  const uint32_t sbase = smem_u32(smem);
  const uint64_t tmo = p.timeout_ns;
  // A CTA pair: each CTA loads its own query tiles and its half of every K/V tile, and the bytes complete
  // on rank 0's barriers (whose MMA consumes both halves); only rank 0 arms them.
  const uint32_t rk = kPair ? cluster_rank() : 0u;
  const uint32_t q_full_bar = kPair ? map_shared(bars.q_full, 0) : bars.q_full;
  uint32_t q_empty_ph = 0;
  int ring = 0;
  int n_item = 0;
  int last_q_item = -1;
  bool ok = true;
  // The work units a CTA (or a pair, whose rank 0 claims for both) takes: its first by its index, then by
  // claiming from the launch's counter; ids go into the item ring of the CTA (or of both CTAs of the pair).
  const int n_workers = kPair ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  int w = kPair ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  int id = w;  // the ring entry: the item id, or with kSplit 2 * item + query tile within the item's pair
  for (;; ++n_item) {
    bool done;
    if (kPair && rk != 0) {  // rank 1 reads what rank 0 published into its ring
      ok = ring_read(ir, n_item, w, tmo, abort_flag, p.err, true);
      if (!ok) break;
      id = w;
      done = w < 0;
      if (done) break;
    } else {
      // claim the next item (kSplit: every item runs as two ring entries, one per query tile of its pair)
      if (n_item > 0 && (!kSplit || (n_item & 1) == 0)) {
        int claimed = 0;
        if (elect_one_sync()) claimed = n_workers + (int)atomicAdd(p.sched, 1u);
        w = __shfl_sync(0xffffffffu, claimed, __ffs(__ballot_sync(0xffffffffu, claimed != 0)) - 1);
      }
      done = w >= p.n_items;
      // publish it (the slot's previous item must have been read by every softmax warp, of both CTAs)
      if (n_item >= kItemRing) {
        const uint32_t need = (uint32_t)(n_item - kItemRing + 1);
#pragma unroll 1
        for (int k = 0; k < 8 && ok; ++k)
          ok = warp_counter_wait(ir.used0 + 4u * k, need, tmo, ERR_TIMEOUT_ITEM_FREE, abort_flag, p.err);
        if constexpr (kPair) {
#pragma unroll 1
          for (int k = 0; k < 8 && ok; ++k)
            ok = warp_remote_counter_wait(map_shared(ir.used0 + 4u * k, 1), need, tmo, ERR_TIMEOUT_ITEM_FREE,
                                          abort_flag, p.err);
        }
        if (!ok) break;
      }
      id = done ? -1 : (kSplit ? 2 * w + (n_item & 1) : w);
      if (elect_one_sync()) {
        ir.ids[n_item % kItemRing] = id;
        smem_counter_add_release(ir.pub, 1u);
        if constexpr (kPair) {
          remote_store(map_shared(smem_u32((const void*)(ir.ids + n_item % kItemRing)), 1), (uint32_t)id);
          counter_add_cluster(map_shared(ir.pub, 1), 1u);
        }
      }
      __syncwarp();
      if (done) break;
    }
    const Item it = decode_item<kPair, kSplit>(p, id);
    if (!it.id_ok && elect_one_sync() && (!kSplit || it.sub == 0)) atomicOr(p.err, ERR_BAD_ITEM);
    if (n_item > 0) {
      ok = warp_mbar_wait(bars.q_empty, q_empty_ph, tmo, ERR_TIMEOUT_Q_EMPTY, abort_flag, p.err);
      q_empty_ph ^= 1;
      if (!ok) break;
    }
    if (elect_one_sync()) {
      const int y0 = it.shard * p.shard_rows;  // the item's shard starts at this global row
      if (rk == 0) mbar_arrive_expect_tx(bars.q_full, (kPair ? 4 : C::kQTiles) * C::kTileBytes);
#pragma unroll
      for (int t = 0; t < C::kQTiles; ++t)
#pragma unroll
        for (int c = 0; c < C::kSub; ++c) {
          const uint32_t dst = sbase + C::kQOff + t * C::kTileBytes + c * 16384;
          if constexpr (kPair)
            tma_load_4d_pair(dst, &tm.q[it.shard], q_full_bar, 64 * c, it.h, it.q_start[t] - y0, it.b);
          else
            tma_load_4d(dst, &tm.q[it.shard], bars.q_full, 64 * c, it.h, it.q_start[t] - y0, it.b);
        }
    }
    __syncwarp();
    last_q_item = n_item;
    StepIter st;
    st.init(p, it, kSplit);
    int kv_start;
    bool k0, k1;
    while (ok && st.next(kv_start, k0, k1)) {
#pragma unroll
      for (int kv = 0; kv < 2; ++kv) {
        const int slot = ring % C::kStages;
        const int lap = ring / C::kStages;
        if (lap > 0) {
          ok = warp_mbar_wait(bars.kv_empty(slot), (lap - 1) & 1, tmo, ERR_TIMEOUT_KV_EMPTY, abort_flag, p.err);
          if (!ok) break;
        }
        if (elect_one_sync()) {
          const uint32_t dst = sbase + C::kKVOff + slot * C::kKVBytes;
          const int y = kv_start - st.shard * p.shard_rows;
          if constexpr (kPair) {
            const uint32_t bar = map_shared(bars.kv_full(slot), 0);
            if (rk == 0) mbar_arrive_expect_tx(bars.kv_full(slot), 2 * C::kKVBytes);
            if (kv == 0) {  // keys [64 rk, 64 rk + 64) of the tile, all D columns
#pragma unroll
              for (int c = 0; c < C::kSub; ++c)
                tma_load_4d_pair(dst + c * C::kKSubBytes, &tm.k64[st.shard], bar, 64 * c, it.h, y + 64 * (int)rk, it.b);
            } else {        // all 128 keys, columns [64 rk, 64 rk + 64)
              tma_load_4d_pair(dst, &tm.v[st.shard], bar, 64 * (int)rk, it.h, y, it.b);
            }
          } else {
            mbar_arrive_expect_tx(bars.kv_full(slot), C::kKVBytes);
            const CUtensorMap* map = kv == 0 ? &tm.k[st.shard] : &tm.v[st.shard];
#pragma unroll
            for (int c = 0; c < C::kSub; ++c)
              tma_load_4d(dst + c * 16384, map, bars.kv_full(slot), 64 * c, it.h, y, it.b);
          }
        }
        __syncwarp();
        ++ring;
      }
    }
  }
  if (*abort_flag) {
    // Do not leave copies in flight into shared memory: wait (bounded) for the most recent load of
    // every slot and for the last Q load.  A pair's rank 1 cannot observe its own loads (their bytes
    // complete on rank 0's barriers): it waits out a fixed interval far longer than a load.
    if (kPair && rk != 0) {
      const uint64_t t0 = global_timer_ns();
      while (global_timer_ns() - t0 < 200000ull) {
      }
    } else {
      for (int pos = max(0, ring - C::kStages); pos < ring; ++pos)
        warp_mbar_wait(bars.kv_full(pos % C::kStages), (pos / C::kStages) & 1, tmo, ERR_TIMEOUT_KV_FULL, nullptr,
                       p.err);
      if (last_q_item >= 0) warp_mbar_wait(bars.q_full, last_q_item & 1, tmo, ERR_TIMEOUT_Q_FULL, nullptr, p.err);
    }
  }
}

// ------------------------------------------------------------------------------------------------
// MMA issuers: one warp per lane walks the work in lockstep (all values warp-uniform, so descriptors
// stay in uniform registers); one elected lane issues the tcgen05 instructions.  With a warp per lane,
// one lane's waits (for its P, or for its previous P V) never hold up the other lane's MMAs; the tensor
// core interleaves the two lanes.  Shared K/V slots and the Q buffer are released when both lanes are
// done with them (the "empty" barriers count two arrivals; a lane that skips a tile arrives directly).
// ------------------------------------------------------------------------------------------------
template <int D, bool kPair, bool kSplit>
__device__ void run_mma(const AttnParams& p, uint8_t* smem, const Bars& bars, const ItemRing& ir, uint32_t tmem_in,
                        int t, volatile int* abort_flag) {
  using C = Cfg<D, kPair, kSplit>;
  const uint32_t sbase = smem_u32(smem);
  const uint64_t tmo = p.timeout_ns;
  const uint32_t tmem = __shfl_sync(0xffffffffu, tmem_in, 0);  // provably warp-uniform
  // Descriptors of K-step 0; later K-steps add their byte offset / 16 to the start-address field.  For a
  // pair the same shared-memory offsets name both CTAs' halves of each operand.
  const uint64_t q_desc = smem_desc_sw128(sbase + C::kQOff + (kSplit ? 0 : t) * C::kTileBytes, 16, 1024);
  const uint64_t kv_desc0 = smem_desc_sw128(sbase + C::kKVOff, 16, 1024);
  const uint64_t v_desc0 = smem_desc_sw128(sbase + C::kKVOff, 16384, 1024);
  const uint32_t s_tmem = tmem + C::kColS + t * 128;  // S_t, and P_t over its last 64 columns
  const uint32_t o_tmem = tmem + C::kColO + t * D;
  const uint32_t s_full = bars.s_full(t), p_full = bars.p_full(t), pv_done = bars.pv_done(t);  // pv_done: for the epilogue
  uint32_t q_full_ph = 0, p_full_ph = 0;
  int ring = 0;
  int n_item = 0;
  bool ok = true;
  int w = 0;
  auto commit = [](uint32_t bar) {
    if constexpr (kPair) mma_commit_pair(bar); else mma_commit(bar);
  };
  // A lane that skips a key tile still releases its slot: in both CTAs of a pair.
  auto release = [&](uint32_t bar) {
    mbar_arrive(bar);
    if constexpr (kPair) mbar_arrive_cluster(map_shared(bar, 1));
  };
  for (;; ++n_item) {
    ok = ring_read(ir, n_item, w, tmo, abort_flag, p.err);
    if (!ok || w < 0) break;
    const Item it = decode_item<kPair, kSplit>(p, w);
    ok = warp_mbar_wait(bars.q_full, q_full_ph, tmo, ERR_TIMEOUT_Q_FULL, abort_flag, p.err);
    q_full_ph ^= 1;
    if (!ok) break;
    tc_fence_after();
    // O_t may be overwritten by this item's first P V only after the softmax warps of lane t (4, or 8 over
    // a pair) have read out the previous item's O: each one's progress word has reached this item.
    bool need_odone = n_item > 0;
    bool first_pv = true;
    StepIter st;
    st.init(p, it, kSplit);
    // A kept step's O_t += P_t V_j is issued lazily, just before this lane's next S MMA (which overwrites
    // P_t: tcgen05 MMAs from one thread execute in issue order, so no wait is needed) or after the item's
    // last step.  Steps this lane does not keep release their K and V slots at once, without waiting for
    // this lane's softmax, so that the other lane (and the producer) can run ahead.
    bool pend = false;  // a P V not yet issued
    int pend_v_pos = 0;
    auto issue_pv = [&]() -> bool {
      const int vs = pend_v_pos % C::kStages;
      bool good = warp_mbar_wait(bars.kv_full(vs), (pend_v_pos / C::kStages) & 1, tmo, ERR_TIMEOUT_KV_FULL,
                                 abort_flag, p.err);
      if (good && need_odone) {
#pragma unroll 1
        for (uint32_t k = 0; k < C::kProgWords && good; ++k)
          good = kPair ? warp_counter_wait_cluster(bars.prog(t, k), (uint32_t)n_item, tmo, ERR_TIMEOUT_O_FREE,
                                                   abort_flag, p.err)
                       : warp_counter_wait(bars.prog(t, k), (uint32_t)n_item, tmo, ERR_TIMEOUT_O_FREE, abort_flag,
                                           p.err);
        need_odone = false;
      }
      if (good) {
        good = warp_mbar_wait(p_full, p_full_ph, tmo, ERR_TIMEOUT_P_FULL, abort_flag, p.err);
        p_full_ph ^= 1;
      }
      if (!good) return false;
      tc_fence_after();
      const uint64_t v_desc = v_desc0 + (uint64_t)((vs * C::kKVBytes) >> 4);
      const uint32_t acc0 = first_pv ? 0u : 1u;
      if (elect_one_sync()) {
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          if constexpr (kPair)
            mma_ts_pair(o_tmem, s_tmem + kPCol + kk * 8, v_desc + (uint64_t)(kk * 128), C::kIdescPV,
                        kk > 0 ? 1u : acc0);
          else
            mma_ts(o_tmem, s_tmem + kPCol + kk * 8, v_desc + (uint64_t)(kk * 128), C::kIdescPV, kk > 0 ? 1u : acc0);
        }
        commit(pv_done);
        commit(bars.kv_empty(vs));
      }
      __syncwarp();
      first_pv = false;
      return true;
    };
    for (;;) {
      int kv_start;
      bool k0, k1;
      if (!st.next(kv_start, k0, k1)) break;
      const bool keep = t ? k1 : k0;
      const int k_pos = ring;
      const int ks = k_pos % C::kStages;
      ring += 2;
      if (!keep) {
        // A pending P V still holds its V slot: issue it before waiting on a position that reuses that slot
        // (its next load needs the slot released), so that the walk can never wait on itself.  Its P needs
        // only this lane's softmax, which depends on nothing of the walk.
        if (pend && k_pos + 1 >= pend_v_pos + C::kStages) {
          ok = issue_pv();
          pend = false;
          if (!ok) break;
        }
        // Not used by this lane: still wait for both loads, so that this warp consumes every phase of every
        // slot (a skipped phase would let a later parity wait see a stale one), and release them.
        ok = warp_mbar_wait(bars.kv_full(ks), (k_pos / C::kStages) & 1, tmo, ERR_TIMEOUT_KV_FULL, abort_flag, p.err);
        if (ok) {
          if (elect_one_sync()) release(bars.kv_empty(ks));
          __syncwarp();
          const int vs = (k_pos + 1) % C::kStages;
          ok = warp_mbar_wait(bars.kv_full(vs), ((k_pos + 1) / C::kStages) & 1, tmo, ERR_TIMEOUT_KV_FULL, abort_flag,
                              p.err);
          if (ok && elect_one_sync()) release(bars.kv_empty(vs));
          __syncwarp();
        }
        if (!ok) break;
        continue;
      }
      if (pend) {  // O_t += P_t V of this lane's previous step
        ok = issue_pv();
        pend = false;
        if (!ok) break;
      }
      // S_t = Q_t K_j^T.  It overwrites P_t, which the P V just issued reads: tcgen05.mma operations
      // issued by one thread execute in issue order, so no wait is needed here, and the commit below
      // (which fires once all earlier MMAs of this thread are complete) also tells the softmax that
      // O_t is no longer being written.
      ok = warp_mbar_wait(bars.kv_full(ks), (k_pos / C::kStages) & 1, tmo, ERR_TIMEOUT_KV_FULL, abort_flag, p.err);
      if (!ok) break;
      tc_fence_after();
      const uint64_t k_desc = kv_desc0 + (uint64_t)((ks * C::kKVBytes) >> 4);
      if (elect_one_sync()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t qo = (uint64_t)(((kk / 4) * 16384 + (kk % 4) * 32) >> 4);
          const uint64_t ko = (uint64_t)(((kk / 4) * C::kKSubBytes + (kk % 4) * 32) >> 4);
          if constexpr (kPair)
            mma_ss_pair(s_tmem, q_desc + qo, k_desc + ko, C::kIdescS, kk > 0 ? 1u : 0u);
          else
            mma_ss(s_tmem, q_desc + qo, k_desc + ko, C::kIdescS, kk > 0 ? 1u : 0u);
        }
        commit(s_full);
        commit(bars.kv_empty(ks));
      }
      __syncwarp();
      pend = true;
      pend_v_pos = k_pos + 1;
    }
    if (!ok) break;
    // This lane's S MMAs of the item are all issued: Q is free once they complete (the producer loads the
    // next item's Q while the last softmax runs).
    if (elect_one_sync()) commit(bars.q_empty);
    __syncwarp();
    if (pend) {
      ok = issue_pv();
      if (!ok) break;
    }
  }
  // Drain: nothing of ours may still run on the tensor cores when TMEM is released.
  if (elect_one_sync()) commit(bars.drain);
  __syncwarp();
  warp_mbar_wait(bars.drain, 0, tmo, ERR_TIMEOUT_DRAIN, nullptr, p.err);
}

// ------------------------------------------------------------------------------------------------
// Epilogue of a launch that merges its rows into a running result (o fp32, lse), the re-merge of one KV
// block's partial into the accumulated earlier blocks ("CHARM+: Cross-Hardware Attention with Re-Merge
// ...", abstract; the Ring-Attention paragraph of "CHARM+: How Cross-Hardware Attention Breaks Through
// ...": each round's partial result is accumulated).  With this block's row maximum m and sum l (log2
// units) and the running lse a (natural log):
//   b = m + log2 l,  c = max(a log2 e, b),  wa = 2^(a log2 e - c),  wb = 2^(b - c),
//   o <- (o wa + (O / l) wb) / (wa + wb),   lse <- (c + log2(wa + wb)) ln 2.
// A row whose running lse is -inf has no running result: its o is not read into the sum (it may hold
// anything).  A row that saw no key of this block keeps o and lse as they are.
// The warp's 32 rows of the running o move as 32 x 32 fp32 boxes: TMA loads into the warp's staging
// buffers (issued before the last P V is awaited, so they overlap it), the merge in shared memory, TMA
// stores from the same buffers.  Returns false when a wait gave up (the error is recorded).
// ------------------------------------------------------------------------------------------------
template <int D, bool kPair, bool kSplit>
__device__ __forceinline__ bool merge_epilogue(const AttnParams& p, const TMaps& tm, uint32_t sbase, const Bars& bars,
                                               uint32_t tO, const Item& it, int q_row, int row, int warp, int lane,
                                               int lane_t, bool row_ok, float l, float m_used, uint32_t total_pv,
                                               uint32_t& stg_ph, volatile int* abort_flag) {
  using C = Cfg<D, kPair, kSplit>;
  constexpr int kBoxes = D / 32;  // fp32 boxes of 32 columns per row
  constexpr int kFirst = C::kStgBufs < kBoxes ? C::kStgBufs : kBoxes;
  const uint64_t tmo = p.timeout_ns;
  const uint32_t stg0 = sbase + C::kStgOff + (uint32_t)warp * (4096u * C::kStgBufs);
  const CUtensorMap* omap = &tm.o[0];
  const int row0 = q_row - row + (warp & 3) * 32;
  if (lane == 0) {
#pragma unroll
    for (int c = 0; c < kFirst; ++c) {
      mbar_arrive_expect_tx(bars.stg_full(warp, c), 4096u);
      tma_load_4d(stg0 + 4096u * c, omap, bars.stg_full(warp, c), 32 * c, it.h, row0, it.b);
    }
  }
  __syncwarp();
  uint32_t pending = (1u << kFirst) - 1u;  // staging buffers with a load in flight
  // Weights of the running result and of this block's rows (no global read yet depends on the MMAs).
  const size_t l_idx = ((size_t)it.b * p.H + it.h) * p.S + q_row;
  const float la = row_ok ? p.lse[l_idx] * 1.4426950408889634f : -INFINITY;
  const bool has = l > 0.f && m_used != -INFINITY;
  float wa = 1.f, wb = 0.f, lnew = la;
  if (has) {
    const float lb = m_used + log2f(l);
    const float c = fmaxf(la, lb);
    const float ea = la == -INFINITY ? 0.f : ex2_approx(la - c);
    const float eb = ex2_approx(lb - c);
    const float inv = 1.f / (ea + eb);
    wa = ea * inv;
    wb = eb * inv / l;  // O in TMEM is not yet divided by l
    lnew = c + log2f(ea + eb);
  }
  bool ok = mbar_wait(bars.pv_done(lane_t), (total_pv - 1) & 1, tmo, ERR_TIMEOUT_PV_DONE, abort_flag, p.err);
  ok = __all_sync(0xffffffffu, ok);
  if (ok) {
    tc_fence_after();
#pragma unroll 1
    for (int c = 0; c < kBoxes; ++c) {
      const int b = c % C::kStgBufs;
      const uint32_t stg = stg0 + 4096u * (uint32_t)b;
      ok = mbar_wait(bars.stg_full(warp, b), (stg_ph >> b) & 1u, tmo, ERR_TIMEOUT_STG, abort_flag, p.err);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      stg_ph ^= 1u << b;
      pending &= ~(1u << b);
      uint32_t v[32];
      tmem_ld32(tO + c * 32, v);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t addr = stg + (uint32_t)lane * 128u + (uint32_t)((e ^ (lane & 7)) << 4);
        uint32_t a[4];
        ld_shared_v4(addr, a[0], a[1], a[2], a[3]);
        uint32_t r[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float x = wa > 0.f ? __uint_as_float(a[j]) * wa : 0.f;
          const float y = wb > 0.f ? __uint_as_float(v[4 * e + j]) * wb : 0.f;
          r[j] = __float_as_uint(x + y);
        }
        st_shared_v4(addr, r[0], r[1], r[2], r[3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_4d(omap, stg, 32 * c, it.h, row0, it.b);
        bulk_commit_group();
        if (c + C::kStgBufs < kBoxes) {  // refill this buffer with a later box once the store has read it
          bulk_wait_read_all();
          mbar_arrive_expect_tx(bars.stg_full(warp, b), 4096u);
          tma_load_4d(stg, omap, bars.stg_full(warp, b), 32 * (c + C::kStgBufs), it.h, row0, it.b);
        }
      }
      if (c + C::kStgBufs < kBoxes) pending |= 1u << b;
      __syncwarp();
    }
  }
  if (!ok) {
    // Leave no load in flight into shared memory: wait (bounded) for every outstanding one.
#pragma unroll 1
    for (int b = 0; b < C::kStgBufs; ++b)
      if (pending & (1u << b)) {
        warp_mbar_wait(bars.stg_full(warp, b), (stg_ph >> b) & 1u, tmo, ERR_TIMEOUT_STG, nullptr, p.err);
        stg_ph ^= 1u << b;
      }
    return false;
  }
  if (lane == 0) bulk_wait_read_all();  // the buffers are free for the next item
  __syncwarp();
  if (row_ok && has) p.lse[l_idx] = lnew * 0.69314718055994531f;
  return true;
}

// ------------------------------------------------------------------------------------------------
// Epilogue of a split-keys item: the two lanes hold one query tile's O_0, O_1 (TMEM), row maxima m_0, m_1
// and sums l_0, l_1 over disjoint halves of its key tiles.  The row's result is their log-sum-exp merge
//   M = max(m_0, m_1),  w_t = 2^(m_t - M),  L = l_0 w_0 + l_1 w_1,  O = (O_0 w_0 + O_1 w_1) / L,
//   lse = (M + log2 L) ln 2
// (the same rule as the KV-block re-merge).  The two warps of a TMEM lane quadrant (one per lane) hand
// (m_1, l_1) to lane 0 and (w_0 / L, w_1 / L) back through shared memory; then each writes half of the D
// columns, reading both lanes' O for them.  A lane that took no tile has weight 0 and its (stale) O is
// never read into the sum.  Returns false when a wait gave up (the error is recorded).
// ------------------------------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ bool split_epilogue(const AttnParams& p, const TMaps& tm, uint32_t sbase, const Bars& bars,
                                               uint32_t trow, const Item& it, int q_row, int row, int warp, int lane,
                                               int lane_t, bool row_ok, float l, float m_used, int n_kept,
                                               uint32_t total_pv, uint32_t n_xch, volatile int* abort_flag) {
  using C = Cfg<D, false, true>;
  const uint64_t tmo = p.timeout_ns;
  const int quad = warp & 3;
  if (n_kept > 0) {
    bool ok = mbar_wait(bars.pv_done(lane_t), (total_pv - 1) & 1, tmo, ERR_TIMEOUT_PV_DONE, abort_flag, p.err);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) return false;
  }
  const bool has = n_kept > 0 && l > 0.f && m_used != -INFINITY;
  const float m = has ? m_used : -INFINITY;
  const float s = has ? l : 0.f;
  const uint32_t slot = sbase + C::kXchOff + (uint32_t)(quad * 32 + lane) * 8u;
  const uint32_t cnt = sbase + C::kXcntOff + 4u * (uint32_t)quad;
  float c0, c1, lse2 = -INFINITY;
  tc_fence_before();  // this lane's O is complete; the other lane's warp reads it after the hand-off
  if (lane_t == 1) {
    st_shared_v2f(slot, m, s);
    __syncwarp();
    if (lane == 0) smem_counter_add_release(cnt, 1u);
    bool ok = counter_wait(cnt, 2u * n_xch + 2u, tmo, ERR_TIMEOUT_XCH, abort_flag, p.err);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) return false;
    ld_shared_v2f(slot, c0, c1);
  } else {
    bool ok = counter_wait(cnt, 2u * n_xch + 1u, tmo, ERR_TIMEOUT_XCH, abort_flag, p.err);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) return false;
    float m1, s1;
    ld_shared_v2f(slot, m1, s1);
    const float mx = fmaxf(m, m1);
    const float w0 = m == -INFINITY ? 0.f : ex2_approx(m - mx);
    const float w1 = m1 == -INFINITY ? 0.f : ex2_approx(m1 - mx);
    const float L = s * w0 + s1 * w1;
    const float inv = L > 0.f ? 1.f / L : 0.f;
    c0 = w0 * inv;
    c1 = w1 * inv;
    if (L > 0.f) lse2 = mx + log2f(L);
    st_shared_v2f(slot, c0, c1);
    __syncwarp();
    if (lane == 0) smem_counter_add_release(cnt, 1u);
  }
  tc_fence_after();
  // Boxes of 128 bytes of each of the warp's 32 rows (64 bf16 or 32 fp32 columns): lane t takes half of them
  // (with one box per row, lane 0 takes it).
  const int n_boxes = p.o_f32 ? D / 32 : D / 64;
  const int b_lo = n_boxes >= 2 ? lane_t * (n_boxes / 2) : 0;
  const int b_hi = n_boxes >= 2 ? (lane_t + 1) * (n_boxes / 2) : (lane_t == 0 ? 1 : 0);
  const uint32_t tO0 = trow + C::kColO, tO1 = trow + C::kColO + D;
  const uint32_t stg0 = sbase + C::kStgOff + (uint32_t)warp * (4096u * C::kStgBufs);
  const CUtensorMap* omap = &tm.o[0];
  const int row0 = q_row - row + quad * 32;
  auto mix = [&](uint32_t a, uint32_t b) {
    const float x = c0 > 0.f ? __uint_as_float(a) * c0 : 0.f;
    const float y = c1 > 0.f ? __uint_as_float(b) * c1 : 0.f;
    return x + y;
  };
#pragma unroll 1
  for (int c = b_lo; c < b_hi; ++c) {
    uint32_t v[32];
    if (p.o_f32) {
      uint32_t a[32], b[32];
      tmem_ld32(tO0 + c * 32, a);
      tmem_ld32(tO1 + c * 32, b);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(mix(a[e], b[e]));
    } else {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t a[32], b[32];
        tmem_ld32(tO0 + c * 64 + h * 32, a);
        tmem_ld32(tO1 + c * 64 + h * 32, b);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) v[16 * h + e] = pack_bf16x2(mix(a[2 * e], b[2 * e]), mix(a[2 * e + 1], b[2 * e + 1]));
      }
    }
    const int k = c - b_lo;
    const uint32_t stg = stg0 + 4096u * (uint32_t)(k % C::kStgBufs);
    if (k >= C::kStgBufs) {  // the store that last used this buffer must have read it
      if (lane == 0) {
        if (C::kStgBufs == 2)
          bulk_wait_read_but1();
        else
          bulk_wait_read_all();
      }
      __syncwarp();
    }
#pragma unroll
    for (int e = 0; e < 8; ++e)
      st_shared_v4(stg + (uint32_t)lane * 128u + (uint32_t)(((e ^ (lane & 7)) << 4)), v[4 * e], v[4 * e + 1],
                   v[4 * e + 2], v[4 * e + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_4d(omap, stg, c * (p.o_f32 ? 32 : 64), it.h, row0, it.b);
      bulk_commit_group();
    }
  }
  if (lane == 0) bulk_wait_read_all();  // the buffers are free for the next item
  __syncwarp();
  if (lane_t == 0 && row_ok && p.lse)
    p.lse[((size_t)it.b * p.H + it.h) * p.S + q_row] = lse2 == -INFINITY ? -INFINITY : lse2 * 0.69314718055994531f;
  return true;
}

// A thread's O row in TMEM multiplied by alpha (warp-collective: every lane of the warp calls it); it runs
// only when a row's maximum grows by more than 2^8 (log2 units).  Inlined: out of line, the call measured
// 10% slower block-sparse launches although it never runs there.
template <int D>
__device__ __forceinline__ void rescale_o_row(uint32_t tO, float alpha) {
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

// The epilogue of one item for one softmax warp (O / l and lse of its 32 rows, or their merge into a running
// result), then the warp's progress word.  Returns false when a wait gave up (the error is recorded).
// (Measured on a B200: out of line, as a called function, every launch was 3-8% slower.)
template <int D, bool kPair, bool kSplit>
__device__ __forceinline__ bool item_epilogue(const AttnParams& p, const TMaps& tm, uint32_t sbase, const Bars& bars,
                                           uint32_t trow, uint32_t tO, int warp, int lane, int row, int lane_t,
                                           bool remote, uint32_t prog_word, uint32_t& n_fin, uint32_t& stg_ph,
                                           uint32_t& n_xch,
                                           volatile int* abort_flag, const Item& it, float l, float m_used,
                                           int n_kept, uint32_t total_pv) {
  using C = Cfg<D, kPair, kSplit>;
  const uint64_t tmo = p.timeout_ns;
  bool ok = true;
  const int q_row = (lane_t ? it.q_start[1] : it.q_start[0]) + row;
  const bool lane_valid = lane_t ? it.valid[1] : it.valid[0];
  // Overlapped launch: nothing is written (or, merging, read) before the kernel before it has completed,
  // unless the caller promised that kernel touches none of this launch's outputs.
  if (p.pdl_wait_epi) pdl_wait();
  // Epilogue: O / l and lse for the rows of this lane.
  if (kSplit && lane_valid) {
    ok = split_epilogue<D>(p, tm, sbase, bars, trow, it, q_row, row, warp, lane, lane_t, q_row < it.q_end, l, m_used,
                           n_kept, total_pv, n_xch, abort_flag);
    ++n_xch;
    if (!ok) return false;
  } else if (lane_valid) {
    const bool row_ok = q_row < it.q_end;  // inside S and inside the pair's shard
    void* obase = p.o;
    int orow = q_row, orows = p.S;
    if (p.n_shards > 1) {  // the pair's sequence shard
      obase = p.o_shard[it.shard];
      orow = q_row - it.shard * p.shard_rows;
      orows = p.shard_rows;
    }
    const size_t o_idx = (((size_t)it.b * orows + orow) * p.H + it.h) * D;
    if (p.o_merge) {
      // Merge into the running result: rows that saw no key of this launch's range keep it unchanged.
      if (n_kept > 0) {
        ok = merge_epilogue<D, kPair, kSplit>(p, tm, sbase, bars, tO, it, q_row, row, warp, lane, lane_t, row_ok, l,
                                      m_used, total_pv, stg_ph, abort_flag);
        if (!ok) return false;
      }
    } else if (n_kept > 0) {
      ok = mbar_wait(bars.pv_done(lane_t), (total_pv - 1) & 1, tmo, ERR_TIMEOUT_PV_DONE, abort_flag, p.err);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) return false;
      tc_fence_after();
      // A row that never saw a visible key is exactly 0 (the FMA-pipe exponentials of its masked
      // entries are tiny but not zero).
      const float inv_l = (l > 0.f && m_used != -INFINITY) ? 1.f / l : 0.f;
      // O / l leaves through a per-warp staging buffer in shared memory, 128 bytes of each of the warp's
      // 32 rows at a time (32 fp32 or 64 bf16 values, 128-byte swizzle), and a TMA store of that box:
      // whole 128-byte lines reach L2, and rows past the shard's (or S's) end are not written.
      const uint32_t stg0 = sbase + C::kStgOff + (uint32_t)warp * (4096u * C::kStgBufs);
      const CUtensorMap* omap = &tm.o[p.n_shards > 1 ? it.shard : 0];
      const int row0 = q_row - row + (warp & 3) * 32 - (p.n_shards > 1 ? it.shard * p.shard_rows : 0);
      const int n_chunks = p.o_f32 ? D / 32 : D / 64;
#pragma unroll 1
      for (int c = 0; c < n_chunks; ++c) {
        uint32_t v[32];
        if (p.o_f32) {
          tmem_ld32(tO + c * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * inv_l);
        } else {
          uint32_t o2[32];
          tmem_ld32(tO + c * 64, v);
          tmem_ld32(tO + c * 64 + 32, o2);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e)
            v[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * inv_l, __uint_as_float(v[2 * e + 1]) * inv_l);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            v[16 + e] = pack_bf16x2(__uint_as_float(o2[2 * e]) * inv_l, __uint_as_float(o2[2 * e + 1]) * inv_l);
        }
        const uint32_t stg = stg0 + 4096u * (uint32_t)(c % C::kStgBufs);
        if (c >= C::kStgBufs) {  // the store that last used this buffer must have read it
          if (lane == 0) {
            if (C::kStgBufs == 2)
              bulk_wait_read_but1();
            else
              bulk_wait_read_all();
          }
          __syncwarp();
        }
#pragma unroll
        for (int e = 0; e < 8; ++e)
          st_shared_v4(stg + (uint32_t)lane * 128u + (uint32_t)(((e ^ (lane & 7)) << 4)), v[4 * e], v[4 * e + 1],
                       v[4 * e + 2], v[4 * e + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_4d(omap, stg, c * (p.o_f32 ? 32 : 64), it.h, row0, it.b);
          bulk_commit_group();
        }
      }
      if (lane == 0) bulk_wait_read_all();  // the buffers are free for the next item
      __syncwarp();
    } else if (row_ok) {
      if (p.o_f32) {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(obase) + o_idx);
        for (int e = 0; e < D / 4; ++e) dst[e] = make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(obase) + o_idx);
        for (int e = 0; e < D / 8; ++e) dst[e] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    if (row_ok && p.lse && !p.o_merge)
      p.lse[((size_t)it.b * p.H + it.h) * p.S + q_row] =
          (l > 0.f && m_used != -INFINITY) ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
  }
  // This warp has read out O (with kSplit, both lanes' O): its progress word moves on to the next item.
  tc_fence_before();
  __syncwarp();
  ++n_fin;
  if (lane == 0) {
    if (remote)
      st_release_cluster(prog_word, n_fin);
    else
      st_release_cta(prog_word, n_fin);
    if (kSplit) st_release_cta(bars.prog(lane_t ^ 1, warp), n_fin);
  }
  return true;
}

// ------------------------------------------------------------------------------------------------
// Softmax + epilogue: 4 warps per lane, one query row per thread.
// ------------------------------------------------------------------------------------------------
template <int D, bool kPair, bool kSplit>
__device__ void run_softmax(const AttnParams& p, const TMaps& tm, uint32_t sbase, const Bars& bars, const ItemRing& ir,
                            uint32_t tmem, int lane_t, volatile int* abort_flag) {
  using C = Cfg<D, kPair, kSplit>;
  // A pair's rank 1 hands its P and its O read-outs to rank 0's barriers and progress words.
  const bool remote = kPair && cluster_rank() != 0;
  const uint32_t p_full_bar = remote ? map_shared(bars.p_full(lane_t), 0) : bars.p_full(lane_t);
  // this warp's progress word for lane t: pair, 4 per CTA; split, one per warp of the CTA
  const int prog_k = kPair ? 4 * (int)cluster_rank() + ((threadIdx.x >> 5) & 3)
                           : (kSplit ? (int)(threadIdx.x >> 5) : (int)((threadIdx.x >> 5) & 3));
  const uint32_t prog_word = remote ? map_shared(bars.prog(lane_t, prog_k), 0) : bars.prog(lane_t, prog_k);
  uint32_t n_fin = 0;  // items whose epilogue this warp has finished

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
  uint32_t stg_ph = 0;  // bit b: phase of this warp's staging-buffer-b load barrier (merging epilogues)
  uint32_t n_xch = 0;   // split keys: epilogue hand-offs this warp has taken part in
  bool ok = true;
  // Split-key launches (block-sparse, items of few kept tiles) run an item's epilogue after this warp's
  // first kept step of the next item (S to P touch only the S columns, not O): the tensor core then has
  // that step's P V queued by the time O has been read out, and the step no longer waits behind the
  // epilogue.  Measured on a B200: block-sparse +5.8%; dense and causal launches -5 to -9% (the state kept
  // through the step loop costs their softmax registers), so they finish each item at once.
  constexpr bool kDefer = kSplit;
  int prev_w = -1;  // kDefer: the item whose epilogue is pending, or -1
  float prev_l = 0.f, prev_m = -INFINITY;
  int prev_kept = 0;
  uint32_t prev_pv = 0;
  auto epilogue = [&](const Item& it_, float l_, float m_, int kept_, uint32_t pv_) -> bool {
    return item_epilogue<D, kPair, kSplit>(p, tm, sbase, bars, trow, tO, warp, lane, row, lane_t, remote, prog_word,
                                           n_fin, stg_ph, n_xch, abort_flag, it_, l_, m_, kept_, pv_);
  };
  auto finish = [&]() -> bool {  // the pending epilogue
    const Item it_ = decode_item<kPair, kSplit>(p, prev_w);
    prev_w = -1;
    return epilogue(it_, prev_l, prev_m, prev_kept, prev_pv);
  };

  for (int n_item = 0;; ++n_item) {
    int w;
    ok = ring_read(ir, n_item, w, tmo, abort_flag, p.err, remote);
    if (!ok || w < 0) break;
    __syncwarp();
    if (lane == 0) smem_counter_add_release(ir.used0 + 4u * warp, 1u);  // this warp is done with the slot
    const Item it = decode_item<kPair, kSplit>(p, w);
    StepIter st;
    st.init(p, it, kSplit);
    const int q_row = (lane_t ? it.q_start[1] : it.q_start[0]) + row;
    const int lim_row = p.causal ? min(p.kv_lim, q_row + 1) : p.kv_lim;
    float m_used = -INFINITY;  // running maximum of the scaled scores, log2 units
    float l = 0.f;             // running sum of exp2(score - m_used)
    int n_kept = 0;
    int kv_start;
    bool k0, k1;
    while (st.next(kv_start, k0, k1)) {
      if (!(lane_t == 0 ? k0 : k1)) continue;  // this lane skips the step
      ok = mbar_wait(bars.s_full(lane_t), s_full_ph, tmo, ERR_TIMEOUT_S_FULL, abort_flag, p.err);
      ok = __all_sync(0xffffffffu, ok);
      s_full_ph ^= 1;
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr[c]);
      tmem_wait_ld();
#define SV(i) __uint_as_float(sr[(i) >> 5][(i) & 31])
      // Keys past the KV range, past S, past the end of the tile's shard, or (causal) after this query:
      // -inf.
      const int n_valid = min(lim_row, st.key_end) - kv_start;
      if (__any_sync(0xffffffffu, n_valid < kTile)) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (c * 32 + e >= n_valid) sr[c][e] = __float_as_uint(-INFINITY);
      }
      const f2 sc2 = {scale_log2, scale_log2};
      // 2^(s * scale - m) for the two columns of pair e of the row (of every 8 pairs, kPoly go through the
      // FMA-pipe polynomial and the rest through ex2.approx).
      constexpr int kPoly = poly_pairs<kSplit>();
      auto exp_pair = [&](int i, int e, f2 nm2) -> f2 {
        const f2 x = ffma2(f2{SV(i), SV(i + 1)}, sc2, nm2);
        f2 pr;
        if (((e >> 1) & 7) >= 8 - kPoly) {
          pr = exp2_poly2(x);
        } else {
          pr.x = ex2_approx(x.x);
          pr.y = ex2_approx(x.y);
        }
        return pr;
      };
      // P = 2^(s * scale - m), bf16, two per column over the last 64 columns of S_t (the A operand of
      // O += P V), each quarter stored as soon as it is packed; returns the row sum.  With the maximum
      // (mx4 given), the row's maximum is formed in the same pass: four chains of three-input maxima on
      // the ALU pipe, beside the FMA and MUFU work.  P over the last 64 columns leaves S's first 64 columns
      // in TMEM, and the pass reads the last 64 from registers last, so a pass can be redone.
      float mx4[4];
      auto exp_pass = [&](float neg_m, auto with_max) -> float {
        const f2 nm2 = {neg_m, neg_m};
        f2 acc[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
        for (int quarter = 0; quarter < 4; ++quarter) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int i = quarter * 32 + e;
            if constexpr (decltype(with_max)::value) {
              const int k = (e >> 1) & 3;
              mx4[k] = (quarter == 0 && e < 8) ? fmaxf(SV(i), SV(i + 1)) : fmax3f(mx4[k], SV(i), SV(i + 1));
            }
            const f2 pr = exp_pair(i, e, nm2);
            acc[(e >> 1) & 3] = fadd2(acc[(e >> 1) & 3], pr);
            pk[e >> 1] = pack_bf16x2(pr.x, pr.y);
          }
          tmem_st16(tS + kPCol + quarter * 16, pk);
        }
        const f2 acc4 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
        return acc4.x + acc4.y;
      };
      float rowsum;
      if (kSplit || n_kept == 0) {
        // The row maximum first, then the exponentials against it: the item's first step for this lane,
        // and every step of split-key items (each lane has half the steps, and measured, the speculative
        // pass below costs them more than the maximum's latency).
        float mx8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = fmaxf(SV(2 * k), SV(2 * k + 1));
#pragma unroll
        for (int i = 16; i < 128; i += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k) mx8[k] = fmax3f(mx8[k], SV(i + 2 * k), SV(i + 2 * k + 1));
        const float m_tile =
            fmax3f(fmax3f(mx8[0], mx8[1], mx8[2]), fmax3f(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])) * scale_log2;
        const bool grow = m_tile > m_used + kRescaleThreshold;
        float alpha = 1.f;
        if (grow) {
          alpha = ex2_approx(m_used - m_tile);  // 0 when nothing was seen before
          l *= alpha;
          m_used = m_tile;
        }
        rowsum = exp_pass(m_used == -INFINITY ? 0.f : -m_used, std::false_type{});
        // O row *= alpha, after the pass (the S registers are free by then): the previous O += P V of
        // this lane has completed (the S_t commit that signalled this step fires only after every earlier
        // MMA of its issuer), and the next one waits for this thread's P, which is announced only after
        // these stores have completed.
        if (n_kept > 0 && __any_sync(0xffffffffu, grow)) rescale_o_row<D>(tO, alpha);
      } else {
        // Later steps: the exponentials run against the running maximum while this tile's maximum is
        // formed in the same pass, so they need not wait for it.  Where it grew by more than 2^8 (log2
        // units) the pass was against too small a reference: that row's sum and O are rescaled and the warp
        // redoes the pass against the new maximum (S's first 64 columns reloaded from TMEM, the last 64 still
        // in registers), which is rare after a row's first tiles.  Otherwise P <= 2^8 stays finite in bf16
        // and the result is exact after the final O / l.
        rowsum = exp_pass(m_used == -INFINITY ? 0.f : -m_used, std::true_type{});
        const float m_tile = fmaxf(fmax3f(mx4[0], mx4[1], mx4[2]), mx4[3]) * scale_log2;
        const bool grow = m_tile > m_used + kRescaleThreshold;
        if (__any_sync(0xffffffffu, grow)) {
          float alpha = 1.f;
          if (grow) {
            alpha = ex2_approx(m_used - m_tile);  // 0 when nothing was seen before
            l *= alpha;
            m_used = m_tile;
          }
          // O row *= alpha.  The previous O += P V of this lane has completed (the S_t commit that
          // signalled this step fires only after every earlier MMA of its issuer), and the next one
          // waits for this thread's P.
          rescale_o_row<D>(tO, alpha);
#pragma unroll
          for (int c = 0; c < 2; ++c) tmem_ld32(tS + c * 32, sr[c]);
          tmem_wait_ld();
          if (n_valid < kTile) {
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (c * 32 + e >= n_valid) sr[c][e] = __float_as_uint(-INFINITY);
          }
          rowsum = exp_pass(m_used == -INFINITY ? 0.f : -m_used, std::false_type{});
        }
      }
#undef SV
      l += rowsum;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (remote)
          mbar_arrive_cluster(p_full_bar);
        else
          mbar_arrive(p_full_bar);
      }
      ++n_kept;
      ++total_pv;
      if constexpr (kDefer) {
        if (prev_w >= 0) {  // the previous item's epilogue, now that this step's P is handed over
          ok = finish();
          if (!ok) break;
        }
      }
    }
    if (!ok) break;
    if constexpr (kDefer) {
      if (prev_w >= 0) {  // the previous item's epilogue is pending and this item kept no step here
        ok = finish();
        if (!ok) break;
      }
      prev_w = w;
      prev_l = l;
      prev_m = m_used;
      prev_kept = n_kept;
      prev_pv = total_pv;
    } else {
      ok = epilogue(it, l, m_used, n_kept, total_pv);
      if (!ok) break;
    }
  }
  if constexpr (kDefer) {
    if (ok && prev_w >= 0) finish();
  }
  if (lane == 0) bulk_wait_all();  // every O store of this warp has landed before the CTA exits
  __syncwarp();
}

template <int D, bool kPair, bool kSplit>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ TMaps tm, const __grid_constant__ AttnParams p) {
  using C = Cfg<D, kPair, kSplit>;
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
  bars.drain = bars.pv_done0 + 16;
  bars.stg_full0 = bars.drain + 8;
  bars.prog0 = smem_u32(smem + C::kProgOff);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  ItemRing ir;
  ir.pub = smem_u32(smem + C::kMiscOff + 8);
  ir.used0 = smem_u32(smem + C::kMiscOff + 16);
  ir.ids = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 48);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bars.q_full, 1);
    mbar_init(bars.q_empty, 2);  // one arrival per MMA warp
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bars.kv_full(s), 1);
      mbar_init(bars.kv_empty(s), 2);  // one arrival per MMA warp
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bars.s_full(t), 1);
      mbar_init(bars.p_full(t), C::kRowWarps);  // one arrival per softmax warp of the lane (pair: both CTAs)
      mbar_init(bars.pv_done(t), 1);
    }
    for (int k = 0; k < 16; ++k)  // the progress words of both lanes
      *reinterpret_cast<volatile uint32_t*>(smem + C::kProgOff + 4 * k) = 0u;
    mbar_init(bars.drain, 2);
    for (int k = 0; k < 16; ++k) mbar_init(bars.stg_full0 + 8u * k, 1);
    if (kSplit)  // the lanes' epilogue hand-off counters
      for (int k = 0; k < 4; ++k) *reinterpret_cast<volatile uint32_t*>(smem + C::kXcntOff + 4 * k) = 0u;
    *abort_flag = 0;
    *reinterpret_cast<volatile uint32_t*>(smem + C::kMiscOff + 8) = 0u;  // items published
    for (int k = 0; k < 8; ++k)                                          // items read, per softmax warp
      *reinterpret_cast<volatile uint32_t*>(smem + C::kMiscOff + 16 + 4 * k) = 0u;
    fence_mbar_init();
  }
  if (warp == kWarpProducer && lane == 0) {
    for (int r = 0; r < p.n_shards; ++r) {
      tma_prefetch_desc(&tm.q[r]);
      if (kPair) {
        tma_prefetch_desc(&tm.k64[r]);
      } else {
        tma_prefetch_desc(&tm.k[r]);
      }
      tma_prefetch_desc(&tm.v[r]);
    }
  }
  if (warp == kWarpMma) {  // a pair allocates the same 512 columns in both CTAs, from the same warp
    if constexpr (kPair) {
      tmem_alloc_pair(smem_u32(tmem_holder), 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_holder), 512);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  // a pair: both CTAs' barriers are initialised before either CTA arrives on the other's
  if constexpr (kPair) cluster_sync(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  if (p.pdl) {
    // Set up: the next launch may start on the SMs this grid frees.  A launch whose tile or item list the
    // kernel before it wrote waits for that kernel here; otherwise it waits before its first epilogue
    // (run_softmax) or, when the caller promised that the kernel before touches none of its outputs, not
    // at all (a merging launch always waits before reading its running result).
    if (threadIdx.x == 0) pdl_launch_dependents();
    if (p.pdl_wait_start) pdl_wait();
  }

  if (warp < 8) {
    regs_inc<kRegsSoftmax>();
    run_softmax<D, kPair, kSplit>(p, tm, smem_u32(smem), bars, ir, tmem, warp >> 2, abort_flag);
  } else {
    regs_dec<kRegsControl>();
    if (warp == kWarpProducer) {
      run_producer<D, kPair, kSplit>(p, tm, smem, bars, ir, abort_flag);
    } else if ((warp == kWarpMma || warp == kWarpMma + 1) && (!kPair || cluster_rank() == 0)) {
      run_mma<D, kPair, kSplit>(p, smem, bars, ir, tmem, warp - kWarpMma, abort_flag);  // a pair's MMAs: rank 0
    }
    __syncwarp();
  }
  tc_fence_before();
  // a pair: neither CTA leaves (or frees TMEM) while the other may still touch its shared memory or the
  // pair's MMAs may still write its TMEM (rank 0 drained them before arriving here)
  if constexpr (kPair) cluster_sync(); else __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    if constexpr (kPair) tmem_dealloc_pair(tmem, 512); else tmem_dealloc(tmem, 512);
  }
  // The last CTA to finish returns this launch's work counter to zero for the next launch that draws
  // the same slot (every CTA has made its last claim before it gets here).
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.sched + 1, 1u) == gridDim.x - 1) {
      atomicExch(p.sched, 0u);
      atomicExch(p.sched + 1, 0u);
    }
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
  p.n_shards = 1;
  p.shard_rows = p.S;
  p.tiles_per_shard = (p.S + kTile - 1) / kTile;
  p.pairs_per_shard = p.n_qpairs;
  p.q_shard[0] = q;
  p.k_shard[0] = k;
  p.v_shard[0] = v;
  p.o_shard[0] = p.o;
  return launch_attn_sharded(p, stream);
}

// CTA pairs (one cluster of two CTAs per TPC) for D = 128 without a mask or item list; SP_ATTN_PAIR=0 in the
// environment keeps every launch on single CTAs.
static bool pair_enabled() {
  static int on = -1;
  if (on < 0) {
    const char* e = std::getenv("SP_ATTN_PAIR");
    on = (e && e[0] == '0') ? 0 : 1;
  }
  return on == 1;
}

// Split keys (both lanes on one query tile, alternate kept key tiles) for block-sparse launches that write
// their result (not merging into a running one); SP_ATTN_SPLIT=0 in the environment walks the union of two
// query tiles' lists instead.
static bool split_enabled() {
  static int on = -1;
  if (on < 0) {
    const char* e = std::getenv("SP_ATTN_SPLIT");
    on = (e && e[0] == '0') ? 0 : 1;
  }
  return on == 1;
}

template <int D, bool kPair, bool kSplit>
static sp_status launch_kernel(const TMaps& tm, const AttnParams& p, int grid, cudaStream_t stream, int dev) {
  using C = Cfg<D, kPair, kSplit>;
  static int regs_ok[kMaxDevices] = {};
  static bool attr_set[kMaxDevices] = {};
  // The warpgroups re-divide the registers the CTA was launched with; a kernel built with another
  // per-thread count would make that division wait forever, so it is never launched.
  if (regs_ok[dev] == 0) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, attn_fwd_kernel<D, kPair, kSplit>) != cudaSuccess) return SP_ERR_CUDA;
    regs_ok[dev] = fa.numRegs == kRegsLaunch ? 1 : -1;
  }
  if (regs_ok[dev] < 0) return SP_ERR_UNSUPPORTED;
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(attn_fwd_kernel<D, kPair, kSplit>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
        cudaSuccess)
      return SP_ERR_CUDA;
    attr_set[dev] = true;
  }
  if (kPair || p.pdl) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int n = 0;
    if (kPair) {
      attr[n].id = cudaLaunchAttributeClusterDimension;
      attr[n].val.clusterDim.x = 2;
      attr[n].val.clusterDim.y = 1;
      attr[n].val.clusterDim.z = 1;
      ++n;
    }
    if (p.pdl) {
      attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[n].val.programmaticStreamSerializationAllowed = 1;
      ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    if (cudaLaunchKernelEx(&cfg, attn_fwd_kernel<D, kPair, kSplit>, tm, p) != cudaSuccess) return SP_ERR_CUDA;
  } else {
    attn_fwd_kernel<D, kPair, kSplit><<<grid, kThreads, C::kSmemBytes, stream>>>(tm, p);
  }
  return cudaGetLastError() == cudaSuccess ? SP_OK : SP_ERR_CUDA;
}

// Rows [0, rows) of heads [h0, h1) of every batch: O = 0 (16-byte stores; each head's D values are 128 or
// 256 bytes) and lse = -inf.  For the query rows of a causal partial launch that no key of its range
// reaches.
__global__ void __launch_bounds__(256) fill_empty_rows_kernel(void* __restrict__ o, int o_elem_bytes,
                                                              float* __restrict__ lse, int B, int S, int H, int D,
                                                              int h0, int h1, int rows) {
  const long long per_row = (long long)(h1 - h0) * D * o_elem_bytes / 16;  // 16-byte chunks per (b, s)
  const long long n_o = (long long)B * rows * per_row;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n_o; i += stride) {
    const long long bs = i / per_row, c = i % per_row;
    const long long b = bs / rows, s = bs % rows;
    uint8_t* row = static_cast<uint8_t*>(o) + (((b * S + s) * H + h0) * (long long)D) * o_elem_bytes;
    reinterpret_cast<uint4*>(row)[c] = make_uint4(0u, 0u, 0u, 0u);
  }
  if (lse) {
    const long long n_l = (long long)B * (h1 - h0) * rows;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n_l; i += stride) {
      const long long bh = i / rows, s = i % rows;
      const long long b = bh / (h1 - h0), h = h0 + bh % (h1 - h0);
      lse[(b * H + h) * S + s] = -INFINITY;
    }
  }
}

sp_status launch_attn_sharded(const AttnParams& p_in, cudaStream_t stream) {
  AttnParams p = p_in;
  if (p.n_shards < 1 || p.n_shards > kMaxShards || p.shard_rows < 1 || (long long)p.n_shards * p.shard_rows != p.S ||
      p.tiles_per_shard != (p.shard_rows + kTile - 1) / kTile || p.pairs_per_shard != (p.tiles_per_shard + 1) / 2 ||
      p.n_qpairs != p.n_shards * p.pairs_per_shard)
    return SP_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SP_ERR_CUDA;
  const int sms = num_sms(dev);
  const int overlap = launch_overlap();
  p.pdl = overlap > 0 ? 1 : 0;
  p.pdl_wait_start = (p.pdl && (p.row_ptr || p.item_list)) ? 1 : 0;  // lists built by the kernel just before
  p.pdl_wait_epi = (p.pdl && (overlap == 1 || p.o_merge)) ? 1 : 0;    // a running result is always waited for
  const bool pair = p.D == 128 && !p.row_ptr && !p.item_list && sms >= 2 && pair_enabled();
  TMaps tm{};  // the kernel argument (copied at launch)
  for (int r = 0; r < p.n_shards; ++r)
    if (!encode_bshd_tmap(&tm.q[r], p.q_shard[r], p.B, p.shard_rows, p.H, p.D) ||
        !encode_bshd_tmap(&tm.k[r], p.k_shard[r], p.B, p.shard_rows, p.H, p.D) ||
        !encode_bshd_tmap(&tm.v[r], p.v_shard[r], p.B, p.shard_rows, p.H, p.D) ||
        (pair && !encode_bshd_tmap(&tm.k64[r], p.k_shard[r], p.B, p.shard_rows, p.H, p.D, 64)) ||
        !encode_o_tmap(&tm.o[r], p.o_shard[r], p.B, p.shard_rows, p.H, p.D, p.o_f32 != 0))
      return SP_ERR_CUDA;
  if (pair) {
    // work units of four query tiles (two per CTA of the pair), per shard
    p.pairs_per_shard = (p.tiles_per_shard + 3) / 4;
    p.n_qpairs = p.n_shards * p.pairs_per_shard;
    long long items = 0;
    for (int c = 0; c < p.n_chunks; ++c) {
      p.chunk_item0[c] = (int)items;
      items += (long long)p.B * (p.chunk_h0[c + 1] - p.chunk_h0[c]) * p.n_qpairs;
    }
    p.chunk_item0[p.n_chunks] = (int)items;
    if (items > 0x7fffffffLL) return SP_ERR_INVALID_ARG;
    p.n_items = (int)items;
  }
  // A causal launch over keys from kv_begin: queries before kv_begin see none of them.  Whole leading
  // work units of such rows get no item; their rows are written here (O = 0, lse = -inf) at HBM speed,
  // except when the launch merges into a running result, which those rows keep unchanged.
  p.qp_skip = 0;
  if (p.causal && p.kv_begin > 0 && p.n_shards == 1 && !p.item_list && !p.row_ptr) {
    const int unit_rows = (pair ? 4 : 2) * kTile;
    p.qp_skip = p.kv_begin / unit_rows < p.n_qpairs ? p.kv_begin / unit_rows : p.n_qpairs;
    const int rows = p.qp_skip * unit_rows < p.S ? p.qp_skip * unit_rows : p.S;
    if (rows > 0 && !p.o_merge) {
      const int h0 = p.chunk_h0[0], h1 = p.chunk_h0[p.n_chunks];
      const long long n = (long long)p.B * rows * (h1 - h0) * p.D * (p.o_f32 ? 4 : 2) / 16;
      long long blocks = (n + 255) / 256;
      if (blocks > (long long)sms * 8) blocks = (long long)sms * 8;
      if (blocks < 1) blocks = 1;
      fill_empty_rows_kernel<<<(int)blocks, 256, 0, stream>>>(p.o, p.o_f32 ? 4 : 2, p.lse, p.B, p.S, p.H, p.D, h0, h1,
                                                              rows);
      if (cudaGetLastError() != cudaSuccess) return SP_ERR_CUDA;
    }
    long long items = 0;
    for (int c = 0; c < p.n_chunks; ++c) {
      p.chunk_item0[c] = (int)items;
      items += (long long)p.B * (p.chunk_h0[c + 1] - p.chunk_h0[c]) * (p.n_qpairs - p.qp_skip);
    }
    p.chunk_item0[p.n_chunks] = (int)items;
    p.n_items = (int)items;
  }
  if (p.n_items <= 0) return SP_OK;
  {
    static unsigned int* sched_base[kMaxDevices] = {};
    static std::atomic<unsigned int> launch_seq{0};
    if (!sched_base[dev]) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_attn_sched) != cudaSuccess || !ptr) return SP_ERR_CUDA;
      sched_base[dev] = static_cast<unsigned int*>(ptr);
    }
    p.sched = sched_base[dev] + 2 * (launch_seq.fetch_add(1) % kSchedSlots);
  }
  if (pair) {
    const long long want = 2LL * p.n_items;
    const int grid = (int)(want < (sms & ~1) ? want : (sms & ~1));
    return launch_kernel<128, true, false>(tm, p, grid, stream, dev);
  }
  const int grid = p.n_items < sms ? p.n_items : sms;
  const bool split = p.row_ptr && !p.o_merge && p.n_shards == 1 && split_enabled();
  if (split)
    return p.D == 128 ? launch_kernel<128, false, true>(tm, p, grid, stream, dev)
                      : launch_kernel<64, false, true>(tm, p, grid, stream, dev);
  return p.D == 128 ? launch_kernel<128, false, false>(tm, p, grid, stream, dev)
                    : launch_kernel<64, false, false>(tm, p, grid, stream, dev);
}

}  // namespace spattn
