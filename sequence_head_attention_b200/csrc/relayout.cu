// relayout.cu -- the Ulysses all-to-all layout permutation between P rank buffers of one GPU.
//
// "HCMS: Head-Chunked Multi-Stream Pipeline ...", abstract (all-to-all based sequence parallelism) and
// "db-SP ...", abstract (parallelism along the head dimension, as in Ulysses).  Before attention, rank r
// holds positions [r S/P, (r+1) S/P) of every head; after it, rank r holds every position of heads
// [r H/P, (r+1) H/P):
//   seq -> head:  out_r[b, s, h', :] = in_{s / (S/P)}[b, s % (S/P), r H/P + h', :]
//   head -> seq:  out_r[b, s', h, :] = in_{h / (H/P)}[b, r S/P + s', h % (H/P), :]
// When the P ranks are separate processes, the all-to-all itself is a collective (NCCL) between contiguous
// per-destination blocks, and each rank's local halves are copies of its own shard:
//   split heads:  out_r[b, s, h', :] = in[b, s, r H/P + h0 + h', :]  (before the exchange)
//   merge heads:  out[b, s, r H/P + h0 + h', :] = in_r[b, s, h', :]  (after the way back)
// for h' < n of a sub-range [h0, h0 + n) of every rank's head group (the whole group, or one stage of a
// chunked exchange).
// All four move contiguous runs of (H/P) * D elements: one warp copies one run with 16-byte vector loads
// and stores, up to 4 KB per lane group in flight, so both sides are fully coalesced.  Bit-exact.
#include <cstdint>

#include "sp_internal.h"

namespace spattn {
namespace {

struct RankPtrs {
  const uint8_t* in[SP_MAX_RANKS];
  uint8_t* out[SP_MAX_RANKS];
};

enum RelayoutMode { kHeadToSeq = 0, kSeqToHead = 1, kSplitHeads = 2, kMergeHeads = 3 };

template <int kMode>
__global__ void __launch_bounds__(256) relayout_kernel(const __grid_constant__ RankPtrs rp, int P, int B,
                                                       int S, int H, long long run_bytes, long long row_bytes,
                                                       long long group_bytes, long long sub_off) {
  const int Sl = S / P;
  const long long n_runs = (long long)P * B * S;
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  const int nvec = (int)(run_bytes / 16);
  for (long long run = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5; run < n_runs; run += warps) {
    const uint8_t* src;
    uint8_t* dst;
    if (kMode == kSplitHeads) {
      // run = (r, b, s): destination out_r[b, s, :, :] (S here is the rank's own sequence length); the source
      // is the sub-range of rank r's head group in the row of (b, s)
      const long long bs = run % ((long long)B * S);
      const int r = (int)(run / ((long long)B * S));
      src = rp.in[0] + bs * row_bytes + r * group_bytes + sub_off;
      dst = rp.out[r] + bs * run_bytes;
    } else if (kMode == kMergeHeads) {
      // run = (b, s, r): destination the sub-range of rank r's head group in out[b, s]
      const int r = (int)(run % P);
      const long long bs = run / P;
      src = rp.in[r] + bs * run_bytes;
      dst = rp.out[0] + bs * row_bytes + r * group_bytes + sub_off;
    } else if (kMode == kSeqToHead) {
      // run = (r, b, s): destination out_r[b, s, :, :], contiguous in s
      const int s = (int)(run % S);
      const long long rb = run / S;
      const int b = (int)(rb % B);
      const int r = (int)(rb / B);
      src = rp.in[s / Sl] + (((long long)b * Sl + (s % Sl)) * P + r) * run_bytes;  // heads r*H/P.. of row
      dst = rp.out[r] + ((long long)b * S + s) * run_bytes;
    } else {
      // run = (r, b, s', g): destination out_r[b, s', g*H/P : (g+1)*H/P, :], contiguous in g
      const int g = (int)(run % P);
      const long long rest = run / P;
      const int sl = (int)(rest % Sl);
      const long long rb = rest / Sl;
      const int b = (int)(rb % B);
      const int r = (int)(rb / B);
      src = rp.in[g] + ((long long)b * S + (long long)r * Sl + sl) * run_bytes;
      dst = rp.out[r] + (((long long)b * Sl + sl) * P + g) * run_bytes;
    }
    // up to 8 vectors per lane in flight (a run of up to 4 KB in one round), loads before stores
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    int v = lane;
    for (; v + 224 < nvec; v += 256) {
      uint4 x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = __ldg(s4 + v + 32 * u);
#pragma unroll
      for (int u = 0; u < 8; ++u) d4[v + 32 * u] = x[u];
    }
    {
      uint4 x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (v + 32 * u < nvec) x[u] = __ldg(s4 + v + 32 * u);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (v + 32 * u < nvec) d4[v + 32 * u] = x[u];
    }
  }
}

}  // namespace

static sp_status launch_runs(const RankPtrs& rp, int mode, int P, int B, int S, int H, int D, int elem_bytes,
                             cudaStream_t stream, int h0 = 0, int n_heads = -1) {
  // A run is the H/P heads of one (rank, b, s): H/P * D elements.  In the seq-sharded layout a row of
  // H heads holds P consecutive runs, which is what the kernel's "* P + r" indexing uses.  The head-group
  // copies move a sub-range [h0, h0 + n_heads) of each group.
  const long long row_bytes = (long long)H * D * elem_bytes, group_bytes = row_bytes / P;
  const long long run_bytes = n_heads < 0 ? group_bytes : (long long)n_heads * D * elem_bytes;
  const long long sub_off = (long long)h0 * D * elem_bytes;
  const long long n_runs = (long long)P * B * S;
  if (n_runs == 0) return SP_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SP_ERR_CUDA;
  long long blocks = (n_runs + 7) / 8;
  const long long cap = (long long)num_sms(dev) * 8;
  if (blocks > cap) blocks = cap;
  switch (mode) {
    case kSeqToHead: relayout_kernel<kSeqToHead><<<(unsigned)blocks, 256, 0, stream>>>(rp, P, B, S, H, run_bytes, row_bytes,
                                                                   group_bytes, sub_off); break;
    case kHeadToSeq: relayout_kernel<kHeadToSeq><<<(unsigned)blocks, 256, 0, stream>>>(rp, P, B, S, H, run_bytes, row_bytes,
                                                                   group_bytes, sub_off); break;
    case kSplitHeads: relayout_kernel<kSplitHeads><<<(unsigned)blocks, 256, 0, stream>>>(rp, P, B, S, H, run_bytes, row_bytes,
                                                                   group_bytes, sub_off); break;
    default: relayout_kernel<kMergeHeads><<<(unsigned)blocks, 256, 0, stream>>>(rp, P, B, S, H, run_bytes, row_bytes,
                                                                   group_bytes, sub_off); break;
  }
  return cudaGetLastError() == cudaSuccess ? SP_OK : SP_ERR_CUDA;
}

sp_status launch_relayout(const void* const* in_ranks, void* const* out_ranks, int P, int B, int S,
                          int H, int D, int elem_bytes, bool seq_to_head, cudaStream_t stream) {
  RankPtrs rp = {};
  for (int r = 0; r < P; ++r) {
    rp.in[r] = static_cast<const uint8_t*>(in_ranks[r]);
    rp.out[r] = static_cast<uint8_t*>(out_ranks[r]);
  }
  return launch_runs(rp, seq_to_head ? kSeqToHead : kHeadToSeq, P, B, S, H, D, elem_bytes, stream);
}

sp_status launch_head_groups(const void* const* in, void* const* out, bool split, int P, int B, int S, int H, int D,
                             int h0, int n_heads, int elem_bytes, cudaStream_t stream) {
  RankPtrs rp = {};
  const int n_in = split ? 1 : P, n_out = split ? P : 1;
  for (int r = 0; r < n_in; ++r) rp.in[r] = static_cast<const uint8_t*>(in[r]);
  for (int r = 0; r < n_out; ++r) rp.out[r] = static_cast<uint8_t*>(out[r]);
  return launch_runs(rp, split ? kSplitHeads : kMergeHeads, P, B, S, H, D, elem_bytes, stream, h0, n_heads);
}

}  // namespace spattn
