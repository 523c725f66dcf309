// tile_list.cu -- compacted per-(head, query tile) list of the key tiles a block mask keeps.
//
// "db-SP: Accelerating Sparse Attention ...", abstract: block-wise sparse attention whose dense blocks
// are irregularly placed and whose density varies across heads.  The attention kernel walks these lists
// so that dropped tiles are never loaded or multiplied.  Output is CSR: row (h, i) lists, in increasing
// order, every j with mask[h][i][j] != 0 -- fully determined, so it is compared bit for bit.
//
// Three small launches: count per row (one warp per row, ballots over 32 bytes at a time), an exclusive
// scan of the counts (one block), and the fill (one warp per row, ballot + popcount for each lane's slot).
#include <cstdint>

#include "sp_internal.h"
#include "sp_ptx.cuh"

namespace spattn {
namespace {

__global__ void __launch_bounds__(256) tile_count_kernel(const uint8_t* mask, int rows, int T, int32_t* counts) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint8_t* m = mask + (size_t)row * T;
  int c = 0;
  for (int j0 = 0; j0 < T; j0 += 32) {
    const int j = j0 + lane;
    const unsigned bal = __ballot_sync(0xffffffffu, j < T && m[j] != 0);
    c += __popc(bal);
  }
  if (lane == 0) counts[row] = c;
}

// Exclusive scan of counts[0..n) into row_ptr[0..n]; one block of 1024 threads.
__global__ void __launch_bounds__(1024) tile_scan_kernel(const int32_t* counts, int n, int32_t* row_ptr) {
  __shared__ int32_t warp_tot[32];
  const int tid = threadIdx.x;
  const int per = (n + 1023) / 1024;
  const int lo = min(n, tid * per), hi = min(n, lo + per);
  int local = 0;
  for (int i = lo; i < hi; ++i) local += counts[i];
  // inclusive scan of `local` over the block
  const int lane = tid & 31, warp = tid >> 5;
  int x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    warp_tot[lane] = t;
  }
  __syncthreads();
  int run = x - local + (warp > 0 ? warp_tot[warp - 1] : 0);  // exclusive prefix of this thread's segment
  for (int i = lo; i < hi; ++i) {
    row_ptr[i] = run;
    run += counts[i];
  }
  if (tid == 1023) row_ptr[n] = run;
}

__global__ void __launch_bounds__(256) tile_fill_kernel(const uint8_t* mask, int rows, int T, const int32_t* row_ptr,
                                                        int32_t* col_idx) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint8_t* m = mask + (size_t)row * T;
  int base = row_ptr[row];
  for (int j0 = 0; j0 < T; j0 += 32) {
    const int j = j0 + lane;
    const bool keep = j < T && m[j] != 0;
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (keep) col_idx[base + __popc(bal & ((1u << lane) - 1u))] = j;
    base += __popc(bal);
  }
}

// Work order of a block-sparse launch: the item ids (b * H + h) * NP + qp (a pair of query tiles 2 qp and
// 2 qp + 1 of head h), head by head, the heads with the most kept tiles first, and within each (b, h) the
// items with the most kept tiles first.  Head by head, the CTAs running at the same time work on one or two
// heads and share their K and V in L2 (sorting every item by its cost, across heads, put all heads in flight
// at once and multiplied the launch's DRAM reads seven-fold); densest heads first and longest items first
// within a head, the dynamically claimed last items of the launch are the sparsest head's short ones
// (longest-processing-time order; per-head densities vary several-fold).  One block per (b, h): its rank
// among the heads by total kept tiles (ties by id), then a counting sort of its NP items, histogram of the
// costs (0 .. 2T) in shared memory, exclusive offsets from the largest cost down, each item placed with a
// shared-memory atomic (items of equal cost land in any order; each item's arithmetic does not depend on it).
constexpr int kMaxOrderBins = 4096;
constexpr int kOrderThreads = 256;
__global__ void __launch_bounds__(kOrderThreads) item_order_kernel(const int32_t* row_ptr, int H, int T, int NP,
                                                                   int32_t* order) {
  __shared__ int32_t bins[kMaxOrderBins];
  __shared__ int32_t warp_tot[kOrderThreads / 32];
  __shared__ int32_t rank_part[kOrderThreads / 32];
  const int seg = blockIdx.x, h = seg % H, n_seg = gridDim.x;  // (b, h)
  const int n_bins = 2 * T + 1, tid = threadIdx.x;
  // the segment's place among the heads: segments with more kept tiles, or as many and a lower id, go first
  auto head_total = [&](int hh) { return row_ptr[hh * T + T] - row_ptr[hh * T]; };
  const int mine = head_total(h);
  int before = 0;
  for (int s2 = tid; s2 < n_seg; s2 += kOrderThreads) {
    const int t2 = head_total(s2 % H);
    before += (t2 > mine || (t2 == mine && s2 < seg)) ? 1 : 0;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) before += __shfl_xor_sync(0xffffffffu, before, o);
  if ((tid & 31) == 0) rank_part[tid >> 5] = before;
  auto cost = [&](int qp) {
    const int r0 = h * T + 2 * qp;
    int c = row_ptr[r0 + 1] - row_ptr[r0];
    if (2 * qp + 1 < T) c += row_ptr[r0 + 2] - row_ptr[r0 + 1];
    return c;
  };
  for (int i = tid; i < n_bins; i += kOrderThreads) bins[i] = 0;
  __syncthreads();
  int rank = 0;
#pragma unroll
  for (int w = 0; w < kOrderThreads / 32; ++w) rank += rank_part[w];
  for (int qp = tid; qp < NP; qp += kOrderThreads) atomicAdd(&bins[cost(qp)], 1);
  __syncthreads();
  // exclusive scan from the largest cost down: bins[c] <- number of the segment's items of cost > c
  const int per = (n_bins + kOrderThreads - 1) / kOrderThreads;
  const int lo = n_bins - 1 - tid * per;  // this thread's bins: lo, lo - 1, ... (descending cost)
  int local = 0;
  for (int k = 0; k < per && lo - k >= 0; ++k) local += bins[lo - k];
  const int lane = tid & 31, warp = tid >> 5;
  int x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = lane < kOrderThreads / 32 ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < kOrderThreads / 32) warp_tot[lane] = t;
  }
  __syncthreads();
  int run = x - local + (warp > 0 ? warp_tot[warp - 1] : 0);
  for (int k = 0; k < per && lo - k >= 0; ++k) {
    const int c = bins[lo - k];
    bins[lo - k] = run;
    run += c;
  }
  __syncthreads();
  int32_t* out = order + (size_t)rank * NP;
  for (int qp = tid; qp < NP; qp += kOrderThreads) out[atomicAdd(&bins[cost(qp)], 1)] = seg * NP + qp;
}

__global__ void debug_wait_kernel(unsigned long long timeout_ns, unsigned int* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
    // Nothing ever arrives on this barrier: the bounded wait must give up and record the error.
    mbar_wait(smem_u32(&bar), 0, timeout_ns, ERR_TIMEOUT_DEBUG, nullptr, err);
  }
}

// Evaluates the attention kernel's FMA-pipe exponential on n inputs (pairs; n even), for testing it
// against CUDA's exp2f.
__global__ void debug_exp2_poly_kernel(const float* x, float* y, int n_pairs) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_pairs) return;
  const f2 r = exp2_poly2(f2{x[2 * i], x[2 * i + 1]});
  y[2 * i] = r.x;
  y[2 * i + 1] = r.y;
}

}  // namespace

sp_status launch_debug_exp2_poly(const float* x, float* y, int n, cudaStream_t stream) {
  const int pairs = n / 2;
  if (pairs == 0) return SP_OK;
  debug_exp2_poly_kernel<<<(pairs + 255) / 256, 256, 0, stream>>>(x, y, pairs);
  return cudaGetLastError() == cudaSuccess ? SP_OK : SP_ERR_CUDA;
}

sp_status launch_tile_list(const uint8_t* mask, int H, int T, int32_t* row_ptr, int32_t* col_idx,
                           int32_t* counts, cudaStream_t stream) {
  const int rows = H * T;
  if (rows == 0) return SP_OK;
  const int blocks = (rows + 7) / 8;
  tile_count_kernel<<<blocks, 256, 0, stream>>>(mask, rows, T, counts);
  tile_scan_kernel<<<1, 1024, 0, stream>>>(counts, rows, row_ptr);
  tile_fill_kernel<<<blocks, 256, 0, stream>>>(mask, rows, T, row_ptr, col_idx);
  return cudaGetLastError() == cudaSuccess ? SP_OK : SP_ERR_CUDA;
}

bool launch_item_order(const int32_t* row_ptr, int B, int H, int T, int NP, int32_t* order, cudaStream_t stream) {
  if (2LL * T + 1 > kMaxOrderBins || (long long)B * H * NP > 0x7fffffffLL || (long long)B * H > 0x7fffffffLL)
    return false;  // no order: the natural one
  if ((long long)B * H * NP == 0) return true;
  item_order_kernel<<<B * H, kOrderThreads, 0, stream>>>(row_ptr, H, T, NP, order);
  return cudaGetLastError() == cudaSuccess;
}

sp_status launch_debug_wait(unsigned long long timeout_ns, cudaStream_t stream) {
  unsigned int* err = device_error_word();
  if (!err) return SP_ERR_CUDA;
  debug_wait_kernel<<<1, 32, 0, stream>>>(timeout_ns, err);
  return cudaGetLastError() == cudaSuccess ? SP_OK : SP_ERR_CUDA;
}

}  // namespace spattn
