// merge.cu -- re-merge of KV-block partials (o_b, lse_b) into the attention over the union of blocks.
//
// "CHARM+: Cross-Hardware Attention with Re-Merge Multistream Mechanism", abstract (re-merge of partial
// results); "CHARM+: How Cross-Hardware Attention Breaks Through ...", Ring-Attention paragraph (each
// round's partial result is accumulated).  For one row (b, s, h):
//   M = max_b lse_b,  L = M + ln sum_b exp(lse_b - M),  o = sum_b exp(lse_b - L) o_b,  lse = L,
// and o = 0, lse = -inf when every lse_b is -inf.
//
// A streaming kernel: every partial byte is read once and every output byte written once.  A warp
// takes 32 consecutive positions s of one (b, h); for each row, D/4 lanes each own 4 consecutive fp32
// of D and issue the n 16-byte loads of the partials back to back.  The n LSE values of a row are read
// by every lane of the row from L1 (they are 128-byte lines shared by the warp's 32 rows).
#include <cstdint>

#include "sp_internal.h"
#include "sp_ptx.cuh"

namespace spattn {
namespace {

struct MergeArgs {
  const float* o[SP_MAX_PARTS];
  const float* lse[SP_MAX_PARTS];
};

template <int D, int NMAX>
__global__ void __launch_bounds__(256) merge_kernel(const __grid_constant__ MergeArgs a, int n, void* o,
                                                    float* lse_out, int o_f32, int B, int S, int H) {
  constexpr int kLanesPerRow = D / 4;
  constexpr int kRowsPerIter = 32 / kLanesPerRow;
  const int warp_global = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int s_blocks = (S + 31) / 32;
  const long long n_tasks = (long long)B * H * s_blocks;
  if (warp_global >= n_tasks) return;
  const int sb = warp_global % s_blocks;
  const int bh = warp_global / s_blocks;
  const int h = bh % H;
  const int b = bh / H;
  const int sub = lane / kLanesPerRow;  // which row of the iteration this lane serves
  const int dl = lane % kLanesPerRow;   // which 4 columns of D
  for (int r0 = 0; r0 < 32; r0 += kRowsPerIter) {
    const int s = sb * 32 + r0 + sub;
    if (s >= S) continue;
    const size_t li = ((size_t)b * H + h) * S + s;
    const size_t oi = (((size_t)b * S + s) * H + h) * D + dl * 4;
    float lp[NMAX];
    float M = -INFINITY;
#pragma unroll
    for (int p = 0; p < NMAX; ++p) {
      lp[p] = p < n ? a.lse[p][li] : -INFINITY;
      M = fmaxf(M, lp[p]);
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float L = -INFINITY;
    if (M != -INFINITY) {
      float4 v[NMAX];
#pragma unroll
      for (int p = 0; p < NMAX; ++p)
        if (p < n) v[p] = __ldcs(reinterpret_cast<const float4*>(a.o[p] + oi));
      float sum = 0.f;
#pragma unroll
      for (int p = 0; p < NMAX; ++p)
        if (p < n && lp[p] != -INFINITY) sum += expf(lp[p] - M);
      L = M + logf(sum);
#pragma unroll
      for (int p = 0; p < NMAX; ++p) {
        if (p < n && lp[p] != -INFINITY) {
          const float w = expf(lp[p] - L);
          acc.x = fmaf(w, v[p].x, acc.x);
          acc.y = fmaf(w, v[p].y, acc.y);
          acc.z = fmaf(w, v[p].z, acc.z);
          acc.w = fmaf(w, v[p].w, acc.w);
        }
      }
    }
    if (o_f32) {
      __stcs(reinterpret_cast<float4*>(static_cast<float*>(o) + oi), acc);
    } else {
      uint2 pk = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
      __stcs(reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(o) + oi), pk);
    }
    if (lse_out && dl == 0) lse_out[li] = L;
  }
}

template <int D, int NMAX>
cudaError_t launch_merge_t(const MergeArgs& a, int n, void* o, float* lse, int o_f32, int B, int S,
                           int H, cudaStream_t stream) {
  const long long tasks = (long long)B * H * ((S + 31) / 32);
  const long long blocks = (tasks + 7) / 8;
  merge_kernel<D, NMAX><<<(unsigned)blocks, 256, 0, stream>>>(a, n, o, lse, o_f32, B, S, H);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_merge_d(const MergeArgs& a, int n, void* o, float* lse, int o_f32, int B, int S,
                           int H, cudaStream_t stream) {
  if (n <= 2) return launch_merge_t<D, 2>(a, n, o, lse, o_f32, B, S, H, stream);
  if (n <= 4) return launch_merge_t<D, 4>(a, n, o, lse, o_f32, B, S, H, stream);
  if (n <= 8) return launch_merge_t<D, 8>(a, n, o, lse, o_f32, B, S, H, stream);
  if (n <= 16) return launch_merge_t<D, 16>(a, n, o, lse, o_f32, B, S, H, stream);
  if (n <= 32) return launch_merge_t<D, 32>(a, n, o, lse, o_f32, B, S, H, stream);
  return launch_merge_t<D, 64>(a, n, o, lse, o_f32, B, S, H, stream);
}

}  // namespace

sp_status launch_merge(const float* const* o_parts, const float* const* lse_parts, int n, void* o,
                       float* lse, int o_f32, int B, int S, int H, int D, cudaStream_t stream) {
  MergeArgs a = {};
  for (int p = 0; p < n; ++p) {
    a.o[p] = o_parts[p];
    a.lse[p] = lse_parts[p];
  }
  if ((long long)B * H * S == 0) return SP_OK;
  cudaError_t e = D == 128 ? launch_merge_d<128>(a, n, o, lse, o_f32, B, S, H, stream)
                           : launch_merge_d<64>(a, n, o, lse, o_f32, B, S, H, stream);
  return e == cudaSuccess ? SP_OK : SP_ERR_CUDA;
}

}  // namespace spattn
