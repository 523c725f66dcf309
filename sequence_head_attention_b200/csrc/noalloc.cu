// noalloc.cu -- block-sparse attention whose scratch lives in a fixed array inside this library, for
// callers that cannot allocate device memory.
//
// Who needs this: code that runs where cudaMalloc is off limits -- a request path that must never block
// on the device-wide synchronisation an allocation can cause, a plug-in that is handed tensors by a host
// framework owning every allocation and exposing no allocator, or a hard-real-time loop that forbids
// allocation after start-up.  Such a caller can provide inputs and outputs but no workspace.
//
// Besides the attention kernel's work counters (a small static array of its own, shared by every
// launch), the only scratch the block-sparse path needs is the compacted tile list of the mask (row
// offsets, per-row counts and kept key-tile indices).  Here it lives in g_noalloc_scratch below: a file-scope
// device array that every GPU which loads this library holds until the process exits.  The array is
// shared by every call on a device, so calls whose execution overlaps on the GPU (different streams, or
// threads without ordering between them) race on it and must be serialised by the caller.  Nothing in
// it needs to start at zero: each call's tile-list build rewrites every entry the attention kernel
// then reads.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "sp_internal.h"

namespace spattn {
namespace {

// Layout of the scratch array, in int32 words: [row_ptr: MAX_ROWS + 1][counts: MAX_ROWS][col_idx: MAX_TILES]
constexpr size_t kRowPtrOff = 0;
constexpr size_t kCountsOff = kRowPtrOff + SP_NOALLOC_MAX_TILE_ROWS + 64;  // keep 256-byte alignment
constexpr size_t kColIdxOff = kCountsOff + SP_NOALLOC_MAX_TILE_ROWS;
constexpr size_t kWords = kColIdxOff + SP_NOALLOC_MAX_TILES;
static_assert(kCountsOff % 64 == 0 && kColIdxOff % 64 == 0, "sections must stay 256-byte aligned");

static __device__ __align__(256) int32_t g_noalloc_scratch[kWords];

std::mutex g_mu;
int32_t* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per device.  The name
// g_noalloc_scratch is only a host-side handle in host code; the address a kernel can use comes from
// cudaGetSymbolAddress with that device current.
int32_t* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    int32_t* ptr = nullptr;
    if (cudaGetSymbolAddress((void**)&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return nullptr;
    g_scratch_addr[dev] = ptr;
  }
  return g_scratch_addr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace spattn

using namespace spattn;

extern "C" sp_status sp_attn_fwd_sparse_noalloc(const void* q, const void* k, const void* v, void* o,
                                                float* lse, int B, int S, int H, int D, int causal,
                                                const uint8_t* block_mask, sp_stream stream) {
  if (B < 1 || S < 1 || H < 1 || (D != 64 && D != 128)) return SP_ERR_INVALID_ARG;
  if (!q || !k || !v || !o || !block_mask) return SP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse && !aligned16(lse)))
    return SP_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SP_ERR_INVALID_ARG;
  if ((double)B * S * H * D >= 9.0e15 || S > (1 << 30)) return SP_ERR_INVALID_ARG;
  const long long T = (S + SP_TILE - 1) / SP_TILE;
  // The scratch has a fixed size: larger masks are refused, never truncated.
  if ((long long)H * T > SP_NOALLOC_MAX_TILE_ROWS || (long long)H * T * T > SP_NOALLOC_MAX_TILES)
    return SP_ERR_UNSUPPORTED;
  const long long n_qpairs = (T + 1) / 2;
  if ((long long)B * H * n_qpairs > 0x7fffffffLL) return SP_ERR_INVALID_ARG;

  int32_t* scratch = scratch_on_current_device();
  if (!scratch) return SP_ERR_CUDA;
  unsigned int* err = device_error_word();
  if (!err) return SP_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t* row_ptr = scratch + kRowPtrOff;
  int32_t* counts = scratch + kCountsOff;
  int32_t* col_idx = scratch + kColIdxOff;
  sp_status s = launch_tile_list(block_mask, H, (int)T, row_ptr, col_idx, counts, st);
  if (s != SP_OK) return s;

  AttnParams p = AttnParams{};
  p.B = B;
  p.S = S;
  p.H = H;
  p.D = D;
  p.n_qpairs = (int)n_qpairs;
  p.n_items = (int)((long long)B * H * n_qpairs);
  p.kv_begin = 0;
  p.kv_lim = S;
  p.n_kv_tiles = (int)T;
  p.causal = causal;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  p.o = o;
  p.o_f32 = 0;
  p.lse = lse;
  p.row_ptr = row_ptr;
  p.col_idx = col_idx;
  p.mask_T = (int)T;
  p.n_chunks = 1;
  p.chunk_h0[0] = 0;
  p.chunk_h0[1] = H;
  p.chunk_item0[0] = 0;
  p.chunk_item0[1] = p.n_items;
  p.timeout_ns = wait_timeout_ns();
  p.err = err;
  return launch_attn(p, q, k, v, st);
}
