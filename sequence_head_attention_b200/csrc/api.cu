// api.cu -- the C entry points of libspattn.so: host-side validation, workspace layout, tensor maps and
// launches.  Declarations and the contract of each call are in include/sp_attn.h.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>
#include <utility>

#include "sp_internal.h"
#include "sp_ptx.cuh"

namespace spattn {

// The device error word: bounded waits that expire OR a code into it (see sp_check_device_error).
__device__ unsigned int g_sp_error = 0;

namespace {

std::mutex g_mu;
int g_num_sms[kMaxDevices] = {};
unsigned int* g_err_addr[kMaxDevices] = {};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
unsigned long long g_timeout_ns = 2000000000ull;
int g_overlap = 0;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct WsLayout {
  size_t parts_o = 0, parts_lse = 0, row_ptr = 0, col_idx = 0, counts = 0, order = 0, total = 0;
};

// Workspace: [n_kv_blocks fp32 O partials][n_kv_blocks fp32 LSE partials][row_ptr][col_idx][counts][order]
WsLayout ws_layout(int B, int S, int H, int D, int n_kv_blocks, int has_mask) {
  WsLayout w;
  size_t off = 0;
  if (n_kv_blocks > 1) {
    w.parts_o = off;
    off += align_up((size_t)n_kv_blocks * B * S * H * D * sizeof(float), 256);
    w.parts_lse = off;
    off += align_up((size_t)n_kv_blocks * B * H * S * sizeof(float), 256);
  }
  if (has_mask) {
    const size_t T = (S + SP_TILE - 1) / SP_TILE;
    w.row_ptr = off;
    off += align_up((H * T + 1) * sizeof(int32_t), 256);
    w.col_idx = off;
    off += align_up(H * T * T * sizeof(int32_t), 256);
    w.counts = off;
    off += align_up(H * T * sizeof(int32_t), 256);
    w.order = off;  // the launch's work order: B * H * ceil(T / 2) item ids
    off += align_up((size_t)B * H * ((T + 1) / 2) * sizeof(int32_t), 256);
  }
  w.total = off;
  return w;
}

bool sizes_ok(int B, int S, int H, int D) {
  if (B < 1 || S < 1 || H < 1) return false;
  if (D != 64 && D != 128) return false;
  // keep every element index inside 63 bits and every tile index inside int
  const double elems = (double)B * S * H * D;
  return elems < 9.0e15 && S <= (1 << 30) && (double)B * H * ((S + 255) / 256) < 2.0e9;
}

cudaStream_t as_stream(sp_stream s) { return reinterpret_cast<cudaStream_t>(s); }

sp_status count_items(AttnParams& p);

sp_status fill_attn_params(AttnParams& p, int B, int S, int H, int D, int kv_begin, int kv_end,
                           int causal, const int* chunk_h0, int n_chunks) {
  p = AttnParams{};
  p.B = B;
  p.S = S;
  p.H = H;
  p.D = D;
  const int n_qtiles = (S + SP_TILE - 1) / SP_TILE;
  p.n_qpairs = (n_qtiles + 1) / 2;
  p.kv_begin = kv_begin;
  p.kv_lim = kv_end < S ? kv_end : S;
  p.n_kv_tiles = p.kv_lim > kv_begin ? (p.kv_lim - kv_begin + SP_TILE - 1) / SP_TILE : 0;
  p.causal = causal;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  p.mask_T = n_qtiles;
  p.timeout_ns = g_timeout_ns;
  p.err = device_error_word();
  if (!p.err) return SP_ERR_CUDA;
  p.n_chunks = n_chunks;
  for (int c = 0; c <= n_chunks; ++c) p.chunk_h0[c] = chunk_h0[c];
  return count_items(p);
}

// Work items per head chunk (B * heads * n_qpairs each) and in all.
sp_status count_items(AttnParams& p) {
  long long items = 0;
  for (int c = 0; c < p.n_chunks; ++c) {
    p.chunk_item0[c] = (int)items;
    items += (long long)p.B * (p.chunk_h0[c + 1] - p.chunk_h0[c]) * p.n_qpairs;
  }
  p.chunk_item0[p.n_chunks] = (int)items;
  if (items > 0x7fffffffLL) return SP_ERR_INVALID_ARG;
  p.n_items = (int)items;
  return SP_OK;
}

}  // namespace

int num_sms(int device) {
  if (device < 0 || device >= kMaxDevices) return 1;
  if (g_num_sms[device] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || v < 1) v = 1;
    g_num_sms[device] = v;
  }
  return g_num_sms[device];
}

unsigned long long wait_timeout_ns() { return g_timeout_ns; }

int launch_overlap() { return g_overlap; }

unsigned int* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_sp_error) != cudaSuccess) return nullptr;
    g_err_addr[dev] = static_cast<unsigned int*>(ptr);
  }
  return g_err_addr[dev];
}

// The driver's tensor-map encoder, looked up once.
static bool have_encoder() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return false;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  return true;
}

bool encode_bshd_tmap(CUtensorMap* map, const void* base, int B, int S, int H, int D, int box_rows) {
  if (!have_encoder()) return false;
  // Dimensions innermost first: d, h, s, b.  Box: 64 head-dim elements (128 bytes, the swizzle span)
  // of one head, box_rows positions (128, or 64 for a CTA pair's half of a key tile), one batch.  Rows
  // past S read as zero.
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)S * H * D * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_o_tmap(CUtensorMap* map, void* base, int B, int S, int H, int D, bool f32) {
  if (!have_encoder()) return false;
  const cuuint64_t es = f32 ? 4 : 2;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * es, (cuuint64_t)H * D * es, (cuuint64_t)S * H * D * es};
  cuuint32_t box[4] = {(cuuint32_t)(128 / es), 1, 32, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace spattn

using namespace spattn;

extern "C" {

size_t sp_attn_fwd_workspace_bytes(int B, int S, int H, int D, int n_kv_blocks, int has_mask) {
  if (!sizes_ok(B, S, H, D) || n_kv_blocks < 1) return 0;
  return ws_layout(B, S, H, D, n_kv_blocks, has_mask).total;
}

const char* sp_status_string(sp_status s) {
  switch (s) {
    case SP_OK: return "SP_OK";
    case SP_ERR_INVALID_ARG: return "SP_ERR_INVALID_ARG";
    case SP_ERR_UNSUPPORTED: return "SP_ERR_UNSUPPORTED";
    case SP_ERR_CUDA: return "SP_ERR_CUDA";
    case SP_ERR_TIMEOUT: return "SP_ERR_TIMEOUT";
  }
  return "SP_ERR_UNKNOWN";
}

const char* sp_version(void) { return "spattn 0.1 (sm_100a)"; }

void sp_set_launch_overlap(int mode) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_overlap = mode <= 0 ? 0 : (mode == 1 ? 1 : 2);
}

void sp_set_wait_timeout_ns(unsigned long long ns) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_timeout_ns = ns < 1000ull ? 1000ull : ns;
}

sp_status sp_check_device_error_bits(sp_stream stream, unsigned int* bits) {
  if (bits) *bits = 0;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return SP_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_sp_error, sizeof(v)) != cudaSuccess) return SP_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_sp_error, &zero, sizeof(zero)) != cudaSuccess) return SP_ERR_CUDA;
  if (bits) *bits = v;
  if (v & ERR_ANY_TIMEOUT) return SP_ERR_TIMEOUT;
  return (v & ERR_BAD_ITEM) ? SP_ERR_INVALID_ARG : SP_OK;
}

sp_status sp_check_device_error(sp_stream stream) { return sp_check_device_error_bits(stream, nullptr); }

sp_status sp_debug_wait_timeout(unsigned long long timeout_ns, sp_stream stream) {
  if (timeout_ns < 1000ull || timeout_ns > 10000000000ull) return SP_ERR_INVALID_ARG;
  return launch_debug_wait(timeout_ns, as_stream(stream));
}

sp_status sp_debug_exp2_poly(const float* x, float* y, int n, sp_stream stream) {
  if (!x || !y || n < 0 || (n & 1)) return SP_ERR_INVALID_ARG;
  return launch_debug_exp2_poly(x, y, n, as_stream(stream));
}

sp_status sp_build_tile_list(const uint8_t* block_mask, int H, int S, int32_t* row_ptr, int32_t* col_idx,
                             int32_t* counts, sp_stream stream) {
  if (!block_mask || !row_ptr || !col_idx || !counts || H < 1 || S < 1) return SP_ERR_INVALID_ARG;
  const long long T = (S + SP_TILE - 1) / SP_TILE;
  if ((long long)H * T * T > 0x7fffffffLL) return SP_ERR_INVALID_ARG;
  return launch_tile_list(block_mask, H, (int)T, row_ptr, col_idx, counts, as_stream(stream));
}

sp_status sp_attn_fwd_partial(const void* q, const void* k, const void* v, float* o_part, float* lse_part,
                              int B, int S, int H, int D, int kv_begin, int kv_end, int causal,
                              const uint8_t* block_mask, void* workspace, size_t workspace_bytes,
                              sp_stream stream) {
  if (!sizes_ok(B, S, H, D)) return SP_ERR_INVALID_ARG;
  if (!q || !k || !v || !o_part || !lse_part) return SP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o_part) || !aligned16(lse_part))
    return SP_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SP_ERR_INVALID_ARG;
  if (kv_begin < 0 || kv_end < kv_begin || kv_end > S) return SP_ERR_INVALID_ARG;
  if (block_mask && kv_begin % SP_TILE != 0) return SP_ERR_INVALID_ARG;
  const WsLayout wl = ws_layout(B, S, H, D, 1, block_mask != nullptr);
  if (wl.total > 0 && (!workspace || workspace_bytes < wl.total || !aligned16(workspace)))
    return SP_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  AttnParams p;
  int h0[2] = {0, H};
  sp_status s = fill_attn_params(p, B, S, H, D, kv_begin, kv_end, causal, h0, 1);
  if (s != SP_OK) return s;
  p.o = o_part;
  p.o_f32 = 1;
  p.lse = lse_part;
  if (block_mask) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int32_t* row_ptr = reinterpret_cast<int32_t*>(ws + wl.row_ptr);
    int32_t* col_idx = reinterpret_cast<int32_t*>(ws + wl.col_idx);
    s = launch_tile_list(block_mask, H, p.mask_T, row_ptr, col_idx, reinterpret_cast<int32_t*>(ws + wl.counts), st);
    if (s != SP_OK) return s;
    p.row_ptr = row_ptr;
    p.col_idx = col_idx;
  }
  return launch_attn(p, q, k, v, st);
}

sp_status sp_attn_fwd_partial_merge(const void* q, const void* k, const void* v, float* o_acc, float* lse_acc,
                                    int B, int S, int H, int D, int kv_begin, int kv_end, int causal,
                                    const uint8_t* block_mask, void* workspace, size_t workspace_bytes,
                                    sp_stream stream) {
  if (!sizes_ok(B, S, H, D)) return SP_ERR_INVALID_ARG;
  if (!q || !k || !v || !o_acc || !lse_acc) return SP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o_acc) || !aligned16(lse_acc))
    return SP_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SP_ERR_INVALID_ARG;
  if (kv_begin < 0 || kv_end < kv_begin || kv_end > S) return SP_ERR_INVALID_ARG;
  if (block_mask && kv_begin % SP_TILE != 0) return SP_ERR_INVALID_ARG;
  // the running result is read and written in place: it may not overlap the inputs
  const size_t tb = (size_t)B * S * H * D * 2, ob = (size_t)B * S * H * D * 4, lb = (size_t)B * H * S * 4;
  for (const void* in : {q, k, v}) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(in);
    for (const auto& out : {std::make_pair((const void*)o_acc, ob), std::make_pair((const void*)lse_acc, lb)}) {
      const uintptr_t b0 = reinterpret_cast<uintptr_t>(out.first);
      if (a0 < b0 + out.second && b0 < a0 + tb) return SP_ERR_INVALID_ARG;
    }
  }
  {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(o_acc), b0 = reinterpret_cast<uintptr_t>(lse_acc);
    if (a0 < b0 + lb && b0 < a0 + ob) return SP_ERR_INVALID_ARG;
  }
  const WsLayout wl = ws_layout(B, S, H, D, 1, block_mask != nullptr);
  if (wl.total > 0 && (!workspace || workspace_bytes < wl.total || !aligned16(workspace)))
    return SP_ERR_INVALID_ARG;
  if (kv_end == kv_begin) return SP_OK;  // no key: every row keeps its running result
  cudaStream_t st = as_stream(stream);
  AttnParams p;
  int h0[2] = {0, H};
  sp_status s = fill_attn_params(p, B, S, H, D, kv_begin, kv_end, causal, h0, 1);
  if (s != SP_OK) return s;
  p.o = o_acc;
  p.o_f32 = 1;
  p.lse = lse_acc;
  p.o_merge = 1;
  if (block_mask) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int32_t* row_ptr = reinterpret_cast<int32_t*>(ws + wl.row_ptr);
    int32_t* col_idx = reinterpret_cast<int32_t*>(ws + wl.col_idx);
    s = launch_tile_list(block_mask, H, p.mask_T, row_ptr, col_idx, reinterpret_cast<int32_t*>(ws + wl.counts), st);
    if (s != SP_OK) return s;
    p.row_ptr = row_ptr;
    p.col_idx = col_idx;
  }
  return launch_attn(p, q, k, v, st);
}

sp_status sp_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int S, int H,
                      int D, const int* head_chunks, int n_head_chunks, int n_kv_blocks, int causal,
                      const uint8_t* block_mask, void* workspace, size_t workspace_bytes, sp_stream stream) {
  if (!sizes_ok(B, S, H, D)) return SP_ERR_INVALID_ARG;
  if (!q || !k || !v || !o) return SP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse && !aligned16(lse)))
    return SP_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SP_ERR_INVALID_ARG;
  const int n_tiles = (S + SP_TILE - 1) / SP_TILE;
  if (n_kv_blocks < 1 || n_kv_blocks > n_tiles || n_kv_blocks > SP_MAX_PARTS) return SP_ERR_INVALID_ARG;
  // head chunks: contiguous, in order, each > 0, summing to H
  int h0[kMaxChunks + 1];
  int n_chunks = 1;
  h0[0] = 0;
  h0[1] = H;
  if (head_chunks) {
    if (n_head_chunks < 1 || n_head_chunks > kMaxChunks) return SP_ERR_INVALID_ARG;
    long long acc = 0;
    for (int c = 0; c < n_head_chunks; ++c) {
      if (head_chunks[c] < 1) return SP_ERR_INVALID_ARG;
      h0[c] = (int)acc;
      acc += head_chunks[c];
      if (acc > H) return SP_ERR_INVALID_ARG;
    }
    if (acc != H) return SP_ERR_INVALID_ARG;
    h0[n_head_chunks] = H;
    n_chunks = n_head_chunks;
  } else if (n_head_chunks != 0 && n_head_chunks != 1) {
    return SP_ERR_INVALID_ARG;
  }
  const WsLayout wl = ws_layout(B, S, H, D, n_kv_blocks, block_mask != nullptr);
  if (wl.total > 0 && (!workspace || workspace_bytes < wl.total || !aligned16(workspace)))
    return SP_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  AttnParams p;
  sp_status s = fill_attn_params(p, B, S, H, D, 0, S, causal, h0, n_chunks);
  if (s != SP_OK) return s;
  if (block_mask) {
    int32_t* row_ptr = reinterpret_cast<int32_t*>(ws + wl.row_ptr);
    int32_t* col_idx = reinterpret_cast<int32_t*>(ws + wl.col_idx);
    s = launch_tile_list(block_mask, H, p.mask_T, row_ptr, col_idx, reinterpret_cast<int32_t*>(ws + wl.counts), st);
    if (s != SP_OK) return s;
    p.row_ptr = row_ptr;
    p.col_idx = col_idx;
  }
  if (n_kv_blocks == 1) {
    p.o = o;
    p.o_f32 = 0;
    p.lse = lse;
    if (block_mask && n_chunks == 1) {
      // claim the items most-kept-tiles first, so that the launch ends with short items
      int32_t* order = reinterpret_cast<int32_t*>(ws + wl.order);
      if (launch_item_order(p.row_ptr, B, H, p.mask_T, p.n_qpairs, order, st)) {
        p.item_list = order;
        p.item_space = p.n_items;
      }
    }
    return launch_attn(p, q, k, v, st);
  }
  // KV blocks: ceil(S / n) keys each (a multiple of 128 with a mask), partials into the workspace, then
  // the log-sum-exp re-merge.
  long long blk = (S + n_kv_blocks - 1) / n_kv_blocks;
  if (block_mask) blk = (blk + SP_TILE - 1) / SP_TILE * SP_TILE;
  float* parts_o = reinterpret_cast<float*>(ws + wl.parts_o);
  float* parts_l = reinterpret_cast<float*>(ws + wl.parts_lse);
  const size_t o_elems = (size_t)B * S * H * D, l_elems = (size_t)B * H * S;
  const float* op[SP_MAX_PARTS];
  const float* lp[SP_MAX_PARTS];
  int n_parts = 0;
  for (int i = 0; i < n_kv_blocks; ++i) {
    const long long a = i * blk, e = (i + 1) * blk < S ? (i + 1) * blk : S;
    // With a mask the block size is rounded up to whole tiles, so trailing blocks can start at or past S:
    // they hold no key and are dropped (never launched with a kv_begin off the tile grid).
    if (a >= S) break;
    AttnParams pi = p;
    pi.kv_begin = (int)a;
    pi.kv_lim = (int)e;
    pi.n_kv_tiles = (pi.kv_lim - pi.kv_begin + SP_TILE - 1) / SP_TILE;
    pi.o = parts_o + i * o_elems;
    pi.o_f32 = 1;
    pi.lse = parts_l + i * l_elems;
    s = launch_attn(pi, q, k, v, st);
    if (s != SP_OK) return s;
    op[n_parts] = parts_o + i * o_elems;
    lp[n_parts] = parts_l + i * l_elems;
    ++n_parts;
  }
  return launch_merge(op, lp, n_parts, o, lse, 0, B, S, H, D, st);
}

sp_status sp_merge_partials(const float* const* o_parts, const float* const* lse_parts, int n, void* o,
                            float* lse, sp_dtype o_dtype, int B, int S, int H, int D, sp_stream stream) {
  if (!sizes_ok(B, S, H, D)) return SP_ERR_INVALID_ARG;
  if (!o_parts || !lse_parts || !o || n < 1 || n > SP_MAX_PARTS) return SP_ERR_INVALID_ARG;
  if (o_dtype != SP_BF16 && o_dtype != SP_F32) return SP_ERR_INVALID_ARG;
  if (!aligned16(o) || (lse && !aligned16(lse))) return SP_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    if (!o_parts[i] || !lse_parts[i] || !aligned16(o_parts[i]) || !aligned16(lse_parts[i]))
      return SP_ERR_INVALID_ARG;
    if (i > 0 && (o_parts[i] == o || (lse && lse_parts[i] == lse))) return SP_ERR_INVALID_ARG;
  }
  if (o_dtype == SP_BF16 && (const void*)o_parts[0] == o) return SP_ERR_INVALID_ARG;
  return launch_merge(o_parts, lse_parts, n, o, lse, o_dtype == SP_F32, B, S, H, D, as_stream(stream));
}

static sp_status relayout_common(const void* const* in_ranks, void* const* out_ranks, int P, int B, int S,
                                 int H, int D, int elem_bytes, bool seq_to_head, sp_stream stream) {
  if (!in_ranks || !out_ranks || P < 1 || P > SP_MAX_RANKS || B < 1 || S < 1 || H < 1 || D < 1)
    return SP_ERR_INVALID_ARG;
  if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8) return SP_ERR_INVALID_ARG;
  if (S % P != 0 || H % P != 0 || ((long long)D * elem_bytes) % 16 != 0) return SP_ERR_INVALID_ARG;
  if ((double)B * S * H * D * elem_bytes > 9.0e15) return SP_ERR_INVALID_ARG;
  const long long in_bytes = seq_to_head ? (long long)B * (S / P) * H * D * elem_bytes
                                         : (long long)B * S * (H / P) * D * elem_bytes;
  const long long out_bytes = seq_to_head ? (long long)B * S * (H / P) * D * elem_bytes
                                          : (long long)B * (S / P) * H * D * elem_bytes;
  for (int r = 0; r < P; ++r) {
    if (!in_ranks[r] || !out_ranks[r] || !aligned16(in_ranks[r]) || !aligned16(out_ranks[r]))
      return SP_ERR_INVALID_ARG;
  }
  // no input buffer may overlap any output buffer
  for (int r = 0; r < P; ++r)
    for (int g = 0; g < P; ++g) {
      const uintptr_t a0 = reinterpret_cast<uintptr_t>(in_ranks[r]), a1 = a0 + in_bytes;
      const uintptr_t b0 = reinterpret_cast<uintptr_t>(out_ranks[g]), b1 = b0 + out_bytes;
      if (a0 < b1 && b0 < a1) return SP_ERR_INVALID_ARG;
    }
  return launch_relayout(in_ranks, out_ranks, P, B, S, H, D, elem_bytes, seq_to_head, as_stream(stream));
}

sp_status sp_attn_fwd_seq_sharded(const void* const* q_shards, const void* const* k_shards,
                                  const void* const* v_shards, void* const* o_shards, float* lse, int P, int B,
                                  int S, int H, int D, int h0, int n_heads, const int* head_chunks,
                                  int n_head_chunks, int causal, sp_stream stream) {
  if (!sizes_ok(B, S, H, D)) return SP_ERR_INVALID_ARG;
  if (!q_shards || !k_shards || !v_shards || !o_shards || P < 1 || P > SP_MAX_SHARDS || S % P != 0)
    return SP_ERR_INVALID_ARG;
  if (h0 < 0 || n_heads < 1 || (long long)h0 + n_heads > H) return SP_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SP_ERR_INVALID_ARG;
  if (lse && !aligned16(lse)) return SP_ERR_INVALID_ARG;
  for (int r = 0; r < P; ++r) {
    if (!q_shards[r] || !k_shards[r] || !v_shards[r] || !o_shards[r]) return SP_ERR_INVALID_ARG;
    if (!aligned16(q_shards[r]) || !aligned16(k_shards[r]) || !aligned16(v_shards[r]) || !aligned16(o_shards[r]))
      return SP_ERR_INVALID_ARG;
  }
  // no output shard may overlap an input shard
  const size_t shard_bytes = (size_t)B * (S / P) * H * D * 2;
  for (int r = 0; r < P; ++r)
    for (int i = 0; i < P; ++i)
      for (const void* in : {q_shards[i], k_shards[i], v_shards[i]}) {
        const uintptr_t a0 = reinterpret_cast<uintptr_t>(o_shards[r]), b0 = reinterpret_cast<uintptr_t>(in);
        if (a0 < b0 + shard_bytes && b0 < a0 + shard_bytes) return SP_ERR_INVALID_ARG;
      }
  // head chunks of [h0, h0 + n_heads): contiguous, in order, each > 0, summing to n_heads
  int c0[kMaxChunks + 1];
  int n_chunks = 1;
  c0[0] = h0;
  c0[1] = h0 + n_heads;
  if (head_chunks) {
    if (n_head_chunks < 1 || n_head_chunks > kMaxChunks) return SP_ERR_INVALID_ARG;
    long long acc = 0;
    for (int c = 0; c < n_head_chunks; ++c) {
      if (head_chunks[c] < 1) return SP_ERR_INVALID_ARG;
      c0[c] = h0 + (int)acc;
      acc += head_chunks[c];
      if (acc > n_heads) return SP_ERR_INVALID_ARG;
    }
    if (acc != n_heads) return SP_ERR_INVALID_ARG;
    c0[n_head_chunks] = h0 + n_heads;
    n_chunks = n_head_chunks;
  } else if (n_head_chunks != 0 && n_head_chunks != 1) {
    return SP_ERR_INVALID_ARG;
  }
  AttnParams p;
  sp_status s = fill_attn_params(p, B, S, H, D, 0, S, causal, c0, n_chunks);
  if (s != SP_OK) return s;
  p.o = o_shards[0];
  p.o_f32 = 0;
  p.lse = lse;
  p.n_shards = P;
  p.shard_rows = S / P;
  p.tiles_per_shard = (p.shard_rows + SP_TILE - 1) / SP_TILE;
  p.pairs_per_shard = (p.tiles_per_shard + 1) / 2;
  p.n_qpairs = P * p.pairs_per_shard;
  p.n_kv_tiles = P * p.tiles_per_shard;
  s = count_items(p);
  if (s != SP_OK) return s;
  for (int r = 0; r < P; ++r) {
    p.q_shard[r] = q_shards[r];
    p.k_shard[r] = k_shards[r];
    p.v_shard[r] = v_shards[r];
    p.o_shard[r] = o_shards[r];
  }
  return launch_attn_sharded(p, as_stream(stream));
}

sp_status sp_attn_fwd_items(const void* q, const void* k, const void* v, void* o, float* lse, int B, int S, int H,
                            int D, const int* items, int n_items, int causal, const uint8_t* block_mask,
                            void* workspace, size_t workspace_bytes, sp_stream stream) {
  if (!sizes_ok(B, S, H, D)) return SP_ERR_INVALID_ARG;
  if (!q || !k || !v || !o || n_items < 0 || (n_items > 0 && !items)) return SP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse && !aligned16(lse)))
    return SP_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SP_ERR_INVALID_ARG;
  const WsLayout wl = ws_layout(B, S, H, D, 1, block_mask != nullptr);
  if (wl.total > 0 && (!workspace || workspace_bytes < wl.total || !aligned16(workspace)))
    return SP_ERR_INVALID_ARG;
  if (n_items == 0) return SP_OK;
  cudaStream_t st = as_stream(stream);
  AttnParams p;
  int h0[2] = {0, H};
  sp_status s = fill_attn_params(p, B, S, H, D, 0, S, causal, h0, 1);
  if (s != SP_OK) return s;
  p.item_space = p.n_items;
  p.item_list = items;
  p.n_items = n_items;
  p.o = o;
  p.o_f32 = 0;
  p.lse = lse;
  if (block_mask) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int32_t* row_ptr = reinterpret_cast<int32_t*>(ws + wl.row_ptr);
    int32_t* col_idx = reinterpret_cast<int32_t*>(ws + wl.col_idx);
    s = launch_tile_list(block_mask, H, p.mask_T, row_ptr, col_idx, reinterpret_cast<int32_t*>(ws + wl.counts), st);
    if (s != SP_OK) return s;
    p.row_ptr = row_ptr;
    p.col_idx = col_idx;
  }
  return launch_attn(p, q, k, v, st);
}

size_t sp_attn_bwd_workspace_bytes(int B, int S, int H, int D) {
  if (!sizes_ok(B, S, H, D)) return 0;
  return ((size_t)B * H * S * sizeof(float) + 255) & ~(size_t)255;
}

sp_status sp_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                      void* dq, void* dk, void* dv, int B, int S, int H, int D, int causal, void* workspace,
                      size_t workspace_bytes, sp_stream stream) {
  if (!sizes_ok(B, S, H, D)) return SP_ERR_INVALID_ARG;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace) return SP_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, o, dout, (const void*)lse, (const void*)dq, (const void*)dk, (const void*)dv,
                          (const void*)workspace})
    if (!aligned16(ptr)) return SP_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SP_ERR_INVALID_ARG;
  if (workspace_bytes < sp_attn_bwd_workspace_bytes(B, S, H, D)) return SP_ERR_INVALID_ARG;
  // the gradients may not overlap any input, one another or the workspace
  const size_t tb = (size_t)B * S * H * D * 2;
  const size_t lb = (size_t)B * H * S * 4;
  struct Span { const void* p; size_t n; };
  const Span ins[] = {{q, tb}, {k, tb}, {v, tb}, {o, tb}, {dout, tb}, {lse, lb}, {workspace, lb}};
  const Span outs[] = {{dq, tb}, {dk, tb}, {dv, tb}};
  auto overlap = [](const Span& x, const Span& y) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(x.p), b0 = reinterpret_cast<uintptr_t>(y.p);
    return a0 < b0 + y.n && b0 < a0 + x.n;
  };
  for (int i = 0; i < 3; ++i) {
    for (const Span& in : ins)
      if (overlap(outs[i], in)) return SP_ERR_INVALID_ARG;
    for (int j = i + 1; j < 3; ++j)
      if (overlap(outs[i], outs[j])) return SP_ERR_INVALID_ARG;
  }
  BwdParams p{};
  p.B = B;
  p.S = S;
  p.H = H;
  p.D = D;
  p.T = (S + SP_TILE - 1) / SP_TILE;
  p.causal = causal;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  p.scale = (float)(1.0 / std::sqrt((double)D));
  p.lse = lse;
  p.delta = static_cast<float*>(workspace);
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.dq_acc = nullptr;
  p.kv_begin = 0;
  p.kv_end = S;
  p.kt0 = 0;
  p.n_kt = p.T;
  p.timeout_ns = g_timeout_ns;
  p.err = device_error_word();
  if (!p.err) return SP_ERR_CUDA;
  return launch_attn_bwd(p, q, k, v, o, dout, as_stream(stream));
}

sp_status sp_attn_bwd_partial(const void* q, const void* k, const void* v, const void* o, const void* dout,
                              const float* lse, float* dq_acc, void* dk, void* dv, int B, int S, int H, int D,
                              int kv_begin, int kv_end, int causal, void* workspace, size_t workspace_bytes,
                              sp_stream stream) {
  if (!sizes_ok(B, S, H, D)) return SP_ERR_INVALID_ARG;
  if (kv_begin < 0 || kv_end <= kv_begin || kv_end > S || kv_begin % SP_TILE != 0) return SP_ERR_INVALID_ARG;
  if (!q || !k || !v || !o || !dout || !lse || !dq_acc || !dk || !dv || !workspace) return SP_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, o, dout, (const void*)lse, (const void*)dq_acc, (const void*)dk,
                          (const void*)dv, (const void*)workspace})
    if (!aligned16(ptr)) return SP_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SP_ERR_INVALID_ARG;
  if (workspace_bytes < sp_attn_bwd_workspace_bytes(B, S, H, D)) return SP_ERR_INVALID_ARG;
  const size_t tb = (size_t)B * S * H * D * 2;
  const size_t lb = (size_t)B * H * S * 4;
  struct Span { const void* p; size_t n; };
  const Span ins[] = {{q, tb}, {k, tb}, {v, tb}, {o, tb}, {dout, tb}, {lse, lb}, {workspace, lb}};
  const Span outs[] = {{dq_acc, 2 * tb}, {dk, tb}, {dv, tb}};
  auto overlap = [](const Span& x, const Span& y) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(x.p), b0 = reinterpret_cast<uintptr_t>(y.p);
    return a0 < b0 + y.n && b0 < a0 + x.n;
  };
  for (int i = 0; i < 3; ++i) {
    for (const Span& in : ins)
      if (overlap(outs[i], in)) return SP_ERR_INVALID_ARG;
    for (int j = i + 1; j < 3; ++j)
      if (overlap(outs[i], outs[j])) return SP_ERR_INVALID_ARG;
  }
  BwdParams p{};
  p.B = B;
  p.S = S;
  p.H = H;
  p.D = D;
  p.T = (S + SP_TILE - 1) / SP_TILE;
  p.causal = causal;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  p.scale = (float)(1.0 / std::sqrt((double)D));
  p.lse = lse;
  p.delta = static_cast<float*>(workspace);
  p.dq = nullptr;
  p.dk = dk;
  p.dv = dv;
  p.dq_acc = dq_acc;
  p.kv_begin = kv_begin;
  p.kv_end = kv_end;
  p.kt0 = kv_begin / SP_TILE;
  p.n_kt = (kv_end - kv_begin + SP_TILE - 1) / SP_TILE;
  p.timeout_ns = g_timeout_ns;
  p.err = device_error_word();
  if (!p.err) return SP_ERR_CUDA;
  return launch_attn_bwd(p, q, k, v, o, dout, as_stream(stream));
}

sp_status sp_convert_f32_to_bf16(const float* in, void* out, long long n, sp_stream stream) {
  if (n < 0 || (n > 0 && (!in || !out)) || n % 4 != 0) return SP_ERR_INVALID_ARG;
  if (!aligned16(in) || ((reinterpret_cast<uintptr_t>(out) & 7u) != 0)) return SP_ERR_INVALID_ARG;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(in), b0 = reinterpret_cast<uintptr_t>(out);
  if (n > 0 && a0 < b0 + (size_t)n * 2 && b0 < a0 + (size_t)n * 4) return SP_ERR_INVALID_ARG;
  return launch_f32_to_bf16(in, out, n, as_stream(stream));
}

static sp_status head_groups_common(const void* const* ins, int n_in, void* const* outs, int n_out, bool split, int P,
                                    int B, int S, int H, int D, int h0, int n_heads, int elem_bytes, sp_stream stream) {
  if (!ins || !outs || P < 1 || P > SP_MAX_RANKS || B < 1 || S < 0 || H < 1 || D < 1) return SP_ERR_INVALID_ARG;
  if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8) return SP_ERR_INVALID_ARG;
  if (H % P != 0 || ((long long)D * elem_bytes) % 16 != 0) return SP_ERR_INVALID_ARG;
  if (h0 < 0 || n_heads < 1 || h0 + n_heads > H / P) return SP_ERR_INVALID_ARG;
  if ((double)B * S * H * D * elem_bytes > 9.0e15) return SP_ERR_INVALID_ARG;
  const long long whole = (long long)B * S * H * D * elem_bytes, group = (long long)B * S * n_heads * D * elem_bytes;
  const long long in_bytes = split ? whole : group, out_bytes = split ? group : whole;
  for (int r = 0; r < n_in; ++r)
    if (!ins[r] || !aligned16(ins[r])) return SP_ERR_INVALID_ARG;
  for (int r = 0; r < n_out; ++r)
    if (!outs[r] || !aligned16(outs[r])) return SP_ERR_INVALID_ARG;
  for (int r = 0; r < n_in; ++r)  // no input may overlap an output
    for (int g = 0; g < n_out; ++g) {
      const uintptr_t a0 = reinterpret_cast<uintptr_t>(ins[r]), b0 = reinterpret_cast<uintptr_t>(outs[g]);
      if (a0 < b0 + out_bytes && b0 < a0 + in_bytes) return SP_ERR_INVALID_ARG;
    }
  for (int r = 0; r < n_out; ++r)  // nor two outputs one another
    for (int g = r + 1; g < n_out; ++g) {
      const uintptr_t a0 = reinterpret_cast<uintptr_t>(outs[r]), b0 = reinterpret_cast<uintptr_t>(outs[g]);
      if (a0 < b0 + out_bytes && b0 < a0 + out_bytes) return SP_ERR_INVALID_ARG;
    }
  return launch_head_groups(ins, outs, split, P, B, S, H, D, h0, n_heads, elem_bytes, as_stream(stream));
}

sp_status sp_split_heads(const void* in, void* const* out_ranks, int P, int B, int S, int H, int D, int h0, int n_heads,
                         int elem_bytes, sp_stream stream) {
  const void* ins[1] = {in};
  return head_groups_common(ins, 1, out_ranks, P, true, P, B, S, H, D, h0, n_heads, elem_bytes, stream);
}

sp_status sp_merge_heads(const void* const* in_ranks, void* out, int P, int B, int S, int H, int D, int h0,
                         int n_heads, int elem_bytes, sp_stream stream) {
  void* outs[1] = {out};
  return head_groups_common(in_ranks, P, outs, 1, false, P, B, S, H, D, h0, n_heads, elem_bytes, stream);
}

sp_status sp_seq_to_head_relayout(const void* const* in_ranks, void* const* out_ranks, int P, int B, int S,
                                  int H, int D, int elem_bytes, sp_stream stream) {
  return relayout_common(in_ranks, out_ranks, P, B, S, H, D, elem_bytes, true, stream);
}

sp_status sp_head_to_seq_relayout(const void* const* in_ranks, void* const* out_ranks, int P, int B, int S,
                                  int H, int D, int elem_bytes, sp_stream stream) {
  return relayout_common(in_ranks, out_ranks, P, B, S, H, D, elem_bytes, false, stream);
}

}  // extern "C"
