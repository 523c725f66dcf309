// sp_internal.h -- declarations shared by the library's translation units (not part of the C ABI).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "../../include/sp_attn.h"

namespace spattn {

constexpr int kMaxDevices = 64;
constexpr int kMaxChunks = 128;
constexpr int kMaxShards = SP_MAX_SHARDS;  // sequence shards one attention launch reads and writes directly

// Parameters of one attention launch (all H heads, all S queries, keys in [kv_begin, kv_lim)).
struct AttnParams {
  int B, S, H, D;
  int n_qpairs;     // ceil(ceil(S/128) / 2): work items per (b, h)
  int n_items;      // B * H * (n_qpairs - qp_skip)
  int qp_skip;      // causal partial launches: leading query pairs per (b, h) that no key of the range
                    // reaches; they get no work item (their rows are filled with O = 0, lse = -inf)
  int kv_begin;     // first key position
  int kv_lim;       // one past the last key position (<= S)
  int n_kv_tiles;   // ceil((kv_lim - kv_begin) / 128)
  int causal;
  float scale_log2; // log2(e) / sqrt(D)
  void* o;          // bf16 or fp32 BSHD
  int o_f32;
  float* lse;       // [B, H, S] or nullptr
  int o_merge;      // 1: o (fp32) and lse hold a running result that this launch's rows are merged into in
                    // place (log-sum-exp rule); rows that see no key of the range are left untouched
  int pdl;          // 1: launched to overlap the kernel before it on the stream (programmatic dependent
                    // launch); reads of what that kernel writes wait for it (pdl_wait below)
  int pdl_wait_start;  // 1: wait for the previous kernel before reading anything (its output is an input here)
  int pdl_wait_epi;    // 1: wait for the previous kernel before the first epilogue (writes, or merging reads)
  const int* item_list; // device list of work-item ids (nullptr: items 0 .. n_items-1); ids index the
                        // one-chunk layout (b * H + h) * n_qpairs + qp, and ids outside it are skipped
  int item_space;       // number of valid ids (B * H * n_qpairs) when item_list is set
  const int* row_ptr;  // block-sparse tile list (nullptr: dense)
  const int* col_idx;
  int mask_T;          // ceil(S/128)
  int n_chunks;
  int chunk_h0[kMaxChunks + 1];     // first head of each chunk, chunk_h0[n_chunks] = H
  int chunk_item0[kMaxChunks + 1];  // first work item of each chunk
  unsigned long long timeout_ns;
  unsigned int* err;    // device error word of this device
  unsigned int* sched;  // this launch's work counter pair [next item, CTAs finished] (set by launch_attn)
  // Sequence sharding.  n_shards == 1: Q, K, V and O are the single [B, S, H, D] tensors (o above).
  // n_shards > 1: each is split along S into n_shards buffers [B, shard_rows, H, D] (row s lives in
  // shard s / shard_rows at local row s % shard_rows); o is unused and O rows go to o_shard.
  int n_shards;
  int shard_rows;
  int tiles_per_shard;  // ceil(shard_rows / 128): query and key tiles lie on each shard's own grid
  int pairs_per_shard;  // ceil(tiles_per_shard / 2); n_qpairs = n_shards * pairs_per_shard
  const void* q_shard[kMaxShards];
  const void* k_shard[kMaxShards];
  const void* v_shard[kMaxShards];
  void* o_shard[kMaxShards];
};

// Parameters of the backward launches (all heads, all S queries and keys, optionally causal).
struct BwdParams {
  int B, S, H, D;
  int T;              // ceil(S / 128)
  int causal;
  float scale_log2;   // log2(e) / sqrt(D)
  float scale;        // 1 / sqrt(D)
  const float* lse;   // forward lse [B, H, S], natural log
  float* delta;       // [B, H, S] fp32 scratch: rowsum(dO * O)
  void* dq;           // bf16 BSHD outputs
  void* dk;
  void* dv;
  float* dq_acc;      // non-null: dq is not written; this launch's dQ contribution is added here (fp32 BSHD)
  const void* q;      // bf16 BSHD inputs read directly by the dQ kernel (its resident operands)
  const void* dout;
  int kv_begin;       // keys [kv_begin, kv_end) only (one KV block of a ring); kv_begin a multiple of 128
  int kv_end;
  int kt0, n_kt;      // their key tiles: kt0 .. kt0 + n_kt - 1
  unsigned long long timeout_ns;
  unsigned int* err;
};

// Device properties and driver entry points (cached per device).
int num_sms(int device);
bool encode_bshd_tmap(CUtensorMap* map, const void* base, int B, int S, int H, int D, int box_rows = 128);
// O of an attention launch as a store target: [B, S, H, D] of bf16 or fp32, boxes of 128 bytes of one head
// (64 bf16 or 32 fp32 values) by 32 positions, 128-byte swizzle.
bool encode_o_tmap(CUtensorMap* map, void* base, int B, int S, int H, int D, bool f32);
unsigned long long wait_timeout_ns();
int launch_overlap();  // sp_set_launch_overlap: 0 off, 1 inputs, 2 inputs and outputs
unsigned int* device_error_word();  // address of the current device's error word, or nullptr

// Launchers (host validation is done by the C entry points before these are called).
int attn_smem_bytes(int D);
sp_status launch_attn(const AttnParams& p, const void* q, const void* k, const void* v,
                      cudaStream_t stream);
// As launch_attn, with Q, K, V (and O) given as the sequence shards in p (n_shards, shard_rows, *_shard).
sp_status launch_attn_sharded(const AttnParams& p, cudaStream_t stream);
sp_status launch_attn_bwd(const BwdParams& p, const void* q, const void* k, const void* v, const void* o,
                          const void* dout, cudaStream_t stream);
sp_status launch_f32_to_bf16(const float* in, void* out, long long n, cudaStream_t stream);  // n % 4 == 0
sp_status launch_merge(const float* const* o_parts, const float* const* lse_parts, int n, void* o,
                       float* lse, int o_f32, int B, int S, int H, int D, cudaStream_t stream);
sp_status launch_relayout(const void* const* in_ranks, void* const* out_ranks, int P, int B, int S,
                          int H, int D, int elem_bytes, bool seq_to_head, cudaStream_t stream);
// The local halves of a multi-process Ulysses exchange: split (in[0] -> out[0..P-1]) or merge
// (in[0..P-1] -> out[0]) of heads [h0, h0 + n_heads) of each of the P head groups of a [B, S, H, D] shard.
sp_status launch_head_groups(const void* const* in, void* const* out, bool split, int P, int B, int S, int H, int D,
                             int h0, int n_heads, int elem_bytes, cudaStream_t stream);
sp_status launch_tile_list(const uint8_t* mask, int H, int T, int32_t* row_ptr, int32_t* col_idx,
                           int32_t* counts, cudaStream_t stream);
// Item ids of a block-sparse launch (one head chunk, pairs of query tiles) ordered by kept tiles, most first,
// into order[B * H * NP]; false (nothing launched) when the costs span more bins than the sort handles.
bool launch_item_order(const int32_t* row_ptr, int B, int H, int T, int NP, int32_t* order, cudaStream_t stream);
sp_status launch_debug_wait(unsigned long long timeout_ns, cudaStream_t stream);
sp_status launch_debug_exp2_poly(const float* x, float* y, int n, cudaStream_t stream);

}  // namespace spattn
