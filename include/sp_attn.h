/*
 * sp_attn.h -- C ABI of libspattn.so: sequence/head-parallel exact attention for NVIDIA B200 (sm_100a).
 *
 * The operations, and the passages that define them:
 *   - exact multi-head scaled-dot-product attention, O = softmax(Q K^T / sqrt(D)) V per head:
 *     "LLM Lab Notes 05: Attention Tensor Parallelism -- Splitting QKV by Head, Megatron Style",
 *     section 2 (code walkthrough) step 4 "local attention" and "Local projections and local attention";
 *   - heads processed as independent, possibly uneven, contiguous head chunks whose outputs are
 *     concatenated in chunk order: "HCMS: Head-Chunked Multi-Stream Pipeline ...", abstract (uneven
 *     head partitions, numerical equivalence) and "LLM Lab Notes 05", sections 4-5 (rank-ordered
 *     concatenation, divisibility of heads by ranks);
 *   - KV processed in blocks whose partial (O, LSE) results are re-merged: "CHARM+: How Cross-Hardware
 *     Attention Breaks Through Distributed Communication Bottlenecks", Ring-Attention paragraph (each
 *     round computes local attention on one KV block and accumulates partial results), and "CHARM+:
 *     Cross-Hardware Attention with Re-Merge Multistream Mechanism", abstract (re-merge);
 *   - a per-head block-sparse mask of 128 x 128 tiles: "db-SP: Accelerating Sparse Attention for
 *     Visual Generative Models with Dual-Balanced Sequence Parallelism", abstract;
 *   - the Ulysses all-to-all layout permutation between P sequence shards and P head shards: "HCMS",
 *     abstract (all-to-all sequence parallelism) and "db-SP", abstract (parallelism along the head
 *     dimension, as in Ulysses).  Here the P "ranks" are P buffers in one GPU's memory.
 *
 * Conventions for every entry point:
 *   - Q, K, V, O are BSHD: [B, S, H, D] contiguous, row-major; element (b, s, h, d) is at index
 *     ((b * S + s) * H + h) * D + d.  Q, K, V and a bf16 O are bfloat16.  D is 64 or 128.
 *   - LSE is fp32 [B, H, S]: the natural-log log-sum-exp of the scaled scores of a row, -inf for a row
 *     that sees no key (whose O row is then 0).
 *   - All pointers named as device pointers are device memory owned by the caller; the library never
 *     allocates or frees device memory and keeps no pointer after a call returns.  Arrays of pointers
 *     (head_chunks, o_parts, lse_parts, in_ranks, out_ranks) are host memory, read during the call.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the legacy default stream) and
 *     returns after enqueuing.  Arguments are validated on the host before anything is launched: any
 *     violation returns SP_ERR_INVALID_ARG (or SP_ERR_UNSUPPORTED) and launches nothing.  A launch
 *     failure returns SP_ERR_CUDA.  A device-side wait that exceeds its time limit (the kernels never
 *     spin without bound) records an error word that sp_check_device_error() reports as SP_ERR_TIMEOUT.
 *   - Device pointers must be 16-byte aligned.
 *   - Concurrency: the attention entry points (sp_attn_fwd, sp_attn_fwd_partial, sp_attn_fwd_seq_sharded,
 *     sp_attn_fwd_partial_merge, sp_attn_fwd_items, sp_attn_fwd_sparse_noalloc) hand out work through per-launch counters in a fixed
 *     device array of 64 slots, given to launches in rotation.  At most 64 attention launches may be in
 *     flight at once on one device (e.g. on different streams, or in graphs replayed concurrently); a
 *     65th concurrent launch would share a counter with the launch 64 before it and both would compute
 *     wrong results.  Launches ordered on one stream never overlap and are unaffected.
 */
#ifndef SP_ATTN_H
#define SP_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SP_API __attribute__((visibility("default")))
#else
#define SP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SP_OK = 0,
  SP_ERR_INVALID_ARG = 1,
  SP_ERR_UNSUPPORTED = 2,
  SP_ERR_CUDA = 3,
  SP_ERR_TIMEOUT = 4
} sp_status;

typedef enum { SP_BF16 = 0, SP_F32 = 1 } sp_dtype;

/* Opaque stream handle: a cudaStream_t. */
typedef void* sp_stream;

/* Tile edge of the block mask and of the kernels' query/key tiles. */
#define SP_TILE 128
/* Largest number of partials sp_merge_partials combines in one call, and of relayout ranks. */
#define SP_MAX_PARTS 64
#define SP_MAX_RANKS 64
/* Largest number of sequence shards sp_attn_fwd_seq_sharded reads and writes directly. */
#define SP_MAX_SHARDS 8

/*
 * Bytes of device workspace sp_attn_fwd / sp_attn_fwd_partial need for these sizes.
 * n_kv_blocks > 1 needs n_kv_blocks fp32 partials (O [B,S,H,D] and LSE [B,H,S] each); has_mask != 0
 * needs the compacted tile list (H * ceil(S/128) + 1 row offsets and up to H * ceil(S/128)^2 tile
 * indices, int32) and the launch's work order (B * H * ceil(ceil(S/128) / 2) item ids, int32: a masked
 * launch claims its work items head by head, the heads with the most kept tiles first, and within a head
 * the items with the most kept tiles first).  Each section is rounded up to 256 bytes.
 * Returns 0 when neither applies, and 0 for invalid sizes.
 */
SP_API size_t sp_attn_fwd_workspace_bytes(int B, int S, int H, int D, int n_kv_blocks, int has_mask);

/*
 * Exact attention, O = softmax(Q K^T / sqrt(D)) V per head (see the header comment for the passages).
 *
 * q, k, v   device, bf16 BSHD [B,S,H,D].
 * o         device, bf16 BSHD [B,S,H,D], written; must not overlap q, k, v.
 * lse       device, fp32 [B,H,S], written; may be NULL.
 * head_chunks  host int[n_head_chunks]: contiguous chunks of heads, in order, each > 0, sum == H.
 *           NULL means one chunk of H heads.  Chunk c covers heads [h0, h0 + head_chunks[c]) and its
 *           output lands at the same head offset of o, which is the rank-ordered concatenation of the
 *           chunks' outputs.  Per-head arithmetic does not depend on the chunking: every chunking gives
 *           bitwise the same o and lse.
 * n_kv_blocks  >= 1 and <= ceil(S/128).  1: keys are processed in one pass.  > 1: the key range is cut
 *           into n_kv_blocks contiguous blocks of ceil(S/n) keys (rounded up to a multiple of 128 when a
 *           block mask is given), each block's partial (O, LSE) is computed over all queries into the
 *           workspace, and the partials are re-merged (sp_merge_partials) into o and lse.  With a mask
 *           the rounding can leave trailing blocks that would start at or past S: they hold no key and
 *           are dropped, so fewer than n_kv_blocks partials may be merged.
 * causal    0 or 1: key j is visible to query i only if j <= i (square, top-left aligned).
 * block_mask  device uint8 [H, ceil(S/128), ceil(S/128)] or NULL (dense).  Tile (i, j) of head h is
 *           computed iff block_mask[h][i][j] != 0; combined with causal by AND.  Shared by all b.
 * workspace, workspace_bytes  device scratch of at least sp_attn_fwd_workspace_bytes(...) bytes
 *           (may be NULL when that is 0).  Contents on entry are ignored; overwritten.
 * Errors: SP_ERR_INVALID_ARG for B < 1, S < 1, H < 1, D not in {64, 128}, bad head chunks, bad
 * n_kv_blocks, causal not 0/1, a NULL or misaligned required pointer, or a short workspace.
 */
SP_API sp_status sp_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int S,
                      int H, int D, const int* head_chunks, int n_head_chunks, int n_kv_blocks,
                      int causal, const uint8_t* block_mask, void* workspace, size_t workspace_bytes,
                      sp_stream stream);

/*
 * One KV block (one Ring-Attention round): every one of the S queries attends only to keys
 * kv_begin <= j < kv_end (positions global, so causal compares global positions).
 *
 * o_part    device, fp32 BSHD [B,S,H,D]: the block's normalised output; rows with no visible key are 0.
 * lse_part  device, fp32 [B,H,S]: the block's LSE, -inf for rows with no visible key.
 * 0 <= kv_begin <= kv_end <= S.  With a block mask, kv_begin must be a multiple of 128.
 * Other arguments as in sp_attn_fwd (no head chunks: all H heads).
 */
SP_API sp_status sp_attn_fwd_partial(const void* q, const void* k, const void* v, float* o_part,
                              float* lse_part, int B, int S, int H, int D, int kv_begin, int kv_end,
                              int causal, const uint8_t* block_mask, void* workspace,
                              size_t workspace_bytes, sp_stream stream);

/*
 * One KV block merged straight into a running result, the form in which a ring consumes its rounds
 * ("CHARM+: How Cross-Hardware Attention Breaks Through ...", Ring-Attention paragraph: each round computes
 * local attention on one KV block and accumulates the partial results; "CHARM+: Cross-Hardware Attention
 * with Re-Merge ...", abstract: re-merge).  It computes the block's partial (O_b, LSE_b) over keys
 * kv_begin <= j < kv_end exactly as sp_attn_fwd_partial does, and instead of writing it, merges it into
 * (o_acc, lse_acc) in place with the log-sum-exp rule of sp_merge_partials:
 *   lse' = ln(e^lse_acc + e^LSE_b),  o_acc' = e^(lse_acc - lse') o_acc + e^(LSE_b - lse') O_b.
 * Rows that see no key of the block (e.g. causal queries before kv_begin) keep o_acc and lse_acc
 * untouched; no partial is ever materialised.  A row whose lse_acc is -inf has no running result yet: its
 * o_acc is not read into the sum (it may hold anything), so a caller starts a ring either with
 * sp_attn_fwd_partial on its first block into (o_acc, lse_acc), or with lse_acc set to -inf.
 * The order of the merges changes the result by rounding only.
 *
 * o_acc     device, fp32 BSHD [B,S,H,D], read and written.
 * lse_acc   device, fp32 [B,H,S], read and written (natural log).  Neither may overlap q, k, v or the other.
 * kv_end == kv_begin is allowed and changes nothing.  Other arguments as in sp_attn_fwd_partial.
 */
SP_API sp_status sp_attn_fwd_partial_merge(const void* q, const void* k, const void* v, float* o_acc,
                                           float* lse_acc, int B, int S, int H, int D, int kv_begin, int kv_end,
                                           int causal, const uint8_t* block_mask, void* workspace,
                                           size_t workspace_bytes, sp_stream stream);

/*
 * Re-merge of n partials with the log-sum-exp rule ("CHARM+ ... Re-Merge", abstract):
 *   M = max_b lse_b,  lse = M + ln sum_b exp(lse_b - M),  o = sum_b exp(lse_b - lse) * o_b;
 * a row whose partials are all -inf gives o = 0, lse = -inf (never NaN).
 *
 * o_parts, lse_parts  host arrays of n device pointers: fp32 BSHD [B,S,H,D] and fp32 [B,H,S].
 * 1 <= n <= SP_MAX_PARTS.
 * o         device, [B,S,H,D] of o_dtype (SP_BF16 rounds to nearest even, or SP_F32).  With SP_F32 it
 *           may alias o_parts[0] (in-place merge); otherwise no overlap with the inputs.
 * lse       device, fp32 [B,H,S], or NULL; may alias lse_parts[0].
 */
SP_API sp_status sp_merge_partials(const float* const* o_parts, const float* const* lse_parts, int n, void* o,
                            float* lse, sp_dtype o_dtype, int B, int S, int H, int D, sp_stream stream);

/*
 * Gradients of the attention of sp_attn_fwd (one head chunk, one KV block, no mask; dense or causal) for
 * an upstream gradient dout of o: the backward pass whose speed "CHARM+ ..." (abstract) reports next to
 * the forward's.  With p_ij = exp(q_i.k_j / sqrt(D) - lse_i) over the keys query i sees,
 *   delta_i = dout_i . o_i,  dv_j = sum_i p_ij dout_i,  ds_ij = p_ij (dout_i . v_j - delta_i),
 *   dq_i = sum_j ds_ij k_j / sqrt(D),  dk_j = sum_i ds_ij q_i / sqrt(D).
 * q, k, v, o, dout  device bf16 [B, S, H, D] (o and lse as sp_attn_fwd wrote them for q, k, v);
 * lse       device fp32 [B, H, S] (natural log);
 * dq, dk, dv  device bf16 [B, S, H, D] outputs, overlapping nothing else;
 * workspace  device, sp_attn_bwd_workspace_bytes(B, S, H, D) bytes (the fp32 delta per row).
 * Three launches on `stream`: delta, then dk and dv (one CTA per key tile), then dq (one per query tile);
 * p and ds are rounded to bf16 for the tensor cores, accumulation is fp32.  Errors as sp_attn_fwd.
 */
SP_API size_t sp_attn_bwd_workspace_bytes(int B, int S, int H, int D);
SP_API sp_status sp_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                             const float* lse, void* dq, void* dk, void* dv, int B, int S, int H, int D, int causal,
                             void* workspace, size_t workspace_bytes, sp_stream stream);

/*
 * The backward of one KV block [kv_begin, kv_end) of a ring ("CHARM+ ...", abstract: the backward of the
 * Ring-Attention scheme; "CHARM+: How Cross-Hardware Attention ...", Ring-Attention paragraph: one KV block
 * per round).  With o and lse the merged result over all blocks (sp_merge_partials), the gradients split
 * by block: this call writes dk and dv for the block's keys (rows [kv_begin, kv_end), other rows untouched)
 * and ADDS the block's contribution to dq into dq_acc (device fp32 [B,S,H,D], zeroed by the caller before
 * the first block); after every block, dq_acc holds dq (convert with sp_convert_f32_to_bf16).
 * kv_begin must be a multiple of 128; 0 <= kv_begin < kv_end <= S.  Other arguments as sp_attn_bwd.
 */
SP_API sp_status sp_attn_bwd_partial(const void* q, const void* k, const void* v, const void* o, const void* dout,
                                     const float* lse, float* dq_acc, void* dk, void* dv, int B, int S, int H,
                                     int D, int kv_begin, int kv_end, int causal, void* workspace,
                                     size_t workspace_bytes, sp_stream stream);

/* out[i] = in[i] rounded to bf16 (nearest even), n a multiple of 4; in 16-byte and out 8-byte aligned. */
SP_API sp_status sp_convert_f32_to_bf16(const float* in, void* out, long long n, sp_stream stream);

/*
 * Ulysses relayout, sequence shards -> head shards, between P buffers of one GPU:
 *   in_ranks[r]  device [B, S/P, H, D]   (rank r's slice of the sequence, all heads)
 *   out_ranks[r] device [B, S, H/P, D]   (all positions of heads [r*H/P, (r+1)*H/P))
 *   out_r[b, s, h', :] = in_{s / (S/P)}[b, s % (S/P), r*H/P + h', :]   (a bit-exact byte copy).
 * Requires 1 <= P <= SP_MAX_RANKS, S % P == 0, H % P == 0 ("LLM Lab Notes 05", section 5: head count
 * divisible by the parallel degree), elem_bytes in {1, 2, 4, 8}, (D * elem_bytes) % 16 == 0,
 * 16-byte aligned buffers and no overlap between any input and any output.
 */
SP_API sp_status sp_seq_to_head_relayout(const void* const* in_ranks, void* const* out_ranks, int P, int B,
                                  int S, int H, int D, int elem_bytes, sp_stream stream);

/* The exact inverse: in_ranks[r] [B, S, H/P, D] -> out_ranks[r] [B, S/P, H, D].  Same requirements. */
SP_API sp_status sp_head_to_seq_relayout(const void* const* in_ranks, void* const* out_ranks, int P, int B,
                                  int S, int H, int D, int elem_bytes, sp_stream stream);

/*
 * The local halves of the Ulysses all-to-all when the P ranks are P processes on P GPUs ("HCMS", abstract:
 * all-to-all based sequence parallelism; "db-SP", abstract: parallelism along the head dimension as in
 * Ulysses).  The exchange itself is a collective between contiguous per-destination blocks (NCCL
 * all-to-all); around it, each rank copies its own sequence shard x [B, S, H, D] (S: the rank's own
 * positions) into P head groups, and back.  With g = H/P and heads [h0, h0 + n) of every group (the whole
 * group, h0 = 0 and n = g, or one stage of an exchange done in head chunks, "HCMS", abstract):
 *   sp_split_heads:  out_ranks[r] [B, S, n, D] = x[:, :, r*g + h0 : r*g + h0 + n, :]  (block sent to rank r)
 *   sp_merge_heads:  out[:, :, r*g + h0 : r*g + h0 + n, :] = in_ranks[r] [B, S, n, D] (block from rank r)
 * Bit-exact byte copies; merge leaves the other heads of out untouched.  Requires 1 <= P <= SP_MAX_RANKS,
 * H % P == 0, 0 <= h0, n >= 1, h0 + n <= H/P, elem_bytes in {1, 2, 4, 8}, (D * elem_bytes) % 16 == 0,
 * 16-byte aligned buffers, no overlap between any input and any output or between two outputs.
 * out_ranks / in_ranks are host arrays of P device pointers.
 */
SP_API sp_status sp_split_heads(const void* in, void* const* out_ranks, int P, int B, int S, int H, int D, int h0,
                                int n_heads, int elem_bytes, sp_stream stream);
SP_API sp_status sp_merge_heads(const void* const* in_ranks, void* out, int P, int B, int S, int H, int D, int h0,
                                int n_heads, int elem_bytes, sp_stream stream);

/*
 * One Ulysses rank's attention straight on the sequence shards, with both relayouts folded into the
 * kernel ("HCMS: ... Ulysses ... all-to-all", abstract: each rank attends over the whole sequence for its
 * share of the heads; "LLM Lab Notes 05", section 2: per head q @ k^T / sqrt(d), softmax, @ v).  It
 * computes what sp_seq_to_head_relayout of Q, K and V, sp_attn_fwd of the rank's heads [h0, h0 + n_heads)
 * with these head chunks, then sp_head_to_seq_relayout of O compute, but no head-sharded copy is ever
 * written: query and key tiles lie on each shard's own 128-row grid (a shard's last tile may be short),
 * each is loaded from its shard, and each O row is written into the shard that owns it.  When S/P is a
 * multiple of 128 the grids coincide and the result is bit for bit that of the three calls; otherwise
 * the keys are grouped into different tiles, so the result differs from theirs by rounding only.
 *
 * q_shards, k_shards, v_shards  host arrays of P device pointers, bf16 [B, S/P, H, D]: shard r holds
 *                               positions [r*S/P, (r+1)*S/P) of every head.
 * o_shards  host array of P device pointers, bf16 [B, S/P, H, D]; heads [h0, h0 + n_heads) of every
 *           row are written, the other heads are left untouched (so P calls with disjoint head ranges
 *           fill them all).  No overlap with any input.
 * lse       device fp32 [B, H, S] (every head of the whole sequence; rows of heads [h0, h0 + n_heads)
 *           written), or NULL.
 * head_chunks  host int[n_head_chunks], each > 0, summing to n_heads (NULL: one chunk).
 * Requires 1 <= P <= SP_MAX_SHARDS, S % P == 0, 0 <= h0, h0 + n_heads <= H, D in {64, 128}, 16-byte
 * aligned pointers.  No block mask.  Errors as sp_attn_fwd.
 */
SP_API sp_status sp_attn_fwd_seq_sharded(const void* const* q_shards, const void* const* k_shards,
                                         const void* const* v_shards, void* const* o_shards, float* lse, int P,
                                         int B, int S, int H, int D, int h0, int n_heads, const int* head_chunks,
                                         int n_head_chunks, int causal, sp_stream stream);

/*
 * db-SP work partition ("db-SP: ... Sparsity-Aware Sequence Parallelism ...", abstract: dual-level
 * partitioning over heads and blocks balancing block-sparse attention; the page gives neither the imbalance
 * formula nor the algorithm, so these are this library's reading).  Host functions on host arrays; no GPU.
 *
 * Work unit: (head h, query-tile pair qp), qp < NP = ceil(T/2), T = ceil(S/128): the kernel's work item.
 * Unit u = h * NP + qp costs the 128 x 128 tiles its two query-tile rows keep (keys j <= i when causal).
 *
 * sp_dbsp_unit_costs  block_mask: host u8 [H, T, T] or NULL (dense); cost: host int64 [H * NP] (out).
 * sp_dbsp_plan        cost [H * NP] -> unit_rank [H * NP] (out, host): level 1 places whole heads, longest
 *                     first, on the least loaded rank; level 2 moves single units from the most to the
 *                     least loaded rank while a unit with 0 < cost < (max - min load) exists (the one with
 *                     2 cost closest to the gap).  Ties: lower head / unit / rank first.  rank_load [P]
 *                     and imbalance (max load / mean load) are optional outputs.  1 <= P <= SP_MAX_RANKS.
 * sp_dbsp_rank_items  the kernel item ids of rank `rank` for batch size B, (b * H + h) * NP + qp, longest
 *                     unit first; items may be NULL to query the count (*n_items), else capacity must hold it.
 */
SP_API sp_status sp_dbsp_unit_costs(const uint8_t* block_mask, int H, int T, int causal, long long* cost);
SP_API sp_status sp_dbsp_plan(const long long* cost, int H, int NP, int P, int* unit_rank, long long* rank_load,
                              double* imbalance);
SP_API sp_status sp_dbsp_rank_items(const long long* cost, const int* unit_rank, int B, int H, int NP, int rank,
                                    int* items, int capacity, int* n_items);

/*
 * Attention over an explicit list of work items: exactly what sp_attn_fwd (one head chunk, one KV block)
 * writes for those items' rows, and nothing else (other rows of o and lse are left untouched).
 * items: device int [n_items], ids (b * H + h) * ceil(ceil(S/128)/2) + qp of the one-chunk layout (e.g.
 * from sp_dbsp_rank_items); each names query tiles 2 qp and 2 qp + 1 of head h, batch b.  An id outside
 * that range is skipped and reported by sp_check_device_error as SP_ERR_INVALID_ARG.  Items are claimed in
 * list order.  Workspace and the other arguments as in sp_attn_fwd (n_kv_blocks = 1).
 */
SP_API sp_status sp_attn_fwd_items(const void* q, const void* k, const void* v, void* o, float* lse, int B, int S,
                                   int H, int D, const int* items, int n_items, int causal,
                                   const uint8_t* block_mask, void* workspace, size_t workspace_bytes,
                                   sp_stream stream);

/*
 * Block-sparse attention that allocates nothing, for callers that cannot call cudaMalloc (a serving
 * path that must not block on the device synchronisation an allocation may cause, a plug-in handed
 * tensors by a framework that owns all device memory, a real-time loop that forbids allocation after
 * start-up).  The pages have no counterpart for this entry point: it exists for those callers only.
 *
 * Computes exactly what sp_attn_fwd computes with this block_mask, one head chunk and n_kv_blocks = 1
 * (same kernels, same results).  The scratch that sp_attn_fwd takes from the caller's workspace (the
 * mask's compacted tile list) lives instead in a fixed array inside the library, 12,714,240 bytes, which
 * every GPU that loads the library keeps until the process exits.  Limits: H * ceil(S/128) <=
 * SP_NOALLOC_MAX_TILE_ROWS and H * ceil(S/128)^2 <= SP_NOALLOC_MAX_TILES; larger problems return
 * SP_ERR_UNSUPPORTED with nothing launched.
 * The first call on a device looks up that array's device address (cudaGetSymbolAddress with the
 * device current); make that first call before any stream capture.  Every call on a device shares the
 * array and leaves its tile list in it (nothing needs to start at zero: each call rewrites what it
 * reads), so calls whose execution overlaps on the GPU race; order them on one stream or with events.
 * Arguments as in sp_attn_fwd; block_mask is required.
 */
#define SP_NOALLOC_MAX_TILE_ROWS 16384
#define SP_NOALLOC_MAX_TILES (3 * 1024 * 1024)
SP_API sp_status sp_attn_fwd_sparse_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                                            int B, int S, int H, int D, int causal, const uint8_t* block_mask,
                                            sp_stream stream);

/*
 * Compacted tile list of a block mask, the form in which the attention kernels skip dropped tiles
 * ("db-SP", abstract: dense blocks irregularly distributed in a per-head mask).
 *   block_mask device uint8 [H, T, T], T = ceil(S/128); nonzero = keep.
 *   row_ptr    device int32 [H*T + 1]: row (h, i) lists col_idx[row_ptr[h*T+i] .. row_ptr[h*T+i+1]).
 *   col_idx    device int32, capacity H*T*T: kept key-tile indices of each row, increasing.
 *   counts     device int32 [H*T] scratch.
 */
SP_API sp_status sp_build_tile_list(const uint8_t* block_mask, int H, int S, int32_t* row_ptr,
                             int32_t* col_idx, int32_t* counts, sp_stream stream);

/* Human-readable name of a status code (static storage). */
SP_API const char* sp_status_string(sp_status s);

/*
 * Synchronises `stream`, then reads and clears the device error word of the current device:
 * SP_ERR_TIMEOUT if a kernel's bounded wait expired since the last check, SP_ERR_CUDA if the stream
 * reports an error, else SP_OK.
 */
SP_API sp_status sp_check_device_error(sp_stream stream);

/*
 * As sp_check_device_error, and also returns the raw error word in *bits (may be NULL): one bit per
 * kind of wait that expired (Q loaded, Q free, K/V loaded, K/V free, S ready, P ready, P V done, O read
 * out, drain, debug, running-O load of a merge), for diagnosing which hand-off gave up.
 */
SP_API sp_status sp_check_device_error_bits(sp_stream stream, unsigned int* bits);

/*
 * Launch overlap (default 0, off).  With it on, every attention launch (sp_attn_fwd and the other attention
 * entry points) may start while the kernel enqueued just before it on the same stream is still finishing:
 * its CTAs take the SMs that kernel frees (programmatic dependent launch), which fills the tail of a
 * sequence of attention launches such as one launch per Ulysses rank or per ring round.
 *   mode 1: an overlapped launch reads only q, k and v early; it writes o and lse (and
 *           sp_attn_fwd_partial_merge reads its running result) only after the kernel before it has
 *           completed.  The caller promises that q, k and v are not written by that kernel.
 *   mode 2: as mode 1, and the caller also promises that the kernel just before neither reads nor writes
 *           the parts of o and lse this launch writes (e.g. launches for disjoint heads of one output), so
 *           the launch writes them without waiting.  sp_attn_fwd_partial_merge still waits before reading
 *           its running result.
 * In both modes a masked or item-list launch waits for the kernel before it (which may have built its tile
 * list) before reading anything.  Kernels enqueued after an attention launch wait for it as usual.  Applies
 * to later launches; process-wide.
 */
SP_API void sp_set_launch_overlap(int mode);

/* Time limit of every device-side wait, in nanoseconds (default 2e9).  Applies to later launches. */
SP_API void sp_set_wait_timeout_ns(unsigned long long ns);

/*
 * Exercises the bounded-wait path: launches one warp that waits on a barrier nothing will complete,
 * with the given limit; the wait gives up, records SP_ERR_TIMEOUT in the device error word and the
 * kernel returns normally.  The next sp_check_device_error() returns SP_ERR_TIMEOUT.
 */
SP_API sp_status sp_debug_wait_timeout(unsigned long long timeout_ns, sp_stream stream);

/*
 * Evaluates, on the GPU, the exponential 2^x that the attention kernels compute on the FMA pipe for part
 * of each softmax row (range split x = n + f, a minimax cubic for 2^f, 2^n through the exponent), for
 * testing it against CUDA's exp2f.  x, y: device fp32 arrays of n elements, n even.  Inputs below -125
 * are clamped to -125.
 */
SP_API sp_status sp_debug_exp2_poly(const float* x, float* y, int n, sp_stream stream);

/* Library version string. */
SP_API const char* sp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SP_ATTN_H */
