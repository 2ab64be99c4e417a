// pa_internal.h -- host-side declarations shared by the libpa translation units.
#pragma once

#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace pa {

// Arguments of one paged-attention launch (decode rows; the chunked-query
// kernel reuses the same struct).  All pointers are device pointers.
struct AttnArgs {
  void *out;
  const void *q;
  const void *k_cache;
  const void *v_cache;
  const int32_t *block_tables;
  const int32_t *context_lens;
  const int32_t *query_start_loc;  // nullable
  float *part_o;                   // split partial outputs  [S][H][max_splits][D]
  float *part_ml;                  // split partial (m, l)   [S][H][max_splits][2]
  unsigned int *err;               // device error word
  int num_seqs;                    // sequences in this launch
  int seq_begin;                   // first sequence of this launch
  int num_heads;
  int num_kv_heads;
  int group;
  int head_dim;
  int block_size;
  int num_blocks;
  int max_blocks_per_seq;
  int split_blocks;   // KV blocks per split
  int max_splits;     // workspace stride (splits per (seq, head))
  int max_query_len;
  int max_context_len;  // host bound; longer sequences are rejected on the device
  int num_q_tokens;
  int rows_mode;      // 1: the decode kernel also takes rows of Q>1 sequences (one item per row)
  int balanced;       // 1: balanced flat partition (records in part_o), 0: fixed splits
  int grid;           // CTAs of the balanced launch (records are per CTA)
  int item_units;     // balanced: units a (sequence, KV head) pair weighs beyond its blocks
  int no_pdl;         // host only: launch the decode and merge kernels without programmatic dependent launch
  int *bal_prefix;    // balanced: [num_seqs + 1] block prefix written by CTA 0
  int *bal_desc;      // balanced: [grid][4] cut-pair descriptors written by the decode kernel
  float scale_log2;   // scale * log2(e)
  // Shared-prefix decode (all null / 0 otherwise).  The decode kernels read
  // only the blocks after a sequence's shared prefix and fold in the prefix
  // partial that the prefix kernel left in pre_rec.
  const int32_t *grp_start;   // [num_groups + 1] first sequence of each group
  const int32_t *grp_blocks;  // [num_groups] leading blocks the group's members share
  int num_groups;
  int grp_chunks;             // prefix kernel: member chunks per group
  int max_group;              // host bound of any group's size
  float *pre_rec;             // [num_seqs][num_heads][D + 4]: o (unnormalised), m, l
  int *seq_pre;               // [num_seqs] shared blocks per sequence (decode kernel CTA 0)
  // FP8 (E4M3) cache: key elements are codes * k_scale (folded into
  // scale_log2), value elements codes * v_scale; v_inv = 1 / v_scale.
  float v_inv;
  float o_scale;      // factor on O / l: v_scale over an FP8 cache staged as its codes, else 1
                      // (chunk rows scale their output by it, prefix records store l / o_scale)
};

// Units a (sequence, KV head) pair weighs in the balanced partition beyond
// its KV blocks (AttnArgs::item_units): the fixed cost of an item (q load,
// cross-warp merge, output store, next-item set-up) measured on B200 at
// 1.3-2.4 us against ~0.9 us per 16-bit block, so a CTA that holds many short
// items is given fewer blocks.  Measured (pa_decode, CUDA graphs): 1 / 2 / 3 /
// 4 units -> Llama-3-8B-shaped batch 0.1700 / 0.1680 / 0.1677 / 0.1691 ms,
// Llama-2-7B-shaped MHA batch 0.1719 / 0.1700 / 0.1681 / 0.1681 ms,
// parallel-sampling shared-prefix call 0.1345 / 0.1266 / 0.1211 / 0.1170 ms.
// An FP8 block moves half the bytes, so the same fixed cost weighs more
// blocks: 3 -> 5 units took pa_decode_fp8 on the Llama-3-8B-shaped batch from
// 0.1209 to 0.1163 ms.
#ifndef PA_ITEM_UNITS
#define PA_ITEM_UNITS 3
#endif
#ifndef PA_ITEM_UNITS_FP8
#define PA_ITEM_UNITS_FP8 5
#endif
constexpr int kItemUnits16 = PA_ITEM_UNITS;
constexpr int kItemUnitsFp8 = PA_ITEM_UNITS_FP8;

struct DevInfo {
  int sm_count;
  unsigned int *err;  // address of this device's error word
};

// Implemented in pa_api.cu
cudaError_t device_info(DevInfo *info);

// A second stream of the device's highest priority for a mixed batch's chunk
// rows, forked from the caller's stream and joined back into it with events
// (pa_api.cu).  side_fork returns it locked, or nullptr (nothing enqueued):
// the work then stays on the caller's stream.  mixed_overlap_wanted() is false
// under PA_MIXED_OVERLAP=0.
struct SideStream {
  std::mutex mu;
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  bool ready = false, failed = false;
};
bool mixed_overlap_wanted();
SideStream *side_fork(cudaStream_t caller);
cudaError_t side_join(SideStream *sd, cudaStream_t caller);

// pa_decode with its arguments; overlap = false keeps a mixed batch's chunk
// rows on the caller's stream after its decode rows (no side stream or events
// are created), as pa_decode_noalloc needs.
int decode_call(void *out, const void *q, const void *k_cache, const void *v_cache,
                const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                const int32_t *query_start_loc, int num_seqs, int num_q_tokens, int max_query_len,
                int num_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
                float scale, int max_context_len, int kv_split_tokens, int dtype, void *workspace,
                size_t workspace_bytes, struct CUstream_st *stream, bool overlap);

// printf-style line on stderr when the environment variable PA_DEBUG is set
// (host-side failures that only surface as PA_ERR_CUDA otherwise).
void debug_log(const char *fmt, ...);

// Raise the dynamic shared-memory limit of kernel `func` to `bytes` on the
// current device, once per (kernel, device); thread-safe.  Later calls for the
// same pair return the first call's result without touching the runtime.
// max_shared also asks for the largest shared-memory carve-out, so that the
// kernel's CTAs and those of another kernel with the same preference can share
// an SM's whole 228 KB (the chunk-row and decode kernels of a mixed batch).
cudaError_t set_smem_limit_once(const void *func, int bytes, bool max_shared = false);

// Split policy: KV blocks per split and the largest split count per sequence.
void split_policy(int num_seqs, int num_kv_heads, int block_size, int max_context_len,
                  int kv_split_tokens, int sm_count, int *split_blocks, int *max_splits);

// Implemented in decode_mma.cu (tensor-core decode for 16-bit caches)
bool decode_mma_supported(const AttnArgs &a, int dtype);
cudaError_t launch_decode_mma(const AttnArgs &a, int dtype, int sm_count, cudaStream_t stream);
int decode_mma_grid(const AttnArgs &a, int dtype, int sm_count);  // CTAs of a balanced launch
cudaError_t launch_balanced_reduce(const AttnArgs &a, int dtype, cudaStream_t stream);
// FP8 (E4M3) caches, q/out of q_dtype (PA_F16 or PA_BF16), balanced scheme only
int decode_mma_grid_fp8(const AttnArgs &a, int q_dtype, int sm_count);
cudaError_t launch_decode_mma_fp8(const AttnArgs &a, int q_dtype, int sm_count,
                                  cudaStream_t stream);
// Workspace of the balanced scheme: per-CTA partial records, the per-CTA
// cut-pair descriptors, then the block prefix.
inline size_t balanced_record_bytes(int grid, int group, int head_dim) {
  return ((size_t)grid * 2 * group * (head_dim + 4) * sizeof(float) + 255) / 256 * 256;
}
inline size_t balanced_desc_bytes(int grid) { return ((size_t)grid * 4 * sizeof(int) + 255) / 256 * 256; }

// 2-D tensor map of a 16-bit cache (rows = blocks * kv heads * block_size,
// columns = head_dim; boxes of 64 columns x block_size rows, 128-byte
// swizzle).  Implemented in decode_mma.cu.
bool make_cache_map(CUtensorMap *map, const void *base, int num_blocks, int num_kv_heads,
                    int head_dim, int block_size, int dtype);

// Implemented in cascade.cu (shared-prefix kernel)
constexpr int kPrefixRows = 64;  // query rows (members x group heads) per prefix CTA
bool prefix_supported(const AttnArgs &a, int dtype);
cudaError_t launch_prefix(const AttnArgs &a, int dtype, int cluster, cudaStream_t stream);

// Implemented in decode.cu (CUDA-core kernel, fixed-split scheme)
cudaError_t launch_decode(const AttnArgs &a, int dtype, int sm_count, cudaStream_t stream);
cudaError_t launch_reduce(const AttnArgs &a, int dtype, cudaStream_t stream);
int decode_max_seqs_per_launch();

// Implemented in chunk_tc.cu (tcgen05 chunked-query kernel, head_dim 128)
bool chunk_tc_supported(const AttnArgs &a, int dtype);
cudaError_t launch_chunk_tc(const AttnArgs &a, int dtype, cudaStream_t stream);
// The same kernel as the shared-prefix pass (group rows, records out)
cudaError_t launch_prefix_tc(const AttnArgs &a, int dtype, cudaStream_t stream);

// Implemented in chunk_pp.cu (tcgen05 chunked-query kernel, two Q tiles in
// ping-pong over 128-key tiles; head_dim 128, 16-bit caches)
bool chunk_pp_supported(const AttnArgs &a, int dtype);
cudaError_t launch_chunk_pp(const AttnArgs &a, int dtype, cudaStream_t stream);
// The same kernel as the shared-prefix pass (member rows of a group over the
// group's shared blocks, records out; uses a.max_group and a.num_groups)
cudaError_t launch_prefix_pp(const AttnArgs &a, int dtype, cudaStream_t stream);

// Implemented in chunk.cu
cudaError_t launch_chunk(const AttnArgs &a, int dtype, int num_q_tokens, cudaStream_t stream);

// FP8 shared prefixes (fp8.cu): stage the shared blocks of every group of `a`
// (an FP8 cache, grp_* set) into 16-bit pools sk/sv of `capacity` blocks with
// tables `tab` (same row stride as a.block_tables; -1 where a member's block
// differs from its group's first sequence), gbase [num_groups + 1] scratch;
// PA_DEVERR_STAGING when the groups hold more than capacity blocks.
cudaError_t launch_fp8_group_stage(const AttnArgs &a, int q_dtype, int *gbase, int32_t *tab,
                                   void *sk, void *sv, int capacity, cudaStream_t s);
// Bytes of one staging pool (K or V) of `staged_blocks` 16-bit blocks, 1 KiB aligned.
size_t fp8_pool_bytes(int staged_blocks, int num_kv_heads, int head_dim, int block_size);

// Implemented in cache_ops.cu
cudaError_t launch_reshape_and_cache(const void *key, const void *value, void *k_cache,
                                     void *v_cache, const int64_t *slot_mapping, int num_tokens,
                                     int num_kv_heads, int head_dim, int block_size,
                                     int num_blocks, int elem_bytes, unsigned int *err,
                                     cudaStream_t stream);
cudaError_t launch_copy_blocks(void *k_cache, void *v_cache, const int64_t *block_mapping,
                               int num_pairs, int num_kv_heads, int head_dim, int block_size,
                               int num_blocks, int elem_bytes, unsigned int *err,
                               cudaStream_t stream);

}  // namespace pa
