// pa_internal.h -- host-side declarations shared by the libpa translation units.
#pragma once

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
  int *bal_prefix;    // balanced: [num_seqs + 1] block prefix written by CTA 0
  int *bal_desc;      // balanced: [grid][4] cut-pair descriptors written by the decode kernel
  float scale_log2;   // scale * log2(e)
};

struct DevInfo {
  int sm_count;
  unsigned int *err;  // address of this device's error word
};

// Implemented in pa_api.cu
cudaError_t device_info(DevInfo *info);

// Split policy: KV blocks per split and the largest split count per sequence.
void split_policy(int num_seqs, int num_kv_heads, int block_size, int max_context_len,
                  int kv_split_tokens, int sm_count, int *split_blocks, int *max_splits);

// Implemented in decode_mma.cu (tensor-core decode for 16-bit caches)
bool decode_mma_supported(const AttnArgs &a, int dtype);
cudaError_t launch_decode_mma(const AttnArgs &a, int dtype, int sm_count, cudaStream_t stream);
int decode_mma_grid(const AttnArgs &a, int dtype, int sm_count);  // CTAs of a balanced launch
cudaError_t launch_balanced_reduce(const AttnArgs &a, int dtype, cudaStream_t stream);
// Workspace of the balanced scheme: per-CTA partial records, the per-CTA
// cut-pair descriptors, then the block prefix.
inline size_t balanced_record_bytes(int grid, int group, int head_dim) {
  return ((size_t)grid * 2 * group * (head_dim + 4) * sizeof(float) + 255) / 256 * 256;
}
inline size_t balanced_desc_bytes(int grid) { return ((size_t)grid * 4 * sizeof(int) + 255) / 256 * 256; }

// Implemented in decode.cu (CUDA-core kernel, fixed-split scheme)
cudaError_t launch_decode(const AttnArgs &a, int dtype, int sm_count, cudaStream_t stream);
cudaError_t launch_reduce(const AttnArgs &a, int dtype, cudaStream_t stream);
int decode_max_seqs_per_launch();

// Implemented in chunk_tc.cu (tcgen05 chunked-query kernel, head_dim 128)
bool chunk_tc_supported(const AttnArgs &a, int dtype);
cudaError_t launch_chunk_tc(const AttnArgs &a, int dtype, cudaStream_t stream);

// Implemented in chunk.cu
cudaError_t launch_chunk(const AttnArgs &a, int dtype, int num_q_tokens, cudaStream_t stream);

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
