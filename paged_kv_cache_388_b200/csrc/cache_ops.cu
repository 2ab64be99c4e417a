// cache_ops.cu -- reshape_and_cache (scatter of new K/V into their slots) and
// copy_blocks (copy-on-write block copy).  Both are pure byte movement: every
// thread moves 16-byte vectors so each (token, kv-head) row or block tile is
// read and written with fully coalesced 128-byte transactions.
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

// One thread per 16-byte vector of a (token, kv-head) row of K (and of V).
// Source index i = (t * Hk + h) * vpr + v is the thread's linear index, so
// reads are perfectly coalesced; the 16*vpr bytes of a row land contiguously
// at (block, h, offset) of the cache.
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(
    const uint4 *__restrict__ key, const uint4 *__restrict__ value, uint4 *__restrict__ k_cache,
    uint4 *__restrict__ v_cache, const int64_t *__restrict__ slot_mapping, int num_tokens,
    int num_kv_heads, int vpr, int block_size, int64_t num_slots, unsigned int *err) {
  // Launched as a programmatic dependent of the previous kernel: wait for its
  // writes before touching memory; then let the next grid (the decode kernel)
  // be scheduled -- it waits for this grid's writes before reading the cache.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t per_token = (int64_t)num_kv_heads * vpr;
  const int64_t total = (int64_t)num_tokens * per_token;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / per_token;
    const int64_t r = i - t * per_token;
    const int64_t slot = slot_mapping[t];
    if (slot < 0) continue;  // padding token
    if (slot >= num_slots) {
      if (r == 0) raise_error(err, PA_DEVERR_SLOT);
      continue;
    }
    const int h = (int)(r / vpr);
    const int v = (int)(r - (int64_t)h * vpr);
    const int64_t blk = slot / block_size;
    const int64_t off = slot - blk * block_size;
    const int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * vpr + v;
    const uint4 kv = __ldcs(key + i);  // read once: do not keep in L2
    const uint4 vv = __ldcs(value + i);
    k_cache[dst] = kv;
    v_cache[dst] = vv;
  }
}

// One CTA per (pair, K|V): copies one whole block (all kv heads) with four
// independent 16-byte loads in flight per thread.
__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4 *__restrict__ k_cache,
                                                          uint4 *__restrict__ v_cache,
                                                          const int64_t *__restrict__ mapping,
                                                          int64_t blk_vecs, int num_blocks,
                                                          unsigned int *err) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int pair = blockIdx.x;
  uint4 *base = blockIdx.y ? v_cache : k_cache;
  const int64_t src = mapping[2 * (int64_t)pair];
  const int64_t dst = mapping[2 * (int64_t)pair + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0) raise_error(err, PA_DEVERR_BLOCK_ID);
    return;
  }
  const uint4 *s = base + src * blk_vecs;
  uint4 *d = base + dst * blk_vecs;
  constexpr int U = 4;
  const int64_t step = (int64_t)blockDim.x * U;
  int64_t i = threadIdx.x;
  for (; i + (U - 1) * blockDim.x < blk_vecs; i += step) {
    uint4 tmp[U];
#pragma unroll
    for (int u = 0; u < U; ++u) tmp[u] = __ldcs(s + i + u * blockDim.x);
#pragma unroll
    for (int u = 0; u < U; ++u) d[i + u * blockDim.x] = tmp[u];
  }
  for (; i < blk_vecs; i += blockDim.x) d[i] = __ldcs(s + i);
}

}  // namespace

cudaError_t launch_reshape_and_cache(const void *key, const void *value, void *k_cache,
                                     void *v_cache, const int64_t *slot_mapping, int num_tokens,
                                     int num_kv_heads, int head_dim, int block_size,
                                     int num_blocks, int elem_bytes, unsigned int *err,
                                     cudaStream_t stream) {
  if (num_tokens == 0) return cudaSuccess;
  const int vpr = head_dim * elem_bytes / 16;
  const int64_t total = (int64_t)num_tokens * num_kv_heads * vpr;
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 16) blocks = 148 * 16;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(threads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, reshape_and_cache_kernel, static_cast<const uint4 *>(key),
                            static_cast<const uint4 *>(value), static_cast<uint4 *>(k_cache),
                            static_cast<uint4 *>(v_cache), slot_mapping, num_tokens, num_kv_heads,
                            vpr, block_size, (int64_t)num_blocks * block_size, err);
}

cudaError_t launch_copy_blocks(void *k_cache, void *v_cache, const int64_t *block_mapping,
                               int num_pairs, int num_kv_heads, int head_dim, int block_size,
                               int num_blocks, int elem_bytes, unsigned int *err,
                               cudaStream_t stream) {
  if (num_pairs == 0) return cudaSuccess;
  const int64_t blk_vecs = (int64_t)num_kv_heads * block_size * head_dim * elem_bytes / 16;
  dim3 grid((unsigned)num_pairs, 2);
  copy_blocks_kernel<<<grid, 256, 0, stream>>>(static_cast<uint4 *>(k_cache),
                                               static_cast<uint4 *>(v_cache), block_mapping,
                                               blk_vecs, num_blocks, err);
  return cudaGetLastError();
}

}  // namespace pa
