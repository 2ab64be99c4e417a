// swap.cu -- pa_swap_blocks: move whole KV blocks between two pools, either
// of which may be page-locked host memory (the CPU tier of the KV cache).
//
// The KV cache is tiered: device memory holds the blocks of running
// sequences, host memory the blocks of sequences that were swapped out when
// device blocks ran short, and blocks move between the tiers
// ("核心概念", section 内存层次结构; preemption, "理解 vLLM PagedAttention",
// section 五).  One kernel does a whole batch of block moves: it reads and
// writes host memory directly through unified addressing (page-locked host
// memory is mapped into the device's address space), so a swap of many
// scattered blocks costs one launch instead of one DMA copy per block, and
// the transfer runs at the host link's speed once enough 16-byte requests are
// in flight.
//
// Work: one warp per (pair, K or V, KV head) tile -- block_size * head_dim
// elements, contiguous in both pools -- each lane moving its 16-byte vectors
// with all loads issued before the stores.
#include "../../include/pa.h"
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kSwapThreads = 256;

template <int VPL>  // 16-byte vectors per lane per tile
__global__ void __launch_bounds__(kSwapThreads) swap_blocks_kernel(
    unsigned char *dst_k, unsigned char *dst_v, const unsigned char *src_k,
    const unsigned char *src_v, const int64_t *block_mapping, int num_pairs, int num_kv_heads,
    int64_t tile_bytes, int num_src_blocks, int num_dst_blocks, unsigned int *err) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t warp = ((int64_t)blockIdx.x * kSwapThreads + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t tiles = (int64_t)num_pairs * 2 * num_kv_heads;
  const int64_t nwarps = ((int64_t)gridDim.x * kSwapThreads) >> 5;
  const int64_t vecs = tile_bytes / 16;
  for (int64_t t = warp; t < tiles; t += nwarps) {
    const int64_t pair = t / (2 * num_kv_heads);
    const int rest = (int)(t - pair * 2 * num_kv_heads);
    const int which = rest / num_kv_heads;  // 0: K, 1: V
    const int h = rest - which * num_kv_heads;
    int64_t s = 0, d = 0;
    if (lane == 0) {
      s = block_mapping[2 * pair];
      d = block_mapping[2 * pair + 1];
    }
    s = __shfl_sync(0xffffffffu, s, 0);
    d = __shfl_sync(0xffffffffu, d, 0);
    if (s < 0 || s >= num_src_blocks || d < 0 || d >= num_dst_blocks) {
      if (lane == 0 && which == 0 && h == 0) raise_error(err, PA_DEVERR_BLOCK_ID);
      continue;
    }
    const uint4 *src = reinterpret_cast<const uint4 *>(
        (which ? src_v : src_k) + (s * num_kv_heads + h) * tile_bytes);
    uint4 *dst = reinterpret_cast<uint4 *>((which ? dst_v : dst_k) + (d * num_kv_heads + h) * tile_bytes);
    for (int64_t base = 0; base < vecs; base += 32 * VPL) {
      uint4 r[VPL];
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int64_t v = base + i * 32 + lane;
        if (v < vecs) r[i] = src[v];
      }
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int64_t v = base + i * 32 + lane;
        if (v < vecs) dst[v] = r[i];
      }
    }
  }
}

// Device-reachable address of `p` (device memory, page-locked host memory or
// managed memory); null for pageable host memory, which a kernel must never
// touch.
const void *device_view(const void *p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();  // clear the (non-sticky) error the query recorded
    return nullptr;
  }
  switch (at.type) {
    case cudaMemoryTypeDevice:
    case cudaMemoryTypeManaged:
      return p;
    case cudaMemoryTypeHost:
      return at.devicePointer;
    default:
      return nullptr;
  }
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" int pa_swap_blocks(void *dst_k, void *dst_v, const void *src_k, const void *src_v,
                              const int64_t *block_mapping, int num_pairs, int num_kv_heads,
                              int head_dim, int block_size, int num_src_blocks,
                              int num_dst_blocks, int dtype, struct CUstream_st *stream) {
  if (num_pairs < 0 || num_kv_heads <= 0 || num_src_blocks <= 0 || num_dst_blocks <= 0)
    return PA_ERR_INVALID_ARG;
  if (dtype != PA_F32 && dtype != PA_F16 && dtype != PA_BF16 && dtype != PA_FP8_E4M3)
    return PA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  if (num_pairs == 0) return PA_OK;
  if (!dst_k || !dst_v || !src_k || !src_v || !block_mapping) return PA_ERR_INVALID_ARG;
  const void *ptrs[5] = {dst_k, dst_v, src_k, src_v, block_mapping};
  const void *dev[5];
  for (int i = 0; i < 5; ++i) {
    dev[i] = device_view(ptrs[i]);
    if (!dev[i] || (reinterpret_cast<uintptr_t>(dev[i]) & 15u)) return PA_ERR_INVALID_ARG;
  }
  DevInfo di;
  if (device_info(&di) != cudaSuccess) return PA_ERR_CUDA;
  const int64_t tile_bytes =
      (int64_t)block_size * head_dim * (dtype == PA_F32 ? 4 : (dtype == PA_FP8_E4M3 ? 1 : 2));
  const int64_t tiles = (int64_t)num_pairs * 2 * num_kv_heads;
  const int64_t warps_per_cta = kSwapThreads / 32;
  int64_t grid = (tiles + warps_per_cta - 1) / warps_per_cta;
  const int64_t cap = (int64_t)di.sm_count * 8;  // 8 CTAs of 8 warps per SM
  if (grid > cap) grid = cap;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kSwapThreads);
  cfg.stream = (cudaStream_t)stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // a tile is 1 to 16 KiB (a multiple of 16 bytes); 4 vectors per lane move
  // 2 KiB per warp pass
  const cudaError_t e = cudaLaunchKernelEx(
      &cfg, swap_blocks_kernel<4>, (unsigned char *)dev[0], (unsigned char *)dev[1],
      (const unsigned char *)dev[2], (const unsigned char *)dev[3], (const int64_t *)dev[4],
      num_pairs, num_kv_heads, tile_bytes, num_src_blocks, num_dst_blocks, di.err);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
