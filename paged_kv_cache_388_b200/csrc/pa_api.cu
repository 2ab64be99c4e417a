// pa_api.cu -- the C ABI of libpa.so: argument checks, split policy, launches.
//
// Nothing here allocates device memory.  The only device state the library
// owns is one error word per device (a file-scope __device__ variable), whose
// address is looked up once per device, and, once a device has served a mixed
// batch through pa_decode, a stream of the device's highest priority and two
// events that let the batch's chunk rows run beside its decode rows.
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <map>
#include <mutex>
#include <utility>

#include "../../include/pa.h"
#include "pa_internal.h"

namespace pa {

__device__ unsigned int g_error_word = 0;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
DevInfo g_dev[kMaxDevices];
bool g_dev_ok[kMaxDevices];

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_bytes(int dtype) { return dtype == PA_F32 ? 4 : (dtype == PA_FP8_E4M3 ? 1 : 2); }

bool dtype_ok(int dtype) { return dtype == PA_F32 || dtype == PA_F16 || dtype == PA_BF16; }

// Byte movers (copy_blocks) also take FP8 caches.
bool byte_dtype_ok(int dtype) { return dtype_ok(dtype) || dtype == PA_FP8_E4M3; }

int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Heads handled by one warp (4, 2 or 1) and how many warps share a KV block.
bool group_supported(int group) {
  if (group <= 0) return false;
  const int gw = group % 4 == 0 ? 4 : (group % 2 == 0 ? 2 : 1);
  return group / gw <= 8;
}

}  // namespace

cudaError_t device_info(DevInfo *info) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_dev_ok[dev]) {
    DevInfo d;
    e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_error_word);
    if (e != cudaSuccess) return e;
    d.err = static_cast<unsigned int *>(p);
    g_dev[dev] = d;
    g_dev_ok[dev] = true;
  }
  *info = g_dev[dev];
  return cudaSuccess;
}

void debug_log(const char *fmt, ...) {
  static const bool on = getenv("PA_DEBUG") != nullptr;
  if (!on) return;
  va_list ap;
  va_start(ap, fmt);
  fputs("[libpa] ", stderr);
  vfprintf(stderr, fmt, ap);
  fputc('\n', stderr);
  va_end(ap);
}

cudaError_t set_smem_limit_once(const void *func, int bytes, bool max_shared) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::mutex mu;
  static std::map<std::pair<const void *, int>, cudaError_t> done;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(func, dev);
  const auto it = done.find(key);
  if (it != done.end()) return it->second;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && max_shared)
    e = cudaFuncSetAttribute(func, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess) done.emplace(key, e);  // failures are retried on the next call
  return e;
}

void split_policy(int num_seqs, int num_kv_heads, int block_size, int max_context_len,
                  int kv_split_tokens, int sm_count, int *split_blocks, int *max_splits) {
  const int nblk_max = max_context_len > 0 ? ceil_div(max_context_len, block_size) : 1;
  int sb;
  if (kv_split_tokens > 0) {
    sb = kv_split_tokens / block_size;
    if (sb < 1) sb = 1;
  } else {
    // Pieces of 512 tokens (256 KiB of K+V per KV head at head_dim 128, 16-bit)
    // keep the merge cost near 1% while giving each CTA many items; very long
    // contexts use at most 64 pieces; small batches split finer (>= 128 tokens)
    // until there are about four items per resident CTA slot.
    int tok = 512;
    if (max_context_len > 64 * 512) tok = ceil_div(ceil_div(max_context_len, 64), block_size) * block_size;
    while (tok > 128 && (int64_t)num_seqs * num_kv_heads * ceil_div(max_context_len, tok) <
                            (int64_t)4 * sm_count)
      tok /= 2;
    sb = tok / block_size;
    if (sb < 1) sb = 1;
  }
  *split_blocks = sb;
  *max_splits = ceil_div(nblk_max, sb);
}


// A mixed batch's chunk rows (tensor-bound) and decode rows (HBM-bound) read
// the same caches and write disjoint output rows, so they need no order between
// them.  The chunk kernel goes to a second stream of the device's highest
// priority, forked from the caller's stream and joined back into it with
// events, and the decode kernel follows on the caller's stream without
// programmatic dependent launch, so that the chunk grid is placed first.  The
// block scheduler places a later grid's CTAs only once the earlier grid has
// none left waiting for an SM, so the decode CTAs start when the chunk grid's
// last wave is placed: on the SMs that wave leaves empty (40 of 148 on the long
// mixed batch) and beside its CTAs (both kernels ask for the largest
// shared-memory carve-out, and a decode CTA fits in what a chunk CTA leaves).
// PA_MIXED_OVERLAP=0 keeps the two on the caller's stream, one after the other.
namespace {
SideStream g_side[kMaxDevices];
}  // namespace

bool mixed_overlap_wanted() {
  static const bool on = [] {
    const char *v = getenv("PA_MIXED_OVERLAP");
    return !(v && strcmp(v, "0") == 0);
  }();
  return on;
}

// Forks the current device's side stream from `caller` and returns it locked,
// or returns nullptr (nothing enqueued, nothing locked): the work then stays on
// the caller's stream.  The stream and events are created on the first mixed
// batch outside a stream capture.
SideStream *side_fork(cudaStream_t caller) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  SideStream &sd = g_side[dev];
  sd.mu.lock();
  if (!sd.ready) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (sd.failed || cudaStreamIsCapturing(caller, &cap) != cudaSuccess ||
        cap != cudaStreamCaptureStatusNone) {
      cudaGetLastError();
      sd.mu.unlock();
      return nullptr;
    }
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) == cudaSuccess &&
        cudaStreamCreateWithPriority(&sd.stream, cudaStreamNonBlocking, greatest) == cudaSuccess &&
        cudaEventCreateWithFlags(&sd.fork, cudaEventDisableTiming) == cudaSuccess &&
        cudaEventCreateWithFlags(&sd.join, cudaEventDisableTiming) == cudaSuccess) {
      sd.ready = true;
    } else {
      debug_log("side stream for mixed batches not created: %s", cudaGetErrorString(cudaGetLastError()));
      sd.failed = true;
      sd.mu.unlock();
      return nullptr;
    }
  }
  if (cudaEventRecord(sd.fork, caller) != cudaSuccess ||
      cudaStreamWaitEvent(sd.stream, sd.fork, 0) != cudaSuccess) {
    debug_log("mixed-batch fork failed: %s", cudaGetErrorString(cudaGetLastError()));
    sd.mu.unlock();
    return nullptr;
  }
  return &sd;
}

// Joins the side stream back into `caller` (also after a failed launch, so that
// a capture in progress stays well formed) and unlocks it.
cudaError_t side_join(SideStream *sd, cudaStream_t caller) {
  cudaError_t e = cudaEventRecord(sd->join, sd->stream);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(caller, sd->join, 0);
  sd->mu.unlock();
  return e;
}


}  // namespace pa

using namespace pa;

extern "C" {

int pa_abi_version(void) { return (1 << 16) | 0; }

const char *pa_status_string(int status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
    case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
    default: return "PA_UNKNOWN_STATUS";
  }
}

int pa_reshape_and_cache(const void *key, const void *value, void *k_cache, void *v_cache,
                         const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                         int head_dim, int block_size, int num_blocks, int dtype,
                         struct CUstream_st *stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0 || !dtype_ok(dtype))
    return PA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
  if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID_ARG;
  DevInfo dev;
  if (device_info(&dev) != cudaSuccess) return PA_ERR_CUDA;
  cudaError_t e = launch_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, num_tokens,
                                           num_kv_heads, head_dim, block_size, num_blocks,
                                           elem_bytes(dtype), dev.err, (cudaStream_t)stream);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *block_mapping, int num_pairs,
                   int num_kv_heads, int head_dim, int block_size, int num_blocks, int dtype,
                   struct CUstream_st *stream) {
  if (num_pairs < 0 || num_kv_heads <= 0 || num_blocks <= 0 || !byte_dtype_ok(dtype))
    return PA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  if (num_pairs == 0) return PA_OK;
  if (!k_cache || !v_cache || !block_mapping) return PA_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(v_cache)) return PA_ERR_INVALID_ARG;
  DevInfo dev;
  if (device_info(&dev) != cudaSuccess) return PA_ERR_CUDA;
  cudaError_t e = launch_copy_blocks(k_cache, v_cache, block_mapping, num_pairs, num_kv_heads,
                                     head_dim, block_size, num_blocks, elem_bytes(dtype), dev.err,
                                     (cudaStream_t)stream);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

size_t pa_decode_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                int block_size, int max_context_len, int kv_split_tokens) {
  if (num_seqs <= 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      max_context_len <= 0)
    return 0;
  DevInfo dev;
  if (device_info(&dev) != cudaSuccess) return 0;
  int sb = 0, ms = 0;
  split_policy(num_seqs, num_kv_heads, block_size, max_context_len, kv_split_tokens,
               dev.sm_count, &sb, &ms);
  size_t fixed = ms <= 1 ? 0 : (size_t)num_seqs * num_heads * ms * (head_dim + 2) * sizeof(float) + 256;
  if (kv_split_tokens > 0 || num_heads % num_kv_heads != 0) return fixed;
  // balanced partition (tensor-core kernel): per-CTA records for at most 8
  // resident CTAs per SM, plus the block prefix of one launch
  const int n = num_seqs < decode_max_seqs_per_launch() ? num_seqs : decode_max_seqs_per_launch();
  const size_t bal = balanced_record_bytes(dev.sm_count * 8, num_heads / num_kv_heads, head_dim) +
                     balanced_desc_bytes(dev.sm_count * 8) + (size_t)(n + 1) * sizeof(int) + 256;
  return fixed > bal ? fixed : bal;
}

}  // extern "C"

namespace pa {

int decode_call(void *out, const void *q, const void *k_cache, const void *v_cache,
                const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                const int32_t *query_start_loc, int num_seqs, int num_q_tokens, int max_query_len,
                int num_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
                float scale, int max_context_len, int kv_split_tokens, int dtype, void *workspace,
                size_t workspace_bytes, struct CUstream_st *stream, bool overlap) {
  if (num_seqs < 0 || num_q_tokens < 0 || num_heads <= 0 || num_kv_heads <= 0 ||
      num_blocks <= 0 || max_blocks_per_seq <= 0 || !dtype_ok(dtype) || kv_split_tokens < 0)
    return PA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  if (num_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
  const int group = num_heads / num_kv_heads;
  if (!group_supported(group)) return PA_ERR_UNSUPPORTED;
  if (!query_start_loc) {
    if (num_q_tokens != num_seqs) return PA_ERR_INVALID_ARG;
    max_query_len = 1;
  } else if (max_query_len < 1) {
    return PA_ERR_INVALID_ARG;
  }
  if (num_seqs == 0 || num_q_tokens == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID_ARG;
  if (out == q) return PA_ERR_INVALID_ARG;
  if ((int64_t)max_blocks_per_seq * block_size > (int64_t)1 << 30) return PA_ERR_UNSUPPORTED;
  const int cap = max_blocks_per_seq * block_size;
  if (max_context_len <= 0 || max_context_len > cap) max_context_len = cap;
  if (max_query_len > 1 && group > 64) return PA_ERR_UNSUPPORTED;

  DevInfo dev;
  if (device_info(&dev) != cudaSuccess) return PA_ERR_CUDA;
  int split_blocks = 0, max_splits = 0;
  split_policy(num_seqs, num_kv_heads, block_size, max_context_len, kv_split_tokens, dev.sm_count,
               &split_blocks, &max_splits);

  AttnArgs a{};
  a.o_scale = 1.f;
  a.out = out;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.query_start_loc = query_start_loc;
  a.err = dev.err;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.group = group;
  a.head_dim = head_dim;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.split_blocks = split_blocks;
  a.max_splits = max_splits;
  a.max_query_len = max_query_len;
  a.max_context_len = max_context_len;
  a.num_q_tokens = num_q_tokens;
  a.scale_log2 = scale * 1.4426950408889634f;
  // fp32 chunk rows have no tensor-core kernel: the decode kernel takes them
  // one query row per work item.
  a.rows_mode = (max_query_len > 1 && dtype == PA_F32) ? 1 : 0;

  // Kernel: tensor cores for 16-bit caches (PA_DECODE_KERNEL=simt forces the
  // CUDA-core kernel, kept for fp32, unusual head groups and comparison).
  const char *sel = getenv("PA_DECODE_KERNEL");
  const bool want_simt = sel && strcmp(sel, "simt") == 0;
  const bool use_mma = !want_simt && !a.rows_mode && decode_mma_supported(a, dtype);
  // Balanced partition unless the caller fixed the split size.
  a.balanced = (use_mma && kv_split_tokens == 0) ? 1 : 0;
  a.item_units = kItemUnits16;
  const int step = decode_max_seqs_per_launch();
  if (a.balanced) {
    AttnArgs probe = a;
    probe.num_seqs = num_seqs < step ? num_seqs : step;
    a.grid = decode_mma_grid(probe, dtype, dev.sm_count);
    if (a.grid <= 0) return PA_ERR_CUDA;
    const size_t rec = balanced_record_bytes(a.grid, group, head_dim);
    const size_t desc = balanced_desc_bytes(a.grid);
    const size_t need = rec + desc + (size_t)(probe.num_seqs + 1) * sizeof(int);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return PA_ERR_WORKSPACE;
    a.part_o = static_cast<float *>(workspace);
    a.bal_desc = reinterpret_cast<int *>(static_cast<char *>(workspace) + rec);
    a.bal_prefix = reinterpret_cast<int *>(static_cast<char *>(workspace) + rec + desc);
  } else if (max_splits > 1) {
    const size_t need = (size_t)num_seqs * num_heads * max_splits * (head_dim + 2) * sizeof(float);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return PA_ERR_WORKSPACE;
    a.part_o = static_cast<float *>(workspace);
    a.part_ml = a.part_o + (size_t)num_seqs * num_heads * max_splits * head_dim;
  }

  cudaStream_t s = (cudaStream_t)stream;
  const bool chunk_rows = max_query_len > 1 && !a.rows_mode;
  SideStream *side = (overlap && chunk_rows && mixed_overlap_wanted()) ? side_fork(s) : nullptr;
  a.no_pdl = side ? 1 : 0;
  cudaError_t e = cudaSuccess;
  for (int s0 = 0; s0 < num_seqs && e == cudaSuccess; s0 += step) {
    a.seq_begin = s0;
    a.num_seqs = num_seqs - s0 < step ? num_seqs - s0 : step;
    // forked: the chunk rows first, so that their CTAs are placed before the decode kernel's
    if (side) e = launch_chunk(a, dtype, num_q_tokens, side->stream);
    if (e == cudaSuccess)
      e = use_mma ? launch_decode_mma(a, dtype, dev.sm_count, s) : launch_decode(a, dtype, dev.sm_count, s);
    if (e == cudaSuccess && a.balanced) e = launch_balanced_reduce(a, dtype, s);
    else if (e == cudaSuccess && max_splits > 1) e = launch_reduce(a, dtype, s);
    if (e == cudaSuccess && chunk_rows && !side) e = launch_chunk(a, dtype, num_q_tokens, s);
  }
  if (side) {
    const cudaError_t j = side_join(side, s);
    if (e == cudaSuccess) e = j;
  }
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace pa

extern "C" {

int pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
              const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
              const int32_t *query_start_loc, int num_seqs, int num_q_tokens, int max_query_len,
              int num_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
              float scale, int max_context_len, int kv_split_tokens, int dtype, void *workspace,
              size_t workspace_bytes, struct CUstream_st *stream) {
  return decode_call(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                     query_start_loc, num_seqs, num_q_tokens, max_query_len, num_heads,
                     num_kv_heads, head_dim, block_size, num_blocks, scale, max_context_len,
                     kv_split_tokens, dtype, workspace, workspace_bytes, stream, true);
}

namespace {

// Workspace of pa_decode_shared_prefix: the balanced decode scheme's records,
// descriptors and block prefix, then the per-sequence shared block counts and
// the prefix kernel's records [num_seqs][num_heads][head_dim + 4].
struct SharedPrefixWs {
  size_t desc, prefix, seq_pre, pre_rec, total;
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

SharedPrefixWs shared_prefix_ws(int num_seqs, int num_heads, int head_dim, int group, int grid) {
  SharedPrefixWs w;
  size_t off = balanced_record_bytes(grid, group, head_dim);
  w.desc = off;
  off += balanced_desc_bytes(grid);
  w.prefix = off;
  off += align256((size_t)(num_seqs + 1) * sizeof(int));
  w.seq_pre = off;
  off += align256((size_t)num_seqs * sizeof(int));
  w.pre_rec = off;
  off += align256((size_t)num_seqs * num_heads * (head_dim + 4) * sizeof(float));
  w.total = off;
  return w;
}

// CTAs per cluster of the prefix kernel (ranges of the shared blocks per
// (group, chunk, KV head)): 1 while there are at least 0.4 units per SM,
// doubled (up to 8) until there are.  Measured on B200 (256 units of 64 blocks): prefix
// kernel 55 us with 1, 81 us with 4.  PA_PREFIX_CLUSTER = 1, 2, 4 or 8
// overrides.
int prefix_cluster(int64_t units, int sm_count) {
  const char *env = getenv("PA_PREFIX_CLUSTER");
  if (env) {
    const int c = atoi(env);
    if (c == 1 || c == 2 || c == 4 || c == 8) return c;
  }
  // one CTA per unit while the units alone give a wave of work: a CTA's
  // fixed cost (Q gather, first loads, merge) then is paid once
  int c = 1;
  while (c < 8 && units * c * 5 < (int64_t)2 * sm_count) c *= 2;
  return c;
}

}  // namespace

size_t pa_decode_shared_prefix_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                              int head_dim, int block_size, int max_context_len) {
  (void)block_size;
  (void)max_context_len;
  if (num_seqs <= 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      num_heads % num_kv_heads != 0)
    return 0;
  DevInfo dev;
  if (device_info(&dev) != cudaSuccess) return 0;
  // the decode grid is at most 8 resident CTAs per SM
  return shared_prefix_ws(num_seqs, num_heads, head_dim, num_heads / num_kv_heads,
                          dev.sm_count * 8).total;
}

int pa_decode_shared_prefix(void *out, const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *block_tables, int max_blocks_per_seq,
                            const int32_t *context_lens, int num_seqs,
                            const int32_t *group_start, const int32_t *group_shared_blocks,
                            int num_groups, int max_group_size, int num_heads, int num_kv_heads,
                            int head_dim, int block_size, int num_blocks, float scale,
                            int max_context_len, int dtype, void *workspace,
                            size_t workspace_bytes, struct CUstream_st *stream) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 ||
      max_blocks_per_seq <= 0 || !dtype_ok(dtype) || num_groups < 0)
    return PA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (num_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
  const int group = num_heads / num_kv_heads;
  if (!group_supported(group)) return PA_ERR_UNSUPPORTED;
  if (num_seqs > decode_max_seqs_per_launch()) return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
    return PA_ERR_INVALID_ARG;
  if (num_groups > 0 && (!group_start || !group_shared_blocks)) return PA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID_ARG;
  if (out == q) return PA_ERR_INVALID_ARG;
  if ((int64_t)max_blocks_per_seq * block_size > (int64_t)1 << 30) return PA_ERR_UNSUPPORTED;
  const int cap = max_blocks_per_seq * block_size;
  if (max_context_len <= 0 || max_context_len > cap) max_context_len = cap;
  if (max_group_size <= 0 || max_group_size > num_seqs) max_group_size = num_seqs;

  DevInfo dev;
  if (device_info(&dev) != cudaSuccess) return PA_ERR_CUDA;
  AttnArgs a{};
  a.o_scale = 1.f;
  a.out = out;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.query_start_loc = nullptr;
  a.err = dev.err;
  a.num_seqs = num_seqs;
  a.seq_begin = 0;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.group = group;
  a.head_dim = head_dim;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.split_blocks = 1;
  a.max_splits = 1;
  a.max_query_len = 1;
  a.max_context_len = max_context_len;
  a.num_q_tokens = num_seqs;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.balanced = 1;
  a.item_units = kItemUnits16;
  if (!decode_mma_supported(a, dtype) || !prefix_supported(a, dtype)) return PA_ERR_UNSUPPORTED;
  a.grid = decode_mma_grid(a, dtype, dev.sm_count);
  if (a.grid <= 0) return PA_ERR_CUDA;
  const SharedPrefixWs w = shared_prefix_ws(num_seqs, num_heads, head_dim, group, a.grid);
  if (!workspace || workspace_bytes < w.total || !aligned16(workspace)) return PA_ERR_WORKSPACE;
  char *ws = static_cast<char *>(workspace);
  a.part_o = reinterpret_cast<float *>(ws);
  a.bal_desc = reinterpret_cast<int *>(ws + w.desc);
  a.bal_prefix = reinterpret_cast<int *>(ws + w.prefix);
  a.seq_pre = reinterpret_cast<int *>(ws + w.seq_pre);
  a.pre_rec = reinterpret_cast<float *>(ws + w.pre_rec);
  a.grp_start = group_start;
  a.grp_blocks = group_shared_blocks;
  a.num_groups = num_groups;
  const int mpc = kPrefixRows / group;
  a.grp_chunks = (max_group_size + mpc - 1) / mpc;
  a.max_group = max_group_size;

  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaSuccess;
  if (num_groups > 0) {
    // the shared blocks on the 5th-generation tensor cores (head_dim 128,
    // group dividing 128): the kernel over 64-key tiles with three S/P
    // buffers; PA_PREFIX_KERNEL=pp selects the ping-pong kernel over 128-key
    // tiles (slower here: a group's rows fill one Q tile at most, so it has no
    // second tile to overlap with -- 0.145 vs 0.122 ms on the parallel-sampling
    // batch), PA_PREFIX_KERNEL=mma the mma.sync cluster kernel, which serves
    // every other shape
    const char *sel = getenv("PA_PREFIX_KERNEL");
    const bool want_mma = sel && strcmp(sel, "mma") == 0;
    const bool want_pp = sel && strcmp(sel, "pp") == 0;
    if (want_pp && chunk_pp_supported(a, dtype)) {
      e = launch_prefix_pp(a, dtype, s);
    } else if (!want_mma && chunk_tc_supported(a, dtype)) {
      e = launch_prefix_tc(a, dtype, s);
    } else {
      const int64_t units = (int64_t)num_groups * a.grp_chunks * num_kv_heads;
      e = launch_prefix(a, dtype, prefix_cluster(units, dev.sm_count), s);
    }
  }
  if (e == cudaSuccess) e = launch_decode_mma(a, dtype, dev.sm_count, s);
  if (e == cudaSuccess) e = launch_balanced_reduce(a, dtype, s);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// Workspace of pa_decode_shared_prefix_fp8: that of pa_decode_shared_prefix,
// then the staging plan (gbase), the staged tables and the two 16-bit pools.
size_t pa_decode_shared_prefix_fp8_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                                  int head_dim, int block_size,
                                                  int max_context_len, int max_blocks_per_seq,
                                                  int num_groups, int staged_blocks) {
  if (max_blocks_per_seq <= 0 || num_groups < 0 || staged_blocks < 0 || block_size <= 0) return 0;
  const size_t base = pa_decode_shared_prefix_workspace_size(num_seqs, num_heads, num_kv_heads,
                                                             head_dim, block_size, max_context_len);
  if (base == 0) return 0;
  auto up = [](size_t x) { return (x + 1023) / 1024 * 1024; };
  return up(base) + up((size_t)(num_groups + 1) * sizeof(int)) +
         up((size_t)num_seqs * max_blocks_per_seq * sizeof(int32_t)) +
         2 * fp8_pool_bytes(staged_blocks, num_kv_heads, head_dim, block_size);
}

int pa_decode_shared_prefix_fp8(void *out, const void *q, const void *k_cache, const void *v_cache,
                                const int32_t *block_tables, int max_blocks_per_seq,
                                const int32_t *context_lens, int num_seqs,
                                const int32_t *group_start, const int32_t *group_shared_blocks,
                                int num_groups, int max_group_size, int num_heads,
                                int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                float scale, float k_scale, float v_scale, int max_context_len,
                                int staged_blocks, int q_dtype, void *workspace,
                                size_t workspace_bytes, struct CUstream_st *stream) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 ||
      max_blocks_per_seq <= 0 || num_groups < 0 || staged_blocks < 0)
    return PA_ERR_INVALID_ARG;
  if (!(k_scale > 0.f && k_scale < 3.0e38f) || !(v_scale > 0.f && v_scale < 3.0e38f))
    return PA_ERR_INVALID_ARG;
  if (q_dtype != PA_F16 && q_dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  if (num_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
  const int group = num_heads / num_kv_heads;
  if (!group_supported(group) || group > 16) return PA_ERR_UNSUPPORTED;
  if (num_seqs > decode_max_seqs_per_launch()) return PA_ERR_UNSUPPORTED;
  if (num_groups > 0 && staged_blocks == 0) return PA_ERR_INVALID_ARG;
  if (num_seqs == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
    return PA_ERR_INVALID_ARG;
  if (num_groups > 0 && (!group_start || !group_shared_blocks)) return PA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID_ARG;
  if (out == q) return PA_ERR_INVALID_ARG;
  if ((int64_t)max_blocks_per_seq * block_size > (int64_t)1 << 30) return PA_ERR_UNSUPPORTED;
  const int cap = max_blocks_per_seq * block_size;
  if (max_context_len <= 0 || max_context_len > cap) max_context_len = cap;
  if (max_group_size <= 0 || max_group_size > num_seqs) max_group_size = num_seqs;

  DevInfo dev;
  if (device_info(&dev) != cudaSuccess) return PA_ERR_CUDA;
  AttnArgs a{};
  a.o_scale = 1.f;
  a.out = out;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.query_start_loc = nullptr;
  a.err = dev.err;
  a.num_seqs = num_seqs;
  a.seq_begin = 0;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.group = group;
  a.head_dim = head_dim;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.split_blocks = 1;
  a.max_splits = 1;
  a.max_query_len = 1;
  a.max_context_len = max_context_len;
  a.num_q_tokens = num_seqs;
  a.scale_log2 = scale * k_scale * 1.4426950408889634f;
  a.v_inv = 1.f / v_scale;
  a.balanced = 1;
  a.item_units = kItemUnitsFp8;
  if (!prefix_supported(a, q_dtype)) return PA_ERR_UNSUPPORTED;
  a.grid = decode_mma_grid_fp8(a, q_dtype, dev.sm_count);
  if (a.grid <= 0) return PA_ERR_CUDA;
  const SharedPrefixWs w = shared_prefix_ws(num_seqs, num_heads, head_dim, group, a.grid);
  auto up = [](size_t x) { return (x + 1023) / 1024 * 1024; };
  const size_t off_g = up(shared_prefix_ws(num_seqs, num_heads, head_dim, group, dev.sm_count * 8).total);
  const size_t off_t = off_g + up((size_t)(num_groups + 1) * sizeof(int));
  const size_t off_k = off_t + up((size_t)num_seqs * max_blocks_per_seq * sizeof(int32_t));
  const size_t pool = fp8_pool_bytes(staged_blocks, num_kv_heads, head_dim, block_size);
  const size_t total = off_k + 2 * pool;
  if (w.total > off_g || !workspace || workspace_bytes < total || !aligned16(workspace))
    return PA_ERR_WORKSPACE;
  char *ws = static_cast<char *>(workspace);
  a.part_o = reinterpret_cast<float *>(ws);
  a.bal_desc = reinterpret_cast<int *>(ws + w.desc);
  a.bal_prefix = reinterpret_cast<int *>(ws + w.prefix);
  a.seq_pre = reinterpret_cast<int *>(ws + w.seq_pre);
  a.pre_rec = reinterpret_cast<float *>(ws + w.pre_rec);
  a.grp_start = group_start;
  a.grp_blocks = group_shared_blocks;
  a.num_groups = num_groups;
  const int mpc = kPrefixRows / group;
  a.grp_chunks = (max_group_size + mpc - 1) / mpc;
  a.max_group = max_group_size;

  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaSuccess;
  if (num_groups > 0) {
    // the shared blocks: staged as 16-bit values of their codes, then the
    // prefix pass of pa_decode_shared_prefix over that pool (k_scale in the
    // logit scale; its records hold l / v_scale, the decode kernel's units)
    int *gbase = reinterpret_cast<int *>(ws + off_g);
    int32_t *tab = reinterpret_cast<int32_t *>(ws + off_t);
    e = launch_fp8_group_stage(a, q_dtype, gbase, tab, ws + off_k, ws + off_k + pool, staged_blocks, s);
    AttnArgs p = a;
    p.k_cache = ws + off_k;
    p.v_cache = ws + off_k + pool;
    p.block_tables = tab;
    p.num_blocks = staged_blocks;
    p.o_scale = v_scale;
    const char *sel = getenv("PA_PREFIX_KERNEL");
    const bool want_mma = sel && strcmp(sel, "mma") == 0;
    const bool want_pp = sel && strcmp(sel, "pp") == 0;
    if (e == cudaSuccess) {
      if (want_pp && chunk_pp_supported(p, q_dtype)) {
        e = launch_prefix_pp(p, q_dtype, s);
      } else if (!want_mma && chunk_tc_supported(p, q_dtype)) {
        e = launch_prefix_tc(p, q_dtype, s);
      } else {
        const int64_t units = (int64_t)num_groups * a.grp_chunks * num_kv_heads;
        e = launch_prefix(p, q_dtype, prefix_cluster(units, dev.sm_count), s);
      }
    }
  }
  if (e == cudaSuccess) e = launch_decode_mma_fp8(a, q_dtype, dev.sm_count, s);
  if (e == cudaSuccess) e = launch_balanced_reduce(a, q_dtype, s);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int pa_get_device_error(unsigned int *code_out, struct CUstream_st *stream) {
  if (!code_out) return PA_ERR_INVALID_ARG;
  DevInfo dev;
  if (device_info(&dev) != cudaSuccess) return PA_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  unsigned int host = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaMemcpyAsync(&host, dev.err, sizeof host, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaMemsetAsync(dev.err, 0, sizeof host, s) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return PA_ERR_CUDA;
  *code_out = host;
  return PA_OK;
}

}  // extern "C"
