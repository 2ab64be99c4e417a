// noalloc.cu -- pa_decode_noalloc: paged decode attention for callers that
// cannot allocate device memory.
//
// pa_decode needs a scratch workspace for partial softmax results when a
// sequence's KV is split across CTAs.  Some callers cannot hand one over: a
// plugin that runs inside a host framework owning all device memory, a
// runtime with a fixed memory budget decided at start-up, or a serving loop
// that must never call cudaMalloc on its hot path (it can synchronise the
// device and is not allowed in every stream-capture mode).  For them this
// entry point uses a scratch area compiled into the library instead: a
// file-scope __device__ array of PA_NOALLOC_SCRATCH_BYTES bytes that every GPU
// loading the library holds until the process exits.
//
// The kernels are pa_decode's own; only where the workspace comes from
// differs.  Nothing in the scratch has to start at zero: every launch writes
// each partial record, descriptor and prefix entry before reading it.
#include <mutex>

#include "../../include/pa.h"
#include "pa_internal.h"

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices];

// Device address of this device's copy of the scratch array.  In host code
// the array's name is only a host-side stand-in, so the address must come
// from cudaGetSymbolAddress, looked up once per device with it current.
int scratch_for_current_device(void **ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return PA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return PA_OK;
}

}  // namespace

extern "C" {

size_t pa_noalloc_scratch_bytes(void) { return (size_t)PA_NOALLOC_SCRATCH_BYTES; }

int pa_decode_noalloc(void *out, const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *block_tables, int max_blocks_per_seq,
                      const int32_t *context_lens, const int32_t *query_start_loc,
                      int num_seqs, int num_q_tokens, int max_query_len, int num_heads,
                      int num_kv_heads, int head_dim, int block_size, int num_blocks,
                      float scale, int max_context_len, int kv_split_tokens, int dtype,
                      struct CUstream_st *stream) {
  void *scratch = nullptr;
  const int rc = scratch_for_current_device(&scratch);
  if (rc != PA_OK) return rc;
  // pa_decode checks the scratch it needs against the array's size and
  // returns PA_ERR_WORKSPACE, launching nothing, when the batch needs more.
  // A mixed batch's chunk rows stay on the caller's stream: the side stream
  // pa_decode forks them onto is created on first use, and this entry point
  // creates nothing.
  return pa::decode_call(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                         query_start_loc, num_seqs, num_q_tokens, max_query_len, num_heads,
                         num_kv_heads, head_dim, block_size, num_blocks, scale, max_context_len,
                         kv_split_tokens, dtype, scratch, (size_t)PA_NOALLOC_SCRATCH_BYTES, stream,
                         false);
}

}  // extern "C"
