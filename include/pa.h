/*
 * pa.h -- C ABI of libpa.so: paged KV-cache attention on NVIDIA B200 (sm_100a).
 *
 * The KV cache of every sequence is stored in fixed-size blocks (16 or 32
 * tokens) that sit anywhere in one global pool; a per-sequence block table
 * maps logical block i to a physical block id, and several sequences may point
 * at the same physical block to share a prefix ("核心概念" (vLLM concepts
 * page), sections 核心概念：块（Block）, 逻辑视图与物理视图分离 and 内存共享;
 * "理解 vLLM PagedAttention", sections 三 and 六).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor arguments are caller-owned DEVICE pointers to contiguous
 *    row-major arrays; the library never allocates, frees or keeps them.
 *  - Element types: PA_F32 (float), PA_F16 (IEEE half), PA_BF16 (bfloat16).
 *    q, out and both caches share one dtype; accumulation is fp32.
 *  - Layouts (fixed by this library; the pages prescribe none):
 *        k_cache, v_cache   [num_blocks][num_kv_heads][block_size][head_dim]
 *        key, value         [num_tokens][num_kv_heads][head_dim]
 *        q, out             [num_q_tokens][num_heads][head_dim]
 *        block_tables       int32 [num_seqs][max_blocks_per_seq]
 *    Every (block, kv-head) tile is one contiguous block_size*head_dim run.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and return once the work is enqueued.
 *  - Supported: head_dim in {64, 128}; block_size in {16, 32};
 *    num_heads % num_kv_heads == 0 with group = num_heads / num_kv_heads a
 *    multiple of one of {4, 2, 1} and group / {4|2|1} <= 8.  Pointers to
 *    caches, q, out, key and value must be 16-byte aligned.
 *  - Errors: a negative pa_status is returned and NOTHING is launched when
 *    an argument is invalid or unsupported (checked on the host).  Values
 *    only the device sees (block ids, slots, context lengths) are checked by
 *    the kernels: a bad item is skipped, its outputs are written as zeros and
 *    a bit is OR-ed into a per-device error word (PA_DEVERR_*), which
 *    pa_get_device_error() reads and clears.  Kernels never trap and every
 *    wait inside them is bounded in time.
 *
 * Departures from the boundary as first planned
 * ----------------------------------------------
 * The planned prototypes were pa_reshape_and_cache, pa_decode,
 * pa_copy_blocks, a four-argument pa_decode_workspace_size(num_q_tokens,
 * num_heads, head_dim, max_context_len), pa_get_device_error(int *, stream)
 * and pa_status_string, with the element type as a pa_dtype.  What ships
 * differs as follows, each for the reason given:
 *  - dtype is an `int` holding a pa_dtype value in every entry point: the
 *    size of a C enum is up to the compiler, an int is not, and the byte
 *    movers take one more value (PA_FP8_E4M3) than the attention calls.
 *  - pa_decode adds num_q_tokens (rows of q/out; with query_start_loc ==
 *    NULL it must equal num_seqs), max_query_len (host bound of any
 *    sequence's query rows: sequences with more than one row go to the
 *    chunked-prefill kernel, whose grid it sizes) and kv_split_tokens (0 =
 *    the library's balanced partition; > 0 forces fixed splits of that many
 *    tokens, used to test the split path on small inputs).
 *  - pa_decode_workspace_size takes (num_seqs, num_heads, num_kv_heads,
 *    head_dim, block_size, max_context_len, kv_split_tokens): the split
 *    policy depends on num_seqs * num_kv_heads and on block_size, the
 *    balanced partition's per-CTA records on group = num_heads /
 *    num_kv_heads and on the device's SM count, and a forced split on
 *    kv_split_tokens; num_q_tokens does not enter.
 *  - pa_get_device_error writes an `unsigned int`: the word is a set of
 *    PA_DEVERR_* bits that kernels OR in atomically.
 *  - Added entry points for the rows after the core path:
 *    pa_decode_shared_prefix (+ its workspace size), pa_reshape_and_cache_fp8,
 *    pa_decode_fp8, pa_decode_fp8_rows (+ its workspace size),
 *    pa_decode_shared_prefix_fp8 (+ its workspace size),
 *    pa_swap_blocks, pa_decode_noalloc (+
 *    pa_noalloc_scratch_bytes) and pa_abi_version.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* cudaStream_t is `struct CUstream_st *` */

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = -1, /* null pointer, bad size, misaligned pointer, ... */
  PA_ERR_UNSUPPORTED = -2, /* head_dim / block_size / group outside the list above */
  PA_ERR_WORKSPACE = -3,   /* workspace missing or smaller than required */
  PA_ERR_CUDA = -4         /* a CUDA runtime call or kernel launch failed */
} pa_status;

/* PA_FP8_E4M3: 1-byte E4M3 codes with one scale per cache tensor; only the
 * caches of the *_fp8 entry points and the byte movers (pa_copy_blocks,
 * pa_swap_blocks) take it. */
typedef enum { PA_F32 = 0, PA_F16 = 1, PA_BF16 = 2, PA_FP8_E4M3 = 3 } pa_dtype;

/* Bits of the device error word. */
#define PA_DEVERR_BLOCK_ID 0x1u    /* block id outside [0, num_blocks) */
#define PA_DEVERR_SLOT 0x2u        /* slot outside [0, num_blocks*block_size) */
#define PA_DEVERR_CONTEXT_LEN 0x4u /* context_len < 0 or > max_blocks_per_seq*block_size */
#define PA_DEVERR_QUERY_LEN 0x8u   /* query rows of a sequence exceed its context */
#define PA_DEVERR_TIMEOUT 0x10u    /* a bounded wait inside a kernel expired */
#define PA_DEVERR_PREFIX 0x20u     /* pa_decode_shared_prefix: malformed group arrays,
                                      a member whose context is shorter than the
                                      group's shared prefix, or a member whose block
                                      table differs from the group's first sequence
                                      over the shared range */
#define PA_DEVERR_STAGING 0x40u    /* pa_decode_fp8_rows / pa_decode_shared_prefix_fp8:
                                      the blocks to stage exceed staged_blocks */

/*
 * pa_reshape_and_cache -- write this step's new K/V into their cache slots.
 *
 * Defined by: each step computes only the current token's K and V and stores
 * them for later steps ("核心概念", section 为什么需要 KV Cache); a token at
 * position pos of a sequence with block table T goes to slot
 * T[pos / block_size] * block_size + pos % block_size, i.e. block
 * slot / block_size, offset slot % block_size (section 逻辑视图与物理视图分离).
 *
 *   key, value      [num_tokens][num_kv_heads][head_dim], dtype
 *   k_cache,v_cache [num_blocks][num_kv_heads][block_size][head_dim], written
 *   slot_mapping    int64 [num_tokens]; a negative slot skips the token
 *                   (padding).  Two tokens must not share a slot.
 * Byte-exact copy; no arithmetic on the values.
 */
int pa_reshape_and_cache(const void *key, const void *value, void *k_cache,
                         void *v_cache, const int64_t *slot_mapping,
                         int num_tokens, int num_kv_heads, int head_dim,
                         int block_size, int num_blocks, int dtype,
                         struct CUstream_st *stream);

/*
 * pa_copy_blocks -- copy-on-write block copy.
 *
 * Defined by: sequences share physical blocks until they diverge; the shared
 * block is then copied so that each writer owns its block ("理解 vLLM
 * PagedAttention", section 六; "PagedAttention 实战", section PagedAttention
 * 的核心, item 3).
 *
 *   block_mapping  int64 [num_pairs][2] = {src, dst}; copies K and V of all
 *                  KV heads of block src onto block dst.  dtype may also be
 *                  PA_FP8_E4M3 (1-byte elements).  A dst must not
 *                  appear twice nor also be a src in the same call (the
 *                  result would depend on ordering).
 * Byte-exact copy.
 */
int pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *block_mapping,
                   int num_pairs, int num_kv_heads, int head_dim,
                   int block_size, int num_blocks, int dtype,
                   struct CUstream_st *stream);

/*
 * pa_swap_blocks -- move whole blocks from one pool to another, either of
 * which may live in page-locked host memory: swap-out (device pool -> host
 * pool) and swap-in (host -> device) of the blocks of preempted or inactive
 * sequences.
 *
 * Defined by: the KV cache is tiered -- device memory holds the blocks of
 * active requests, host memory the blocks that overflow, and blocks move
 * between the tiers ("核心概念", section 内存层次结构); preemption frees device
 * blocks when memory runs short ("理解 vLLM PagedAttention", section 五).
 *
 *   dst_k, dst_v    [num_dst_blocks][num_kv_heads][block_size][head_dim], written
 *   src_k, src_v    [num_src_blocks][num_kv_heads][block_size][head_dim]
 *   block_mapping   int64 [num_pairs][2] = {src block, dst block}
 * Each of the five pointers may be device memory, managed memory or
 * page-locked host memory (cudaHostAlloc / cudaHostRegister, or a pinned
 * PyTorch tensor); the kernel reads and writes host memory directly over the
 * host link.  Pageable host memory is rejected (PA_ERR_INVALID_ARG, nothing
 * launched).  All five must be 16-byte aligned.  A dst block must not appear
 * twice; when both pools are the same arrays, a dst must also not be a src
 * of the same call.  Byte-exact copy.
 * Device checks: a pair with src outside [0, num_src_blocks) or dst outside
 * [0, num_dst_blocks) is skipped and PA_DEVERR_BLOCK_ID is set.
 */
int pa_swap_blocks(void *dst_k, void *dst_v, const void *src_k,
                   const void *src_v, const int64_t *block_mapping,
                   int num_pairs, int num_kv_heads, int head_dim,
                   int block_size, int num_src_blocks, int num_dst_blocks,
                   int dtype, struct CUstream_st *stream);

/*
 * pa_reshape_and_cache_fp8 -- pa_reshape_and_cache into an FP8 (E4M3) cache.
 *
 * Defined by: KV-cache quantisation ("理解 vLLM PagedAttention", 版本矩阵:
 * 量化 FP8 ... 权重 KV cache 量化); slots as pa_reshape_and_cache.  Element x of
 * a new key is stored as the E4M3 code (1 sign, 4 exponent bits with bias 7,
 * 3 mantissa bits, no infinities, largest magnitude 448) of the IEEE binary32
 * quotient x / k_scale, rounded to nearest with ties to even and saturated
 * to +-448 (NaN -> NaN); values likewise with v_scale.
 *
 *   key, value       [num_tokens][num_kv_heads][head_dim] of in_dtype
 *                    (PA_F32, PA_F16 or PA_BF16)
 *   k_cache, v_cache uint8 [num_blocks][num_kv_heads][block_size][head_dim]
 *   k_scale, v_scale positive finite per-tensor scales
 * The codes are bit-exact functions of the inputs (no other arithmetic).
 */
int pa_reshape_and_cache_fp8(const void *key, const void *value, void *k_cache,
                             void *v_cache, const int64_t *slot_mapping,
                             int num_tokens, int num_kv_heads, int head_dim,
                             int block_size, int num_blocks, int in_dtype,
                             float k_scale, float v_scale,
                             struct CUstream_st *stream);

/*
 * pa_decode_fp8 -- pa_decode (one query row per sequence) over FP8 (E4M3)
 * caches written by pa_reshape_and_cache_fp8: key element = code * k_scale,
 * value element = code * v_scale, and out = softmax(scale * q . K^T) V in
 * fp32 accumulation.  The cache holds one byte per element, so decode reads
 * half the bytes of a 16-bit cache.
 *
 *   q, out           [num_seqs][num_heads][head_dim] of q_dtype (PA_F16 or PA_BF16)
 *   k_cache, v_cache uint8 codes as above
 *   workspace        >= pa_decode_workspace_size(num_seqs, num_heads,
 *                    num_kv_heads, head_dim, block_size, max_context_len, 0) bytes
 * Other arguments, checks and device error reporting as for pa_decode.
 * Supported: num_seqs <= 2048 and group = num_heads / num_kv_heads <= 16.
 */
int pa_decode_fp8(void *out, const void *q, const void *k_cache,
                  const void *v_cache, const int32_t *block_tables,
                  int max_blocks_per_seq, const int32_t *context_lens,
                  int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                  int block_size, int num_blocks, float scale, float k_scale,
                  float v_scale, int max_context_len, int q_dtype,
                  void *workspace, size_t workspace_bytes,
                  struct CUstream_st *stream);

/*
 * pa_decode_fp8_rows -- pa_decode_fp8 for a batch that also holds chunked-
 * prefill rows (query_start_loc, num_q_tokens and max_query_len as in
 * pa_decode): decode rows as pa_decode_fp8; the rows of a sequence with Q > 1
 * see keys 0 .. L-Q+t ("PagedAttention 实战", section Chunked Prefill) over the
 * same FP8 codes (key = code * k_scale, value = code * v_scale).
 *
 * The chunk rows run on the 16-bit tensor-core chunk kernel: the blocks of
 * every sequence with Q > 1 are first copied out of the cache into a staging
 * pool inside the workspace as the 16-bit values of their codes (q's type;
 * every E4M3 value is exact there), k_scale folded into the logit scale and
 * v_scale applied to O / l.
 *
 *   staged_blocks  host-side bound of the staging pool in blocks: at least
 *                  sum over the sequences with Q > 1 of
 *                  ceil(context_len / block_size); > 0 when max_query_len > 1.
 *                  A batch holding more blocks sets PA_DEVERR_STAGING, and the
 *                  rows of the sequences whose blocks did not fit are written
 *                  as zeros (with PA_DEVERR_BLOCK_ID).
 *   workspace      >= pa_decode_fp8_rows_workspace_size(...) bytes.
 * Other arguments as for pa_decode_fp8; the chunk rows need head_dim 128 and
 * group <= 64 for the tensor-core kernels (else the mma.sync chunk kernel).
 * The chunk rows (staging and chunk kernel) run on the library's
 * high-priority stream beside the decode rows, forked from `stream` and
 * joined back into it as in pa_decode (PA_MIXED_OVERLAP=0: one after the
 * other on `stream`).
 */
size_t pa_decode_fp8_rows_workspace_size(int num_seqs, int num_heads,
                                         int num_kv_heads, int head_dim,
                                         int block_size, int max_context_len,
                                         int max_blocks_per_seq,
                                         int staged_blocks);

int pa_decode_fp8_rows(void *out, const void *q, const void *k_cache,
                       const void *v_cache, const int32_t *block_tables,
                       int max_blocks_per_seq, const int32_t *context_lens,
                       const int32_t *query_start_loc, int num_seqs,
                       int num_q_tokens, int max_query_len, int num_heads,
                       int num_kv_heads, int head_dim, int block_size,
                       int num_blocks, float scale, float k_scale,
                       float v_scale, int max_context_len, int staged_blocks,
                       int q_dtype, void *workspace, size_t workspace_bytes,
                       struct CUstream_st *stream);

/*
 * pa_decode_workspace_size -- bytes of device scratch pa_decode needs for
 * split-KV partial results (0 when no sequence is split).  Arguments as for
 * pa_decode; depends on the current device's SM count.
 */
size_t pa_decode_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                int head_dim, int block_size,
                                int max_context_len, int kv_split_tokens);

/*
 * pa_decode -- attention of each sequence's query token(s) over its paged KV.
 *
 * Defined by: at each step the new token attends to all earlier tokens of its
 * sequence, whose K/V are read from the cache ("核心概念", section 为什么需要
 * KV Cache); decode reads the whole KV history and is bound by memory
 * traffic ("PagedAttention 实战", section 先理解 KV Cache, Decode).  For query
 * head h (KV head h / group), context length L and query rows t = 0..Q-1 of
 * a sequence (Q = 1 for decode, Q > 1 for a chunked-prefill chunk, section
 * Chunked Prefill), row t sees keys 0 .. L-Q+t and
 *     out = softmax(scale * q . K^T) V        (fp32 accumulation).
 * Long contexts are split across CTAs (split-KV) and merged by a second
 * kernel, following the decode-scheduling idea of organising work by page,
 * KV-head group and sequence split ("PagedAttention 实战", section 2026 年的
 * 新变化).
 *
 *   out, q            [num_q_tokens][num_heads][head_dim]; out must not alias q
 *   block_tables      int32 [num_seqs][max_blocks_per_seq]; only the first
 *                     ceil(context_len / block_size) entries of a row are read
 *   context_lens      int32 [num_seqs]: tokens in the cache for the sequence,
 *                     this step's tokens included (they must already have been
 *                     written with pa_reshape_and_cache)
 *   query_start_loc   int32 [num_seqs + 1] prefix offsets of each sequence's
 *                     query rows in q, or NULL for one row per sequence
 *                     (num_q_tokens == num_seqs)
 *   max_query_len     host-side upper bound of the rows of any sequence (1 for
 *                     pure decode); rows of sequences with Q > 1 go to the
 *                     chunked-query kernel
 *   scale             softmax scale (typically 1/sqrt(head_dim))
 *   max_context_len   host-side upper bound of context_lens (0: use
 *                     max_blocks_per_seq * block_size)
 *   kv_split_tokens   0: library policy; > 0: split every sequence's KV into
 *                     pieces of this many tokens (rounded down to blocks)
 *   workspace         device scratch of >= pa_decode_workspace_size(...) bytes
 *                     (may be NULL when that size is 0); contents need no
 *                     initialisation and are not meaningful after the call.
 * Context length 0 gives zero output.
 * A batch with both decode rows and chunk rows (max_query_len > 1) runs its
 * chunk rows on a library stream of the device's highest priority, forked
 * from `stream` and joined back into it with events: work enqueued on
 * `stream` after the call is ordered after all of it, also inside a CUDA
 * graph capture.  That stream and its two events are created on the first
 * such call on a device made outside a stream capture (until then, and with
 * the environment variable PA_MIXED_OVERLAP=0, both parts run on `stream`,
 * one after the other).  One fork-join at a time per device: concurrent
 * calls from several host threads serialise their enqueueing.
 */
int pa_decode(void *out, const void *q, const void *k_cache,
              const void *v_cache, const int32_t *block_tables,
              int max_blocks_per_seq, const int32_t *context_lens,
              const int32_t *query_start_loc, int num_seqs, int num_q_tokens,
              int max_query_len, int num_heads, int num_kv_heads, int head_dim,
              int block_size, int num_blocks, float scale, int max_context_len,
              int kv_split_tokens, int dtype, void *workspace,
              size_t workspace_bytes, struct CUstream_st *stream);

/*
 * pa_decode_noalloc -- pa_decode without a caller-supplied workspace.
 *
 * The pages have no counterpart to this entry point: it exists for callers
 * that cannot allocate device memory -- a plugin whose host framework owns
 * all device memory, a runtime whose memory budget is fixed at start-up, or a
 * serving loop that must not call cudaMalloc on its hot path (an allocation
 * can synchronise the device and is not allowed in every stream-capture
 * mode).  The scratch that pa_decode would take from `workspace` comes
 * instead from a static device array of PA_NOALLOC_SCRATCH_BYTES bytes built
 * into the library; every GPU that loads the library holds it until the
 * process exits.  This function allocates nothing and calls no allocating
 * routine; a mixed batch's chunk rows run on `stream` after its decode rows
 * (no side stream or event is created).
 *
 * Arguments and results are those of pa_decode (without workspace).
 * PA_ERR_WORKSPACE (nothing launched) if the batch needs more scratch than
 * the array holds.  The call checks what its own launch needs, which can be
 * less than pa_decode_workspace_size() reports: that function is an upper
 * bound sized for 8 resident CTAs per SM.  16-bit caches with
 * kv_split_tokens = 0 need at most 8 * SMs * 2 * group * (head_dim + 4) * 4
 * bytes plus a few KiB, so on a 148-SM B200 every group <= 8 at head_dim
 * 128 and every group <= 16 at head_dim 64 fits whatever the occupancy;
 * group 16 at head_dim 128 fits at the occupancy the decode kernel reaches
 * for groups above 8 (2 CTAs per SM at its 232 registers per thread, about
 * 5 MiB) but not at the bound.  Fixed splits
 * (kv_split_tokens > 0) need num_seqs * num_heads * splits * (head_dim + 2)
 * * 4 bytes.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress); make that first call before any stream capture.
 * All calls share the one array and it keeps the last call's contents:
 * nothing in it has to start at zero, but calls whose kernels overlap on the
 * GPU (other streams, other host threads) race on it -- serialise them.
 */
#define PA_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

int pa_decode_noalloc(void *out, const void *q, const void *k_cache,
                      const void *v_cache, const int32_t *block_tables,
                      int max_blocks_per_seq, const int32_t *context_lens,
                      const int32_t *query_start_loc, int num_seqs,
                      int num_q_tokens, int max_query_len, int num_heads,
                      int num_kv_heads, int head_dim, int block_size,
                      int num_blocks, float scale, int max_context_len,
                      int kv_split_tokens, int dtype, struct CUstream_st *stream);

/* Size of the static scratch array pa_decode_noalloc uses, in bytes. */
size_t pa_noalloc_scratch_bytes(void);

/*
 * pa_decode_shared_prefix -- decode attention for batches in which groups of
 * sequences share the leading blocks of their block tables.
 *
 * Defined by: sequences forked from one prompt (parallel sampling, beam
 * search) map the prompt's logical blocks to the same physical blocks and
 * own only the blocks written after the fork ("理解 vLLM PagedAttention",
 * section 六; "核心概念", section 内存共享; "PagedAttention 实战", section
 * PagedAttention 的核心, item 3).  The result is exactly pa_decode's (the
 * sharing changes where the keys live, not the attention): for every
 * sequence i and head h, out = softmax(scale * q . K_i^T) V_i over all
 * context_lens[i] keys.  Only the work differs: the shared blocks of a group
 * are read once for all of its sequences' query rows (members x GROUP heads
 * of one KV head form one matrix product), the private tails are read per
 * sequence, and the two partial softmax results are merged.
 *
 *   out, q, k_cache, v_cache, block_tables, context_lens, scale,
 *   max_context_len: as for pa_decode with one query row per sequence
 *                    (num_q_tokens == num_seqs, no query_start_loc).
 *   group_start      int32 [num_groups + 1], device: group j is sequences
 *                    group_start[j] .. group_start[j+1]-1.  Nondecreasing,
 *                    within [0, num_seqs]; sequences outside every group
 *                    are plain decode sequences.
 *   group_shared_blocks int32 [num_groups], device: P_j, the number of
 *                    leading block-table entries that every member of group
 *                    j holds in common (the ids of the group's first
 *                    sequence are used); those blocks must be full
 *                    (P_j * block_size <= every member's context length).
 *                    P_j = 0 makes the group plain decode sequences.
 *   max_group_size   host-side upper bound of any group's size (<= 0: num_seqs)
 *   workspace        >= pa_decode_shared_prefix_workspace_size(...) bytes;
 *                    contents need no initialisation.
 * Supported: 16-bit caches (PA_F16, PA_BF16), num_seqs <= 2048, and the
 * head_dim / block_size / group list above.
 * Device checks: malformed group arrays (decreasing or out of range) make
 * every sequence plain decode -- results stay correct -- and set
 * PA_DEVERR_PREFIX; a member whose context is shorter than P_j * block_size
 * or whose table differs from the first sequence's in the shared range gets
 * zero output and PA_DEVERR_PREFIX.
 */
int pa_decode_shared_prefix(void *out, const void *q, const void *k_cache,
                            const void *v_cache, const int32_t *block_tables,
                            int max_blocks_per_seq, const int32_t *context_lens,
                            int num_seqs, const int32_t *group_start,
                            const int32_t *group_shared_blocks, int num_groups,
                            int max_group_size, int num_heads, int num_kv_heads,
                            int head_dim, int block_size, int num_blocks,
                            float scale, int max_context_len, int dtype,
                            void *workspace, size_t workspace_bytes,
                            struct CUstream_st *stream);

/* Workspace bytes pa_decode_shared_prefix needs (current device). */
size_t pa_decode_shared_prefix_workspace_size(int num_seqs, int num_heads,
                                              int num_kv_heads, int head_dim,
                                              int block_size,
                                              int max_context_len);

/*
 * pa_decode_shared_prefix_fp8 -- pa_decode_shared_prefix over FP8 (E4M3)
 * caches written by pa_reshape_and_cache_fp8 (key = code * k_scale, value =
 * code * v_scale), q/out of q_dtype (PA_F16 or PA_BF16).  The shared blocks of
 * each group's first sequence are copied into a staging pool inside the
 * workspace as the 16-bit values of their codes (exact) and the prefix pass
 * of pa_decode_shared_prefix runs over that pool (k_scale in the logit scale,
 * its partial sums kept in units of 1/v_scale); the private tails run on the
 * FP8 decode kernel, which folds the prefix partials in.  A member whose
 * table differs from its group's first sequence over the shared range is
 * reported and zeroed as in pa_decode_shared_prefix.
 *
 *   staged_blocks  host-side bound of the staging pool in blocks: at least
 *                  sum over groups of group_shared_blocks[j]; > 0 when
 *                  num_groups > 0.  A batch holding more sets
 *                  PA_DEVERR_STAGING (the groups past the bound read as bad
 *                  blocks: their members' rows are zeros).
 *   workspace      >= pa_decode_shared_prefix_fp8_workspace_size(...) bytes.
 * Supported: group = num_heads / num_kv_heads <= 16, num_seqs <= 2048.
 */
int pa_decode_shared_prefix_fp8(void *out, const void *q, const void *k_cache,
                                const void *v_cache, const int32_t *block_tables,
                                int max_blocks_per_seq,
                                const int32_t *context_lens, int num_seqs,
                                const int32_t *group_start,
                                const int32_t *group_shared_blocks,
                                int num_groups, int max_group_size,
                                int num_heads, int num_kv_heads, int head_dim,
                                int block_size, int num_blocks, float scale,
                                float k_scale, float v_scale,
                                int max_context_len, int staged_blocks,
                                int q_dtype, void *workspace,
                                size_t workspace_bytes,
                                struct CUstream_st *stream);

/* Workspace bytes pa_decode_shared_prefix_fp8 needs (current device). */
size_t pa_decode_shared_prefix_fp8_workspace_size(int num_seqs, int num_heads,
                                                  int num_kv_heads,
                                                  int head_dim, int block_size,
                                                  int max_context_len,
                                                  int max_blocks_per_seq,
                                                  int num_groups,
                                                  int staged_blocks);

/*
 * pa_get_device_error -- synchronise `stream`, then read and clear the
 * current device's error word (PA_DEVERR_* bits, 0 = none) into *code_out.
 */
int pa_get_device_error(unsigned int *code_out, struct CUstream_st *stream);

/* Human-readable name of a pa_status value (static string). */
const char *pa_status_string(int status);

/* ABI version of this header: (major << 16) | minor. */
int pa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
