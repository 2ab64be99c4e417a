// decode_common.cuh -- work enumeration and output merge shared by the paged
// decode kernels (CUDA-core and tensor-core variants).
//
// Work items.  An item is (sequence, KV head, split): the GROUP query heads
// that read one KV head share every K/V byte loaded for the item, and long
// contexts are cut into splits of `split_blocks` KV blocks so that the SMs
// stay busy and the tail stays short (sequence split / KV-head group / work
// queue, "PagedAttention 实战", section 2026 年的新变化).  Every CTA of a
// persistent grid scans the batch once into shared memory -- context length,
// first query row and row count per sequence, and the prefix sum of items --
// and then walks items blockIdx.x, blockIdx.x + gridDim.x, ...; the dense
// enumeration gives all CTAs item counts within one of each other.
#pragma once

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace dec {

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Items contributed by a sequence: its splits for a decode sequence (one query
// row); for a chunk of Q > 1 rows, Q single-row items in row mode and none
// otherwise (the chunk kernel takes them).
__device__ __forceinline__ int seq_items(const AttnArgs &a, int L, int qlen) {
  if (qlen <= 0) return 0;
  if (qlen > 1) return a.rows_mode ? qlen : 0;
  if (L <= 0 || L > a.max_context_len) return 1;  // zero-output item
  return ceil_div(ceil_div(L, a.block_size), a.split_blocks);
}

struct Item {
  int seq;     // global sequence index
  int qrow;    // query row (token index into q / out)
  int split;
  int nsplit;
  int kvh;
  int b0, b1;  // KV blocks [b0, b1) of the sequence
  int L;       // keys visible to the row
  unsigned int bad_bits;  // PA_DEVERR_* of an invalid sequence (0: ok)
};

// Shared-memory copies of the batch made by scan_batch().
struct BatchSmem {
  int *len;     // [n] context length
  int *q0;      // [n] first query row
  int *ql;      // [n] query rows
  int *prefix;  // [n+1] items before sequence s (in units of KV-head groups)
  int *scan;    // [32] scratch
  static constexpr int bytes(int n) { return 4 * (4 * n + 1) + 4 * 32 + 16; }
  __device__ void carve(unsigned char *base, int n) {
    len = reinterpret_cast<int *>(base);
    q0 = len + n;
    ql = q0 + n;
    prefix = ql + n;
    scan = reinterpret_cast<int *>(base + align_up(4 * (4 * n + 1), 16));
  }
};

// Called by every thread of the CTA; ends with __syncthreads().
__device__ __forceinline__ void scan_batch(const AttnArgs &a, const BatchSmem &b, int n) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nthreads = blockDim.x;
  const int per = ceil_div(n, nthreads);
  const int s0 = min(n, tid * per), s1 = min(n, s0 + per);
  int local = 0;
  for (int s = s0; s < s1; ++s) {
    const int gs = a.seq_begin + s;
    int q0 = gs, q1 = gs + 1;
    if (a.query_start_loc) {
      q0 = a.query_start_loc[gs];
      q1 = a.query_start_loc[gs + 1];
      if (q0 < 0 || q1 < q0 || q1 > a.num_q_tokens) {  // rows outside q: no items
        raise_error(a.err, PA_DEVERR_QUERY_LEN);
        q1 = q0 = 0;
      }
    }
    const int L = a.context_lens[gs];
    b.len[s] = L;
    b.q0[s] = q0;
    b.ql[s] = q1 - q0;
    local += seq_items(a, L, q1 - q0);
  }
  int x = local;  // block exclusive scan of `local`
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) b.scan[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int nw = nthreads >> 5;
    int w = lane < nw ? b.scan[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) b.scan[lane] = w;  // inclusive warp totals
  }
  __syncthreads();
  int run = (warp ? b.scan[warp - 1] : 0) + x - local;
  for (int s = s0; s < s1; ++s) {
    b.prefix[s] = run;
    run += seq_items(a, b.len[s], b.ql[s]);
  }
  if (tid == nthreads - 1) b.prefix[n] = run;
  __syncthreads();
}

__device__ __forceinline__ Item decode_item(const AttnArgs &a, const BatchSmem &b, int n, int w) {
  Item it;
  const int f = w / a.num_kv_heads;
  it.kvh = w - f * a.num_kv_heads;
  int lo = 0, hi = n;  // find s with prefix[s] <= f < prefix[s+1]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (b.prefix[mid] <= f) lo = mid; else hi = mid;
  }
  it.seq = a.seq_begin + lo;
  const int L = b.len[lo];
  const int q0 = b.q0[lo];
  const int qlen = b.ql[lo];
  it.bad_bits = 0;
  if (L < 0 || L > a.max_context_len) it.bad_bits = PA_DEVERR_CONTEXT_LEN;
  else if (qlen > L && L > 0) it.bad_bits = PA_DEVERR_QUERY_LEN;
  if (qlen > 1) {  // row mode: one item per query row, never split
    const int t = f - b.prefix[lo];
    it.qrow = q0 + t;
    it.split = 0;
    it.nsplit = 1;
    it.L = L - qlen + t + 1;
  } else {
    it.qrow = q0;
    it.split = f - b.prefix[lo];
    it.nsplit = b.prefix[lo + 1] - b.prefix[lo];
    it.L = L;
  }
  if (it.bad_bits || it.L <= 0) {
    it.b0 = it.b1 = 0;
  } else {
    const int nblk = ceil_div(it.L, a.block_size);
    it.b0 = qlen > 1 ? 0 : it.split * a.split_blocks;
    it.b1 = qlen > 1 ? nblk : min(nblk, it.b0 + a.split_blocks);
  }
  return it;
}

template <typename T>
__device__ __forceinline__ void store4(T *dst, float4 v);
template <>
__device__ __forceinline__ void store4<float>(float *dst, float4 v) {
  *reinterpret_cast<float4 *>(dst) = v;
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16 *dst, float4 v) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t *>(&lo);
  u.y = *reinterpret_cast<uint32_t *>(&hi);
  *reinterpret_cast<uint2 *>(dst) = u;
}
template <>
__device__ __forceinline__ void store4<__half>(__half *dst, float4 v) {
  __half2 lo = __floats2half2_rn(v.x, v.y), hi = __floats2half2_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t *>(&lo);
  u.y = *reinterpret_cast<uint32_t *>(&hi);
  *reinterpret_cast<uint2 *>(dst) = u;
}

// Merge area written by the consumer warps at the end of an item: warp w, its
// head h (of `gw` heads per warp) at merge + w*mstride + h*(D+4):
//   [0, D) unnormalised accumulator, [D] running max (base 2), [D+1] running
//   sum, [D+2] nonzero if the item saw a bad block.
// Warp w = bl*hsplit + hs handled heads hs*gw .. hs*gw+gw-1 of the group for
// the blocks j = bl (mod nbl).  All consumer threads (ncw*32) call this;
// direct items go to `out`, split items to the workspace.
template <typename T, int D>
__device__ __forceinline__ void merge_store(const AttnArgs &a, const Item &item,
                                            const float *merge, int mstride, int gw,
                                            int hsplit, int nbl, int ncw, int tid) {
  constexpr int D4 = D / 4;
  const int total4 = a.group * D4;
  const bool direct = item.nsplit == 1;
  for (int idx = tid; idx < total4; idx += ncw * 32) {
    const int hg = idx / D4;  // head within the group
    const int d4 = idx - hg * D4;
    const int hsub = hg / gw, h = hg - hsub * gw;
    float M = -INFINITY;
    bool anybad = false;
    for (int b2 = 0; b2 < nbl; ++b2) {
      const float *src = merge + (b2 * hsplit + hsub) * mstride + h * (D + 4);
      M = fmaxf(M, src[D]);
      anybad |= src[D + 2] != 0.f;
    }
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    float Lsum = 0.f;
    for (int b2 = 0; b2 < nbl; ++b2) {
      const float *src = merge + (b2 * hsplit + hsub) * mstride + h * (D + 4);
      const float mb = src[D];
      const float wgt = mb == -INFINITY ? 0.f : fast_exp2(mb - M);
      Lsum += wgt * src[D + 1];
      const float4 x = *reinterpret_cast<const float4 *>(src + d4 * 4);
      o.x += wgt * x.x;
      o.y += wgt * x.y;
      o.z += wgt * x.z;
      o.w += wgt * x.w;
    }
    const int head = item.kvh * a.group + hg;
    if (direct) {
      const float inv = (Lsum > 0.f && !anybad) ? 1.f / Lsum : 0.f;
      T *dst = static_cast<T *>(a.out) + ((int64_t)item.qrow * a.num_heads + head) * D + d4 * 4;
      store4<T>(dst, make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv));
    } else {
      const int64_t pidx = ((int64_t)item.seq * a.num_heads + head) * a.max_splits + item.split;
      *reinterpret_cast<float4 *>(a.part_o + pidx * D + d4 * 4) = o;
      if (d4 == 0) {
        a.part_ml[2 * pidx] = M;
        a.part_ml[2 * pidx + 1] = anybad ? __int_as_float(0x7fc00000) : Lsum;
      }
    }
  }
}

}  // namespace dec
}  // namespace pa
