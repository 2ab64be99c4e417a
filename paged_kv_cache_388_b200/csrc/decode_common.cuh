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
  int L;       // keys visible to the row, counted from block boff
  int boff;    // leading blocks of the sequence left to the shared-prefix kernel
  unsigned int bad_bits;  // PA_DEVERR_* of an invalid sequence (0: ok)
};

// Shared-memory copies of the batch made by scan_batch().
struct BatchSmem {
  int *len;     // [n] context length
  int *q0;      // [n] first query row
  int *ql;      // [n] query rows
  int *pre;     // [n] leading blocks shared with the sequence's group (0: none)
  int *prefix;  // [n+1] items before sequence s (in units of KV-head groups)
  int *scan;    // [32] scratch
  static constexpr int bytes(int n) { return 4 * (5 * n + 1) + 4 * 32 + 16; }
  __device__ void carve(unsigned char *base, int n) {
    len = reinterpret_cast<int *>(base);
    q0 = len + n;
    ql = q0 + n;
    pre = ql + n;
    prefix = pre + n;
    scan = reinterpret_cast<int *>(base + align_up(4 * (5 * n + 1), 16));
  }
};


// Partition units of a decode sequence (one query row, valid length) per KV
// head: its KV blocks after the `pre` shared-prefix blocks plus kItemUnits,
// or 0 when it has no block of its own.
__device__ __forceinline__ int unit_blocks(const AttnArgs &a, int L, int qlen, int pre) {
  if (qlen != 1 || L <= 0 || L > a.max_context_len) return 0;
  const int tail = L - pre * a.block_size;
  return tail > 0 ? ceil_div(tail, a.block_size) + a.item_units : 0;
}

// Shared-prefix groups -> b.pre[s], the leading KV blocks of sequence s that
// the prefix kernel attends (0 outside every group and when the call has no
// groups).  The group arrays are one list of boundaries, so checking that
// every group is an in-range, nondecreasing range [start_j, start_j+1) with a
// block count inside the table proves that the groups are disjoint.  When any
// group fails, no sequence takes the shared path: each is attended in full by
// the decode kernel (the result is the same) and PA_DEVERR_PREFIX is raised.
// Called by every thread of the CTA; ends with a barrier.
__device__ __forceinline__ void scan_groups(const AttnArgs &a, const BatchSmem &b, int n) {
  for (int s = threadIdx.x; s < n; s += blockDim.x) b.pre[s] = 0;
  bool ok = true;
  if (a.pre_rec) {
    for (int j = threadIdx.x; j < a.num_groups; j += blockDim.x) {
      const int s0 = a.grp_start[j], s1 = a.grp_start[j + 1], nb = a.grp_blocks[j];
      ok = ok && 0 <= s0 && s0 <= s1 && s1 <= n && 0 <= nb && nb <= a.max_blocks_per_seq;
    }
  }
  const bool all_ok = __syncthreads_and(ok) != 0;
  if (!a.pre_rec) return;
  if (!all_ok) {
    if (threadIdx.x == 0 && blockIdx.x == 0) raise_error(a.err, PA_DEVERR_PREFIX);
    return;
  }
  for (int j = threadIdx.x; j < a.num_groups; j += blockDim.x) {
    const int s0 = a.grp_start[j], s1 = a.grp_start[j + 1], nb = a.grp_blocks[j];
    for (int s = s0; s < s1; ++s) b.pre[s] = nb;
  }
  __syncthreads();
}

// Called by every thread of the CTA; ends with __syncthreads().  prefix[s]
// counts items (BAL = false) or KV blocks per KV head (BAL = true) of the
// sequences before s.
template <bool BAL = false>
__device__ __forceinline__ void scan_batch(const AttnArgs &a, const BatchSmem &b, int n) {
  scan_groups(a, b, n);
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
    local += BAL ? unit_blocks(a, L, q1 - q0, b.pre[s]) : seq_items(a, L, q1 - q0);
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
    run += BAL ? unit_blocks(a, b.len[s], b.ql[s], b.pre[s]) : seq_items(a, b.len[s], b.ql[s]);
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
  it.boff = 0;
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

// ---------------------------------------------------------------------------
// Balanced partition.  The work of the launch is the concatenation, over
// decode sequences s and then KV heads, of each (s, kvh) pair's units:
// item_units leading units that stand for the pair's fixed cost, then one
// unit per KV block; W = sum_s units(s) * Hk.  CTA i of G takes the flat
// range [i*W/G, (i+1)*W/G), so every CTA carries the same cost (+-1 unit)
// whatever the length mix; a CTA whose piece of a pair holds leading units
// only has nothing to do for it.  A pair wholly inside one CTA's range is finished
// there (written to `out`); a pair cut by range boundaries leaves one partial
// (m, l, acc) record per covering CTA -- a CTA cuts at most its first and its
// last segment -- and balanced_reduce_kernel merges them.
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ int64_t bal_start(int i, int64_t W, int G) {
  return (int64_t)i * W / G;
}

// Largest i with bal_start(i) <= pos (pos < W).
__device__ __forceinline__ int bal_owner(int64_t pos, int64_t W, int G) {
  int i = (int)(pos * G / W);
  if (i >= G) i = G - 1;
  while (i + 1 < G && bal_start(i + 1, W, G) <= pos) ++i;
  while (i > 0 && bal_start(i, W, G) > pos) --i;
  return i;
}

// Output of a segment: direct to `out`, a fixed-split partial (index = split)
// or a balanced-partition record (index = 0 first / 1 last segment of the CTA).
enum SegOut { kOutDirect = 0, kOutSplit = 1, kOutRecord = 2 };

struct Seg {
  Item it;      // seq, qrow, kvh, b0, b1, L, bad_bits (+ split for kOutSplit)
  int out;      // SegOut
  int index;
};

// Iterates the segments of this CTA in either scheme; producer and consumer
// warps call it in lock step and see the same sequence.
struct SegIter {
  int w;             // fixed scheme: next item
  int64_t pos, end;  // balanced scheme: flat block range still to do
  bool first;
  int s;             // balanced scheme: sequence holding pos (-1 before the first)
  __device__ void init(const AttnArgs &a, const BatchSmem &b, int n) {
    w = blockIdx.x;
    s = -1;
    if (a.balanced) {
      const int64_t W = (int64_t)b.prefix[n] * a.num_kv_heads;
      pos = bal_start(blockIdx.x, W, gridDim.x);
      end = bal_start(blockIdx.x + 1, W, gridDim.x);
      first = true;
    }
  }
  __device__ bool next(const AttnArgs &a, const BatchSmem &b, int n, Seg *seg) {
    if (!a.balanced) {
      if (w >= b.prefix[n] * a.num_kv_heads) return false;
      seg->it = decode_item(a, b, n, w);
      seg->out = seg->it.nsplit == 1 ? kOutDirect : kOutSplit;
      seg->index = seg->it.split;
      w += gridDim.x;
      return true;
    }
    while (pos < end) {
      // sequence holding flat position pos: prefix[lo]*Hk <= pos < prefix[lo+1]*Hk.
      // A binary search for the first segment; after that pos only grows, so
      // the sequence is the current one or a later one (usually the next).
      const int Hk = a.num_kv_heads;
      int lo = 0;
      if (s < 0) {
        int hi = n;
        while (hi - lo > 1) {
          const int mid = (lo + hi) >> 1;
          if ((int64_t)b.prefix[mid] * Hk <= pos) lo = mid; else hi = mid;
        }
      } else {
        lo = s;
        while (lo + 1 < n && (int64_t)b.prefix[lo + 1] * Hk <= pos) ++lo;
      }
      s = lo;
      const int nu = b.prefix[lo + 1] - b.prefix[lo];  // units per KV head (> 0 here)
      const int nb = nu - a.item_units;                // KV blocks per KV head
      const int off = (int)(pos - (int64_t)b.prefix[lo] * Hk);  // < nu * Hk
      const int kvh = off / nu;
      const int u0 = off - kvh * nu;
      const int64_t left = end - pos;
      const int u1 = left < nu - u0 ? u0 + (int)left : nu;
      pos += u1 - u0;
      const int b0 = max(0, u0 - a.item_units), b1 = max(0, u1 - a.item_units);
      if (b1 == b0) continue;  // leading units only
      Item &it = seg->it;
      it.seq = a.seq_begin + lo;
      it.qrow = b.q0[lo];
      it.split = 0;
      it.nsplit = 1;
      it.kvh = kvh;
      it.b0 = b0;
      it.b1 = b1;
      it.boff = b.pre[lo];
      it.L = b.len[lo] - it.boff * a.block_size;
      it.bad_bits = 0;
      const bool complete = b0 == 0 && b1 == nb;
      seg->out = complete ? kOutDirect : kOutRecord;
      seg->index = first ? 0 : 1;
      first = false;
      return true;
    }
    return false;
  }
};

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

// Merge one partial softmax result (accumulator slice x, running max m in
// base 2, running sum l; l = NaN marks a poisoned record) into (M, Lsum, o).
__device__ __forceinline__ void fold_record(float4 x, float m, float l, float *M,
                                            float *Lsum, float4 *o, bool *bad) {
  if (isnan(l)) {
    *bad = true;
    return;
  }
  const float Mn = fmaxf(*M, m);
  if (Mn == -INFINITY) return;
  const float sa = *M == -INFINITY ? 0.f : fast_exp2(*M - Mn);
  const float sb = m == -INFINITY ? 0.f : fast_exp2(m - Mn);
  o->x = o->x * sa + x.x * sb;
  o->y = o->y * sa + x.y * sb;
  o->z = o->z * sa + x.z * sb;
  o->w = o->w * sa + x.w * sb;
  *Lsum = *Lsum * sa + l * sb;
  *M = Mn;
}

// Merge area written by the consumer warps at the end of an item: warp w, its
// head h (of `gw` heads per warp) at merge + w*mstride + h*(D+4):
//   [0, D) unnormalised accumulator, [D] running max (base 2), [D+1] running
//   sum, [D+2] nonzero if the item saw a bad block.
// Warp w = bl*hsplit + hs handled heads hs*gw .. hs*gw+gw-1 of the group for
// the blocks j = bl (mod nbl).  All consumer threads (ncw*32) call this;
// direct items go to `out`, split items to the workspace.
// The prefix kernel's partial (o, m, l) of head hg of a shared-prefix item,
// read from the workspace.
struct PreFromGlobal {
  const float *rec;  // the item's first group head: [group heads][D + 4]
  int D;
  __device__ __forceinline__ void operator()(int hg, int d4, float4 *x, float *m, float *l) const {
    const float *r = rec + hg * (D + 4);
    *x = *reinterpret_cast<const float4 *>(r + d4 * 4);
    *m = r[D];
    *l = r[D + 1];
  }
};

// `pre` gives the prefix partial of a direct item of a shared-prefix
// sequence (item.boff > 0), which is folded in before the store.
template <typename T, int D, typename Pre>
__device__ __forceinline__ void merge_store(const AttnArgs &a, const Seg &seg,
                                            const float *merge, int mstride, int gw,
                                            int hsplit, int nbl, int ncw, int tid, const Pre &pre) {
  const Item &item = seg.it;
  constexpr int D4 = D / 4;
  const int total4 = a.group * D4;
  const bool fold = seg.out == kOutDirect && item.boff > 0;
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
      const float4 y = *reinterpret_cast<const float4 *>(src + d4 * 4);
      o.x += wgt * y.x;
      o.y += wgt * y.y;
      o.z += wgt * y.z;
      o.w += wgt * y.w;
    }
    const int head = item.kvh * a.group + hg;
    if (fold) {  // the sequence's shared prefix: fold in the prefix kernel's partial
      float4 x;
      float xm, xl;
      pre(hg, d4, &x, &xm, &xl);
      fold_record(x, xm, xl, &M, &Lsum, &o, &anybad);
    }
    if (seg.out == kOutDirect) {
      const float inv = (Lsum > 0.f && !anybad) ? 1.f / Lsum : 0.f;
      T *dst = static_cast<T *>(a.out) + ((int64_t)item.qrow * a.num_heads + head) * D + d4 * 4;
      store4<T>(dst, make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv));
    } else {
      float *po, *pml;
      if (seg.out == kOutSplit) {
        const int64_t pidx = ((int64_t)item.seq * a.num_heads + head) * a.max_splits + seg.index;
        po = a.part_o + pidx * D;
        pml = a.part_ml + 2 * pidx;
      } else {  // record of this CTA: [cta][slot][group head][D + 4] (16-byte rows)
        const int64_t ridx = ((int64_t)blockIdx.x * 2 + seg.index) * a.group + hg;
        po = a.part_o + ridx * (D + 4);
        pml = po + D;
      }
      *reinterpret_cast<float4 *>(po + d4 * 4) = o;
      if (d4 == 0) {
        pml[0] = M;
        pml[1] = anybad ? __int_as_float(0x7fc00000) : Lsum;
      }
    }
  }
}

template <typename T, int D>
__device__ __forceinline__ void merge_store(const AttnArgs &a, const Seg &seg,
                                            const float *merge, int mstride, int gw,
                                            int hsplit, int nbl, int ncw, int tid) {
  const PreFromGlobal pre{
      a.pre_rec + ((int64_t)seg.it.seq * a.num_heads + seg.it.kvh * a.group) * (D + 4), D};
  merge_store<T, D>(a, seg, merge, mstride, gw, hsplit, nbl, ncw, tid, pre);
}

}  // namespace dec
}  // namespace pa
