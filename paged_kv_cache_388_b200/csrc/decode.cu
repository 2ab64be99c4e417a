// decode.cu -- paged decode attention (one query token per sequence) for B200.
//
// Work decomposition
//   A work item is (sequence, KV head, split): the GROUP query heads that read
//   one KV head share every K/V byte loaded for that item (GQA), and long
//   contexts are cut into splits of `split_blocks` KV blocks so that the 148
//   SMs stay busy and the tail is short (sequence split / KV-head group /
//   work queue, "PagedAttention 实战", section 2026 年的新变化).  The kernel is
//   persistent: each CTA scans context_lens once, builds the prefix sum of
//   per-sequence split counts in shared memory and then walks items
//   blockIdx.x, blockIdx.x + gridDim.x, ... (dense enumeration, so CTAs get
//   item counts within one of each other).
//
// Data movement (the whole cost of decode: "PagedAttention 实战", section
// 先理解 KV Cache, Decode is memory-bound)
//   One producer warp walks the block table of each item and, for every KV
//   block, issues two bulk asynchronous copies (TMA, non-tensor form) of the
//   contiguous (block, kv-head) K and V tiles -- block_size*head_dim elements
//   each -- into a ring of shared-memory stages guarded by full/empty
//   mbarriers.  The block table is read 32 entries at a time with one
//   coalesced load.
//
// Math (fp32 on the CUDA cores; decode is not a dense contraction)
//   Consumer warps take whole KV blocks round-robin; warps that share a block
//   (group > 4) split the query heads between them.  Within a warp a lane
//   owns one 16-byte slice of a K/V row: q.K partial dot products are formed
//   with packed fp32x2 FMAs, combined with a butterfly reduce-scatter across
//   the lanes of a row, and fed to an online softmax in base 2 (scale*log2 e
//   folded into q).  P.V accumulates into per-lane fp32 registers.  At the end
//   of an item the warps' (m, l, acc) states are merged through shared memory
//   and either written to `out` (single split) or to the split workspace,
//   which reduce_kernel combines.
#include <float.h>
#include <stdlib.h>
#include <string.h>

#include "decode_common.cuh"

namespace pa {
namespace {

using namespace dec;

// Tunables (compile-time): ring of K/V stages per CTA and the CTAs per SM the
// 4-consumer-warp variant is register-limited to.
#ifndef PA_DECODE_RING_KB
#define PA_DECODE_RING_KB 48
#endif
#ifndef PA_DECODE_MIN_CTAS
#define PA_DECODE_MIN_CTAS 3
#endif

constexpr int kMaxSeqsPerLaunch = 2048;
constexpr int kRingBytes = PA_DECODE_RING_KB * 1024;

template <typename T, int D, int BS, int GW>
struct DecodeCfg {
  static constexpr int kElem = sizeof(T);
  static constexpr int ELEMS = 16 / kElem;      // elements per 16-byte vector
  static constexpr int PAIRS = ELEMS / 2;
  static constexpr int LPR = D / ELEMS;         // lanes per K/V row
  static constexpr int RPP = 32 / LPR;          // rows per pass (row groups per warp)
  static constexpr int CHUNK = 16;              // rows per softmax step
  static constexpr int PASSES = CHUNK / RPP;
  // Scores are reduced in sub-chunks of PPS passes so that a sub-chunk holds at
  // most LPR partial sums per lane (registers) and leaves one reduced score per
  // lane (DUP lanes share it when a sub-chunk has fewer scores than lanes).
  static constexpr int PPS = PASSES * GW >= LPR ? LPR / GW : PASSES;  // passes per sub-chunk
  static constexpr int NSUB = PASSES / PPS;     // sub-chunks per chunk = scores kept per lane
  static constexpr int NVS = PPS * GW;          // partial scores per lane per sub-chunk
  static constexpr int DUP = LPR / NVS;         // lanes holding the same reduced score
  static constexpr int LPH = LPR / GW;          // lanes of one head in a row group
  static constexpr int TILE = BS * D * kElem;   // bytes of one (block, kv-head) tile
  static constexpr int STAGE = 2 * TILE;        // K tile + V tile
  static constexpr int STAGES = kRingBytes / STAGE < 2 ? 2 : kRingBytes / STAGE;
  static_assert(LPR >= 1 && LPR <= 32 && (32 % LPR) == 0, "row must map onto whole lanes");
  static_assert(PASSES >= 1 && CHUNK % RPP == 0, "chunk must hold whole passes");
  static_assert(GW <= LPR, "a lane's reduced scores must belong to one head");
  static_assert(NVS <= LPR && LPR % NVS == 0 && PASSES % PPS == 0, "sub-chunk shape");
  static_assert(BS % CHUNK == 0, "block size must be a multiple of 16");
};

// Dynamic shared-memory layout; depends on the launch (sequences in this
// launch, consumer warps, group size), computed identically on host and device.
template <typename C>
struct Layout {
  int ring, qbuf, full, empty, qfull, qempty, bad, misc, batch, p, merge, bytes;
  int qbytes;  // bytes of one item's query rows (GROUP heads)
  __host__ __device__ Layout(int n, int ncw, int group) {
    constexpr int D = C::LPR * C::ELEMS;
    qbytes = group * D * C::kElem;
    ring = 0;
    qbuf = ring + C::STAGES * C::STAGE;
    full = align_up(qbuf + 2 * qbytes, 128);
    empty = full + 8 * C::STAGES;
    qfull = empty + 8 * C::STAGES;
    qempty = qfull + 16;
    bad = qempty + 16;
    misc = align_up(bad + 4 * C::STAGES, 16);
    batch = misc + 16;
    p = align_up(batch + BatchSmem::bytes(n), 128);
    merge = align_up(p + ncw * 16 * 4 * 4, 128);
    bytes = merge + ncw * 4 * (D + 4) * 4;
  }
};

template <int NV, int LPR>
__device__ __forceinline__ void reduce_scatter(float (&v)[NV], int lane) {
  int cnt = NV;
#pragma unroll
  for (int m = LPR / 2; m >= 1; m >>= 1) {
    if (cnt > 1) {
      const int half = cnt / 2;
      const bool up = (lane & m) != 0;
#pragma unroll
      for (int i = 0; i < NV / 2; ++i) {
        if (i < half) {
          const float send = up ? v[i] : v[i + half];
          const float keep = up ? v[i + half] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
      }
      cnt = half;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
    }
  }
}

// MAXW = most consumer warps a launch of this variant uses (4: three CTAs per
// SM fit; 8: the wide variant for large head groups).
template <typename T, int D, int BS, int GW, int MAXW>
__global__ void __launch_bounds__(32 * (MAXW + 1), MAXW == 4 ? PA_DECODE_MIN_CTAS : 1)
    paged_decode_kernel(const AttnArgs a, int ncw, int hsplit) {
  using C = DecodeCfg<T, D, BS, GW>;
  extern __shared__ __align__(128) unsigned char smem[];
  const int n = a.num_seqs;
  const Layout<C> lay(n, ncw, a.group);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + lay.full);
  uint64_t *empty = reinterpret_cast<uint64_t *>(smem + lay.empty);
  uint64_t *qfull = reinterpret_cast<uint64_t *>(smem + lay.qfull);
  uint64_t *qempty = reinterpret_cast<uint64_t *>(smem + lay.qempty);
  int *bad = reinterpret_cast<int *>(smem + lay.bad);
  volatile int *abort_flag = reinterpret_cast<int *>(smem + lay.misc);
  BatchSmem bsm;
  bsm.carve(smem + lay.batch, n);
  unsigned char *ring = smem + lay.ring;
  unsigned char *qbuf = smem + lay.qbuf;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // ---- prologue: barriers, per-sequence lengths and rows, item prefix sum --
  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], ncw);  // every consumer warp releases every stage
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&qfull[s], 1);
      mbar_init(&qempty[s], ncw);
    }
    *abort_flag = 0;
    mbar_init_fence();
  }
  scan_batch(a, bsm, n);
  const int total_items = bsm.prefix[n] * a.num_kv_heads;

  if (warp == ncw) {
    // ======================= producer warp ===================================
    uint32_t it = 0, k = 0;
    for (int w = blockIdx.x; w < total_items; w += gridDim.x, ++k) {
      const Item item = decode_item(a, bsm, n, w);
      // this item's query rows -> qbuf[k & 1]
      {
        const uint32_t qs = k & 1u;
        bool ok = !*abort_flag;
        if (ok) ok = mbar_wait(&qempty[qs], ((k >> 1) & 1u) ^ 1u);
        if (lane == 0) {
          if (!ok) {
            if (!*abort_flag) raise_error(a.err, PA_DEVERR_TIMEOUT);
            *abort_flag = 1;
            mbar_arrive(&qfull[qs]);
          } else {
            mbar_arrive_expect_tx(&qfull[qs], lay.qbytes);
            bulk_load(qbuf + qs * lay.qbytes,
                      static_cast<const T *>(a.q) +
                          ((int64_t)item.qrow * a.num_heads + item.kvh * a.group) * D,
                      lay.qbytes, &qfull[qs]);
          }
        }
        __syncwarp();
      }
      const int32_t *table = a.block_tables + (int64_t)item.seq * a.max_blocks_per_seq;
      for (int b = item.b0; b < item.b1; b += 32) {
        const int cnt = min(32, item.b1 - b);
        const int my_id = lane < cnt ? table[b + lane] : 0;
        for (int j = 0; j < cnt; ++j) {
          const int pb = __shfl_sync(0xffffffffu, my_id, j);
          const uint32_t slot = it % C::STAGES;
          const uint32_t par = ((it / C::STAGES) & 1u) ^ 1u;
          ++it;
          bool ok = !*abort_flag;
          if (ok) ok = mbar_wait(&empty[slot], par);
          if (lane == 0) {
            if (!ok) {
              if (!*abort_flag) raise_error(a.err, PA_DEVERR_TIMEOUT);
              *abort_flag = 1;
              bad[slot] = 1;
              mbar_arrive(&full[slot]);
            } else if (pb < 0 || pb >= a.num_blocks) {
              raise_error(a.err, PA_DEVERR_BLOCK_ID);
              bad[slot] = 1;
              mbar_arrive(&full[slot]);
            } else {
              bad[slot] = 0;
              const int64_t tile = ((int64_t)pb * a.num_kv_heads + item.kvh) * (BS * D);
              unsigned char *dst = ring + slot * C::STAGE;
              mbar_arrive_expect_tx(&full[slot], C::STAGE);
              bulk_load(dst, static_cast<const T *>(a.k_cache) + tile, C::TILE, &full[slot]);
              bulk_load(dst + C::TILE, static_cast<const T *>(a.v_cache) + tile, C::TILE,
                        &full[slot]);
            }
          }
          __syncwarp();
        }
      }
    }
    // the copies this warp started land before the CTA may exit
    if (lane == 0 && !(drain_ring(full, C::STAGES, it) & drain_ring(qfull, 2, k))) {
      if (!*abort_flag) raise_error(a.err, PA_DEVERR_TIMEOUT);
      *abort_flag = 1;
    }
    return;
  }

  // ======================= consumer warps ==================================
  const int hs = warp % hsplit;   // which GW-head subset of the group
  const int bl = warp / hsplit;   // block lane: blocks bl, bl+nbl, ...
  const int nbl = ncw / hsplit;
  const int rg = lane / C::LPR;   // row group
  const int li = lane % C::LPR;   // lane within row
  // reduced-score ownership of this lane (see reduce_scatter): in every
  // sub-chunk the lane keeps score v = li / DUP, i.e. head v / PPS of pass
  // v % PPS of that sub-chunk.
  const int vsub = li / C::DUP;
  const int my_head = vsub / C::PPS;
  const int my_pass = vsub % C::PPS;
  const bool owner = (li % C::DUP) == 0;

  float *p_s = reinterpret_cast<float *>(smem + lay.p) + warp * 16 * GW;
  float *merge = reinterpret_cast<float *>(smem + lay.merge);
  const int mstride = GW * (D + 4);  // floats per warp in the merge area

  uint32_t it_base = 0, k = 0;
  for (int w = blockIdx.x; w < total_items; w += gridDim.x, ++k) {
    const Item item = decode_item(a, bsm, n, w);
    const int nblocks = item.b1 - item.b0;

    // q slice of this lane from the prefetched rows, pre-scaled by scale*log2(e)
    float2 q2[GW][C::PAIRS];
    {
      const uint32_t qs = k & 1u;
      bool ok = !*abort_flag;
      if (ok) {
        ok = mbar_wait(&qfull[qs], (k >> 1) & 1u);
        if (!ok && lane == 0) {
          if (!*abort_flag) raise_error(a.err, PA_DEVERR_TIMEOUT);
          *abort_flag = 1;
        }
      }
      const T *qrow = reinterpret_cast<const T *>(qbuf + qs * lay.qbytes) + hs * GW * D;
#pragma unroll
      for (int h = 0; h < GW; ++h) {
        const uint4 raw = *reinterpret_cast<const uint4 *>(qrow + h * D + li * C::ELEMS);
        Elem<T>::to_f2(raw, q2[h]);
#pragma unroll
        for (int e = 0; e < C::PAIRS; ++e) {
          q2[h][e].x *= a.scale_log2;
          q2[h][e].y *= a.scale_log2;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&qempty[qs]);
    }

    float m[GW];
    float2 acc[GW][C::PAIRS];
#pragma unroll
    for (int h = 0; h < GW; ++h) {
      m[h] = -INFINITY;
#pragma unroll
      for (int e = 0; e < C::PAIRS; ++e) acc[h][e] = make_float2(0.f, 0.f);
    }
    float l_lane = 0.f;
    bool item_bad = item.bad_bits != 0;
    if (item.bad_bits && tid == 0 && item.kvh == 0) raise_error(a.err, item.bad_bits);

    // Every consumer warp waits for and releases every stage in ring order
    // (so no parity wait is ever more than one phase ahead of its barrier),
    // but computes only the blocks j = bl, bl + nbl, ... of this item.
    auto wait_stage = [&](uint32_t itn) -> bool {
      const uint32_t slot = itn % C::STAGES;
      bool ok = !*abort_flag;
      if (ok) {
        ok = mbar_wait(&full[slot], (itn / C::STAGES) & 1u);
        if (!ok && lane == 0) {
          if (!*abort_flag) raise_error(a.err, PA_DEVERR_TIMEOUT);
          *abort_flag = 1;
        }
      }
      return ok && !bad[slot];
    };
    auto release_stage = [&](uint32_t itn) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[itn % C::STAGES]);
    };
    int next = 0;  // first block of the item not yet waited for by this warp
    for (int j = bl; j < nblocks; j += nbl) {
      for (; next < j; ++next) {
        wait_stage(it_base + next);
        release_stage(it_base + next);
      }
      next = j + 1;
      const uint32_t itn = it_base + j;
      const uint32_t slot = itn % C::STAGES;
      const bool ok = wait_stage(itn);
      if (!ok) {
        item_bad = true;
      } else {
        const int b = item.b0 + j;
        const int nvalid = min(BS, item.L - b * BS);
        const unsigned char *ks = ring + slot * C::STAGE;
        const unsigned char *vs = ks + C::TILE;
#pragma unroll
        for (int r0 = 0; r0 < BS; r0 += C::CHUNK) {
          if (r0 < nvalid) {
            // ---- scores: partial dot products over this lane's slice, reduced
            //      across the row's lanes one sub-chunk at a time ----
            float sc[C::NSUB];
#pragma unroll
            for (int u = 0; u < C::NSUB; ++u) {
              float part[C::NVS];
#pragma unroll
              for (int pp = 0; pp < C::PPS; ++pp) {
                const int row = r0 + (u * C::PPS + pp) * C::RPP + rg;
                const uint4 raw =
                    *reinterpret_cast<const uint4 *>(ks + (row * D + li * C::ELEMS) * C::kElem);
                float2 k2[C::PAIRS];
                Elem<T>::to_f2(raw, k2);
#pragma unroll
                for (int h = 0; h < GW; ++h) {
                  float2 d2 = make_float2(0.f, 0.f);
#pragma unroll
                  for (int e = 0; e < C::PAIRS; ++e) d2 = ffma2(q2[h][e], k2[e], d2);
                  part[h * C::PPS + pp] = d2.x + d2.y;
                }
              }
              reduce_scatter<C::NVS, C::LPR>(part, lane);
              sc[u] = part[0];
            }

            // ---- online softmax (base 2) ----
            float cmax = -INFINITY;
#pragma unroll
            for (int u = 0; u < C::NSUB; ++u) {
              const int row = r0 + (u * C::PPS + my_pass) * C::RPP + rg;
              if (row >= nvalid) sc[u] = -INFINITY;
              cmax = fmaxf(cmax, sc[u]);
            }
#pragma unroll
            for (int o = C::DUP; o < C::LPH; o <<= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
#pragma unroll
            for (int o = C::LPR; o < 32; o <<= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
            float alpha[GW];
            float m_mine = 0.f, a_mine = 1.f;
#pragma unroll
            for (int h = 0; h < GW; ++h) {
              const float cm = __shfl_sync(0xffffffffu, cmax, h * C::LPH);
              const float mn = fmaxf(m[h], cm);
              alpha[h] = fast_exp2(m[h] - mn);
              m[h] = mn;
              if (h == my_head) {
                m_mine = mn;
                a_mine = alpha[h];
              }
            }
            float psum = 0.f;
#pragma unroll
            for (int u = 0; u < C::NSUB; ++u) {
              const float pv = fast_exp2(sc[u] - m_mine);
              psum += pv;
              const int crow = (u * C::PPS + my_pass) * C::RPP + rg;  // row within chunk
              if (owner) p_s[crow * GW + my_head] = pv;
            }
            l_lane = l_lane * a_mine + (owner ? psum : 0.f);
            __syncwarp();

            // ---- rescale and accumulate P.V ----
#pragma unroll
            for (int h = 0; h < GW; ++h) {
              const float2 a2 = make_float2(alpha[h], alpha[h]);
#pragma unroll
              for (int e = 0; e < C::PAIRS; ++e) acc[h][e] = __fmul2_rn(acc[h][e], a2);
            }
#pragma unroll
            for (int p = 0; p < C::PASSES; ++p) {
              const int crow = p * C::RPP + rg;
              const int row = r0 + crow;
              const uint4 raw =
                  *reinterpret_cast<const uint4 *>(vs + (row * D + li * C::ELEMS) * C::kElem);
              float2 v2[C::PAIRS];
              Elem<T>::to_f2(raw, v2);
              if (row >= nvalid) {
#pragma unroll
                for (int e = 0; e < C::PAIRS; ++e) v2[e] = make_float2(0.f, 0.f);
              }
              float pr[GW];
              if constexpr (GW == 4) {
                const float4 t = *reinterpret_cast<const float4 *>(p_s + crow * 4);
                pr[0] = t.x; pr[1] = t.y; pr[2] = t.z; pr[3] = t.w;
              } else if constexpr (GW == 2) {
                const float2 t = *reinterpret_cast<const float2 *>(p_s + crow * 2);
                pr[0] = t.x; pr[1] = t.y;
              } else {
                pr[0] = p_s[crow];
              }
#pragma unroll
              for (int h = 0; h < GW; ++h) {
                const float2 pp = make_float2(pr[h], pr[h]);
#pragma unroll
                for (int e = 0; e < C::PAIRS; ++e) acc[h][e] = ffma2(pp, v2[e], acc[h][e]);
              }
            }
            __syncwarp();
          }
        }
      }
      release_stage(itn);
    }
    for (; next < nblocks; ++next) {
      wait_stage(it_base + next);
      release_stage(it_base + next);
    }
    it_base += nblocks;

    // ---- per-warp totals: sum acc over row groups, l over the head's lanes ----
#pragma unroll
    for (int o = C::LPR; o < 32; o <<= 1) {
#pragma unroll
      for (int h = 0; h < GW; ++h)
#pragma unroll
        for (int e = 0; e < C::PAIRS; ++e) {
          acc[h][e].x += __shfl_xor_sync(0xffffffffu, acc[h][e].x, o);
          acc[h][e].y += __shfl_xor_sync(0xffffffffu, acc[h][e].y, o);
        }
    }
#pragma unroll
    for (int o = 1; o < C::LPH; o <<= 1) l_lane += __shfl_xor_sync(0xffffffffu, l_lane, o);
#pragma unroll
    for (int o = C::LPR; o < 32; o <<= 1) l_lane += __shfl_xor_sync(0xffffffffu, l_lane, o);

    float *mw = merge + warp * mstride;
    if (rg == 0) {
#pragma unroll
      for (int h = 0; h < GW; ++h) {
        float4 *dst = reinterpret_cast<float4 *>(mw + h * (D + 4) + li * C::ELEMS);
#pragma unroll
        for (int e = 0; e < C::PAIRS; e += 2)
          dst[e / 2] = make_float4(acc[h][e].x, acc[h][e].y, acc[h][e + 1].x, acc[h][e + 1].y);
      }
    }
#pragma unroll
    for (int h = 0; h < GW; ++h) {
      const float lh = __shfl_sync(0xffffffffu, l_lane, h * C::LPH);
      if (lane == 0) {
        mw[h * (D + 4) + D] = m[h];
        mw[h * (D + 4) + D + 1] = lh;
        mw[h * (D + 4) + D + 2] = item_bad ? 1.f : 0.f;
      }
    }
    named_sync(1, ncw * 32);

    // ---- merge the warps that worked on the same heads; write out ----------
    {
      Seg seg;
      seg.it = item;
      seg.out = item.nsplit == 1 ? kOutDirect : kOutSplit;
      seg.index = item.split;
      merge_store<T, D>(a, seg, merge, mstride, GW, hsplit, nbl, ncw, tid);
    }
    named_sync(1, ncw * 32);
  }
}

// Combine split partials: one warp per (sequence, head).
template <typename T, int D>
__global__ void __launch_bounds__(256) reduce_kernel(const AttnArgs a) {
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= a.num_seqs * a.num_heads) return;
  const int s = gw / a.num_heads;
  const int head = gw - s * a.num_heads;
  const int gs = a.seq_begin + s;
  int qrow = gs, qlen = 1;
  if (a.query_start_loc) {
    qrow = a.query_start_loc[gs];
    qlen = a.query_start_loc[gs + 1] - qrow;
    if (qrow < 0 || qlen != 1 || qrow + 1 > a.num_q_tokens) return;
  }
  const int L = a.context_lens[gs];
  if (L <= 0 || L > a.max_context_len) return;  // written by the main kernel
  const int nsplit = ceil_div(ceil_div(L, a.block_size), a.split_blocks);
  if (nsplit <= 1 || nsplit > a.max_splits) return;
  const int64_t base = ((int64_t)gs * a.num_heads + head) * a.max_splits;

  float M = -INFINITY;
  bool poisoned = false;
  for (int sp = lane; sp < nsplit; sp += 32) {
    M = fmaxf(M, a.part_ml[2 * (base + sp)]);
    poisoned |= isnan(a.part_ml[2 * (base + sp) + 1]);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  poisoned = __any_sync(0xffffffffu, poisoned);

  constexpr int PER = D / 32;  // elements per lane
  float o[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) o[e] = 0.f;
  float Lsum = 0.f;
  for (int sp = 0; sp < nsplit; ++sp) {
    const float ms = a.part_ml[2 * (base + sp)];
    const float wgt = ms == -INFINITY ? 0.f : fast_exp2(ms - M);
    Lsum += wgt * a.part_ml[2 * (base + sp) + 1];
    const float *src = a.part_o + (base + sp) * D + lane * PER;
    if constexpr (PER == 4) {
      const float4 x = *reinterpret_cast<const float4 *>(src);
      o[0] += wgt * x.x; o[1] += wgt * x.y; o[2] += wgt * x.z; o[3] += wgt * x.w;
    } else {
      const float2 x = *reinterpret_cast<const float2 *>(src);
      o[0] += wgt * x.x; o[1] += wgt * x.y;
    }
  }
  const float inv = (Lsum > 0.f && !poisoned) ? 1.f / Lsum : 0.f;
  T *dst = static_cast<T *>(a.out) + ((int64_t)qrow * a.num_heads + head) * D + lane * PER;
#pragma unroll
  for (int e = 0; e < PER; ++e) dst[e] = Elem<T>::from_f(o[e] * inv);
}

template <typename T, int D, int BS, int GW, int MAXW>
cudaError_t launch_variant(const AttnArgs &a, int sm_count, int ncw, int hsplit,
                           cudaStream_t stream) {
  using C = DecodeCfg<T, D, BS, GW>;
  auto kern = paged_decode_kernel<T, D, BS, GW, MAXW>;
  const Layout<C> lay(a.num_seqs, ncw, a.group);
  // Opt in to the largest layout once; resident CTAs per SM for this launch.
  const Layout<C> big(kMaxSeqsPerLaunch, MAXW, 32);
  cudaError_t e = set_smem_limit_once(reinterpret_cast<const void *>(kern), big.bytes);
  if (e != cudaSuccess) return e;
  int occ = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, 32 * (ncw + 1),
                                                                lay.bytes);
  if (e != cudaSuccess) return e;
  if (occ < 1) occ = 1;
  const int64_t max_items = (int64_t)a.num_seqs * a.num_kv_heads *
                            (a.rows_mode ? (a.max_splits > a.max_query_len ? a.max_splits : a.max_query_len)
                                         : a.max_splits);
  int64_t grid = (int64_t)sm_count * occ;
  if (grid > max_items) grid = max_items;
  if (grid < 1) grid = 1;
  kern<<<(unsigned)grid, 32 * (ncw + 1), lay.bytes, stream>>>(a, ncw, hsplit);
  return cudaGetLastError();
}

template <typename T, int D, int BS, int GW>
cudaError_t launch_decode_t(const AttnArgs &a, int sm_count, cudaStream_t stream) {
  const int hsplit = a.group / GW;
  const int nbl = hsplit >= 4 ? 1 : 4 / hsplit;
  const int ncw = hsplit * nbl;
  if (ncw <= 4) return launch_variant<T, D, BS, GW, 4>(a, sm_count, ncw, hsplit, stream);
  return launch_variant<T, D, BS, GW, 8>(a, sm_count, ncw, hsplit, stream);
}

template <typename T, int D, int BS>
cudaError_t dispatch_gw(const AttnArgs &a, int sm_count, cudaStream_t s) {
  if (a.group % 4 == 0) return launch_decode_t<T, D, BS, 4>(a, sm_count, s);
  if (a.group % 2 == 0) return launch_decode_t<T, D, BS, 2>(a, sm_count, s);
  return launch_decode_t<T, D, BS, 1>(a, sm_count, s);
}

template <typename T, int D>
cudaError_t dispatch_bs(const AttnArgs &a, int sm_count, cudaStream_t s) {
  return a.block_size == 16 ? dispatch_gw<T, D, 16>(a, sm_count, s)
                            : dispatch_gw<T, D, 32>(a, sm_count, s);
}

template <typename T>
cudaError_t dispatch_d(const AttnArgs &a, int sm_count, cudaStream_t s) {
  return a.head_dim == 64 ? dispatch_bs<T, 64>(a, sm_count, s) : dispatch_bs<T, 128>(a, sm_count, s);
}

template <typename T>
cudaError_t launch_reduce_t(const AttnArgs &a, cudaStream_t stream) {
  const int64_t warps = (int64_t)a.num_seqs * a.num_heads;
  const int64_t blocks = (warps * 32 + 255) / 256;
  if (a.head_dim == 64)
    reduce_kernel<T, 64><<<(unsigned)blocks, 256, 0, stream>>>(a);
  else
    reduce_kernel<T, 128><<<(unsigned)blocks, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

int decode_max_seqs_per_launch() { return kMaxSeqsPerLaunch; }

cudaError_t launch_decode(const AttnArgs &a, int dtype, int sm_count, cudaStream_t stream) {
  if (dtype == PA_F32) return dispatch_d<float>(a, sm_count, stream);
  if (dtype == PA_F16) return dispatch_d<__half>(a, sm_count, stream);
  return dispatch_d<__nv_bfloat16>(a, sm_count, stream);
}

cudaError_t launch_reduce(const AttnArgs &a, int dtype, cudaStream_t stream) {
  if (dtype == PA_F32) return launch_reduce_t<float>(a, stream);
  if (dtype == PA_F16) return launch_reduce_t<__half>(a, stream);
  return launch_reduce_t<__nv_bfloat16>(a, stream);
}

}  // namespace pa
