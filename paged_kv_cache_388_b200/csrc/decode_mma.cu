// decode_mma.cu -- paged decode attention on the tensor cores (16-bit caches).
//
// Why tensor cores here: with GQA, the GROUP query heads that share a KV head
// all read every K/V element of the item, so the per-block products
//     S^T[keys x heads] = K[keys x D] . Q^T[D x heads]
//     O^T[D x heads]   += V^T[D x keys] . P^T[keys x heads]
// are dense contractions of the loaded tile with a GROUP-wide operand.  Done
// on the CUDA cores they cost ~1000 instructions per 16-key block (fp32 FMAs,
// bf16 widening, cross-lane reductions) and the kernel is issue-bound well
// below HBM speed; as mma.sync m16n8k16 (keys / head dims on M, the group's
// heads on N) they take 24 MMAs and 16 ldmatrix per block and leave the
// kernel bound by HBM, which is what decode is ("PagedAttention 实战",
// section 先理解 KV Cache, Decode).  The operands are consumed straight from the
// staged cache tiles; nothing is rearranged in memory to form them.
//
// Data movement: one producer warp per CTA walks each item's block table and,
// per KV block, issues tensor-map TMA loads of the (block, kv-head) K and V
// tiles (two 64-column boxes each at head_dim 128) with the 128-byte swizzle,
// so that ldmatrix reads of 8 rows at one column are bank-conflict free.
// Stages live in a shared-memory ring guarded by full/empty mbarriers.
//
// Softmax: online, base 2 (scale*log2 e applied to S in fp32).  P is rounded
// to the cache type for the P.V product; for bf16 (8 significant bits) P is
// split into hi + lo bf16 parts, two products, so P enters exact to ~2^-17.
//
// Work items, the batch scan and the final merge are shared with the
// CUDA-core kernel (decode_common.cuh).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp8.h>

#include <type_traits>

#include "decode_common.cuh"

namespace pa {
namespace {

using namespace dec;

// CTA shape: PA_MMA_WARPS consumer warps + 1 producer, a K/V ring of
// PA_MMA_RING_KB KiB, register budget for PA_MMA_MIN_CTAS resident CTAs per
// SM.  Many small CTAs (2 consumer warps, 3 blocks of 16 tokens in flight
// each, 5 per SM) keep more independent (sequence, KV head) pieces streaming
// per SM than a few large ones: each piece ends with a cross-warp merge and
// starts with a dependent block-table read, and short contexts have many
// pieces.  Measured on B200: decode of 256 x U[1,512]-token sequences 105 ->
// 75 us, the Llama-3-8B-shaped batch 178 -> 172 us against 4 warps / 48 KiB /
// 3 per SM.
#ifndef PA_MMA_RING_KB
#define PA_MMA_RING_KB 24
#endif
#ifndef PA_MMA_MIN_CTAS
#define PA_MMA_MIN_CTAS 5
#endif
#ifndef PA_MMA_WARPS
#define PA_MMA_WARPS 2
#endif

constexpr int kMaxSeqsPerLaunch = 2048;

template <typename T>
struct MmaT;

template <>
struct MmaT<__nv_bfloat16> {
  static constexpr bool kSplitP = true;
  static constexpr CUtensorMapDataType kTmaType = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  __device__ __forceinline__ static void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  __device__ __forceinline__ static uint16_t bits(float x) {
    __nv_bfloat16 h = __float2bfloat16_rn(x);
    return *reinterpret_cast<uint16_t *>(&h);
  }
  __device__ __forceinline__ static float back(uint16_t u) {
    return __uint_as_float(static_cast<uint32_t>(u) << 16);
  }
};

template <>
struct MmaT<__half> {
  static constexpr bool kSplitP = false;
  static constexpr CUtensorMapDataType kTmaType = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  __device__ __forceinline__ static void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  __device__ __forceinline__ static uint16_t bits(float x) {
    __half h = __float2half_rn(x);
    return *reinterpret_cast<uint16_t *>(&h);
  }
  __device__ __forceinline__ static float back(uint16_t u) {
    return __half2float(*reinterpret_cast<__half *>(&u));
  }
};

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

// Transpose of an 8x8 16-bit matrix held as the warp's m8n8 fragment (lane
// 4r + c holds row r, columns 2c and 2c + 1; lower column in the low half).
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
// Four E4M3 codes (byte i = code i) -> two fp16 pairs (exact): lo = codes
// 0, 1 and hi = codes 2, 3, the lower code in the lower half.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t four, uint32_t &lo, uint32_t &hi) {
  asm("{\n\t.reg .b16 l, h;\n\t"
      "mov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(four));
}

// A staged tile is BS rows x D columns of 16-bit values held as D/64 boxes of
// BS rows x 128 bytes, each written by TMA with the 128-byte swizzle: the
// 16-byte chunk c of row r sits at chunk position c ^ (r % 8).  Box bases are
// 1024-byte aligned.  Byte address of the 8-element group (r, c8*8):
template <int BS>
__device__ __forceinline__ uint32_t swz(uint32_t tile, int r, int c8) {
  const int box = c8 >> 3, chunk = c8 & 7;
  return tile + box * (BS * 128) + r * 128 + ((chunk ^ (r & 7)) << 4);
}

// F8: the cache holds FP8 E4M3 codes (1 byte) in the tile layout of
// pa_reshape_and_cache_fp8; consumer warps convert them straight into fp16
// mma fragments.
template <int D, int BS, int NT, int NCW, bool F8 = false>
struct MmaLayout {
  static constexpr int kElem = F8 ? 1 : 2;        // bytes per cached element
  static constexpr int kTile = BS * D * kElem;    // bytes of one (block, kv-head) K or V tile
  static constexpr int kStage = 2 * kTile;
  static constexpr int kStages = (PA_MMA_RING_KB * 1024) / kStage < 2 ? 2 : (PA_MMA_RING_KB * 1024) / kStage;
  int ring, qbuf, full, empty, qfull, qempty, bad, misc, batch, merge, bytes, qbytes;
  // merge area: [warp][group heads][D + 4] floats
  __host__ __device__ MmaLayout(int n, int group) {
    qbytes = group * D * 2;
    ring = 0;  // relative to a 1024-byte aligned base
    qbuf = ring + kStages * kStage;
    full = align_up(qbuf + 2 * qbytes, 128);
    empty = full + 8 * kStages;
    qfull = empty + 8 * kStages;
    qempty = qfull + 16;
    bad = qempty + 16;
    misc = align_up(bad + 4 * kStages, 16);
    batch = misc + 16;
    merge = align_up(batch + BatchSmem::bytes(n), 128);
    bytes = merge + NCW * group * (D + 4) * 4 + 1024;  // + alignment slack
  }
};

// T is the type of q and out.  With F8 the cache holds E4M3 codes and the
// products run in fp16 (Tc): every E4M3 value is exact in fp16, and a bf16 q
// row is scaled by a power of two into fp16 range (the scale is divided out
// of its logits).
template <typename T, int D, int BS, int NT, int NCW, bool F8 = false>
__global__ void __launch_bounds__(32 * (NCW + 1), NT == 1 ? PA_MMA_MIN_CTAS : 2)
    paged_decode_mma_kernel(const AttnArgs a, const __grid_constant__ CUtensorMap tmk,
                            const __grid_constant__ CUtensorMap tmv) {
  using L = MmaLayout<D, BS, NT, NCW, F8>;
  using Tc = typename std::conditional<F8, __half, T>::type;
  // a prefix partial of up to NT * 8 heads must fit the ring at once
  static_assert((NT * 8 * (D + 4) * 4 + L::kStage - 1) / L::kStage <= L::kStages, "ring too small");
  constexpr int KS = D / 16;    // k-steps of the QK product (head dim)
  constexpr int MT = D / 16;    // m-tiles of the PV product (head dim)
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int n = a.num_seqs;
  const L lay(n, a.group);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + lay.full);
  uint64_t *empty = reinterpret_cast<uint64_t *>(smem + lay.empty);
  uint64_t *qfull = reinterpret_cast<uint64_t *>(smem + lay.qfull);
  uint64_t *qempty = reinterpret_cast<uint64_t *>(smem + lay.qempty);
  int *bad = reinterpret_cast<int *>(smem + lay.bad);
  volatile int *abort_flag = reinterpret_cast<int *>(smem + lay.misc);
  BatchSmem bsm;
  bsm.carve(smem + lay.batch, n);
  const uint32_t ring = smem_addr(smem + lay.ring);
  unsigned char *qbuf = smem + lay.qbuf;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NCW);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&qfull[s], 1);
      mbar_init(&qempty[s], NCW);
    }
    *abort_flag = 0;
    mbar_init_fence();
  }
  // Launched as a programmatic dependent of the previous kernel: nothing is
  // read from global memory before that kernel's writes are visible.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // ... and let the merge kernel that follows get scheduled while this runs.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (a.balanced && tid == 0) a.bal_desc[4 * blockIdx.x] = -1;  // no cut pair starts here (yet)
  if (a.balanced) {
    scan_batch<true>(a, bsm, n);
    if (blockIdx.x == 0) {  // block prefix (and shared blocks) for the merge kernel
      for (int s = tid; s <= n; s += blockDim.x) a.bal_prefix[s] = bsm.prefix[s];
      if (a.seq_pre)
        for (int s = tid; s < n; s += blockDim.x) a.seq_pre[s] = bsm.pre[s];
    }
    // Decode sequences with no KV blocks of their own (empty or invalid
    // context, or every key inside the group's shared prefix) own no part of
    // the partition: their rows are written here, from the prefix kernel's
    // partial when all keys are shared, else as zeros.
    if (warp < NCW) {
      for (int s = blockIdx.x; s < n; s += gridDim.x) {
        if (bsm.ql[s] != 1 || bsm.prefix[s + 1] != bsm.prefix[s]) continue;
        const int L = bsm.len[s];
        const int pre = bsm.pre[s];
        const bool valid = L >= 0 && L <= a.max_context_len;
        const bool shared_only = valid && pre > 0 && L >= pre * a.block_size;
        if (tid == 0 && !shared_only && (L != 0 || pre > 0))
          raise_error(a.err, valid && pre > 0 ? PA_DEVERR_PREFIX : PA_DEVERR_CONTEXT_LEN);
        T *row = static_cast<T *>(a.out) + (int64_t)bsm.q0[s] * a.num_heads * D;
        for (int i = tid; i < a.num_heads * D / 4; i += NCW * 32) {
          float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
          if (shared_only) {
            const int h = i / (D / 4), d4 = i - h * (D / 4);
            const float *r = a.pre_rec + ((int64_t)(a.seq_begin + s) * a.num_heads + h) * (D + 4);
            const float l = r[D + 1];
            const float inv = (l > 0.f && !isnan(l)) ? 1.f / l : 0.f;
            const float4 x = *reinterpret_cast<const float4 *>(r + d4 * 4);
            v = make_float4(x.x * inv, x.y * inv, x.z * inv, x.w * inv);
          }
          store4<T>(row + 4 * i, v);
        }
      }
    }
  } else {
    scan_batch<false>(a, bsm, n);
  }

  if (warp == NCW) {
    // ======================= producer warp ===================================
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmk)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmv)) : "memory");
    }
    uint32_t it = 0, k = 0;
    SegIter iter;
    iter.init(a, bsm, n);
    // Block ids are read 32 at a time, one group ahead: the ids of the
    // following group (the rest of this item, else the next item's first) are
    // loaded while the current group's tiles are issued, so that no dependent
    // table read stalls the ring at an item boundary (a balanced CTA can hold
    // a dozen short items).
    Seg seg, nxt;
    bool have = iter.next(a, bsm, n, &seg);
    bool have_nxt = have && iter.next(a, bsm, n, &nxt);
    auto load_ids = [&](const Seg &sg, int b) -> int {
      const int32_t *tb = a.block_tables + (int64_t)sg.it.seq * a.max_blocks_per_seq + sg.it.boff;
      return lane < min(32, sg.it.b1 - b) ? tb[b + lane] : 0;
    };
    int ids = have ? load_ids(seg, seg.it.b0) : 0;
    for (; have; ++k) {
      const Item &item = seg.it;
      {  // the segment's GROUP query rows -> qbuf[k & 1]
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
      for (int b = item.b0; b < item.b1; b += 32) {
        const int cnt = min(32, item.b1 - b);
        const int my_id = ids;
        ids = b + 32 < item.b1 ? load_ids(seg, b + 32) : (have_nxt ? load_ids(nxt, nxt.it.b0) : 0);
        for (int j = 0; j < cnt; ++j) {
          const int pb = __shfl_sync(0xffffffffu, my_id, j);
          const uint32_t slot = it % L::kStages;
          const uint32_t par = ((it / L::kStages) & 1u) ^ 1u;
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
              const int row = (pb * a.num_kv_heads + item.kvh) * BS;
              const uint32_t dst = ring + slot * L::kStage;
              mbar_arrive_expect_tx(&full[slot], L::kStage);
#ifdef PA_TEST_LOST_COPY
              // Test build only (libpa_waittest.so): ring use PA_TEST_LOST_COPY
              // of CTA 0 is announced on its barrier but never copied, so the
              // consumers' wait for it expires and the CTA unwinds.
              if (blockIdx.x == 0 && it - 1 == (uint32_t)PA_TEST_LOST_COPY) {
              } else
#endif
              if constexpr (F8) {  // each E4M3 tile is one contiguous run of BS * D bytes
                const int64_t off = (int64_t)row * D;
                bulk_load(smem + lay.ring + slot * L::kStage,
                          static_cast<const unsigned char *>(a.k_cache) + off, L::kTile, &full[slot]);
                bulk_load(smem + lay.ring + slot * L::kStage + L::kTile,
                          static_cast<const unsigned char *>(a.v_cache) + off, L::kTile, &full[slot]);
              } else {
#pragma unroll
                for (int bx = 0; bx < D / 64; ++bx) {
                  tma_load_2d(dst + bx * (BS * 128), &tmk, bx * 64, row, &full[slot]);
                  tma_load_2d(dst + L::kTile + bx * (BS * 128), &tmv, bx * 64, row, &full[slot]);
                }
              }
            }
          }
          __syncwarp();
        }
      }
      if (seg.out == kOutDirect && item.boff > 0) {
        // The prefix kernel's partial that this item folds in at its end
        // ([group heads][D + 4] floats) comes through the next ring stages,
        // kStage bytes each: issued behind the item's last block, it lands
        // while that block is computed, where a global read at the fold
        // would wait a full round trip of a saturated memory system.
        const int rec_bytes = a.group * (D + 4) * 4;
        const unsigned char *pr = reinterpret_cast<const unsigned char *>(
            a.pre_rec + ((int64_t)item.seq * a.num_heads + item.kvh * a.group) * (D + 4));
        for (int c = 0; c * L::kStage < rec_bytes; ++c) {
          const uint32_t slot = it % L::kStages;
          const uint32_t par = ((it / L::kStages) & 1u) ^ 1u;
          ++it;
          bool ok = !*abort_flag;
          if (ok) ok = mbar_wait(&empty[slot], par);
          if (lane == 0) {
            if (!ok) {
              if (!*abort_flag) raise_error(a.err, PA_DEVERR_TIMEOUT);
              *abort_flag = 1;
              bad[slot] = 1;
              mbar_arrive(&full[slot]);
            } else {
              bad[slot] = 0;
              const int bytes = min(L::kStage, rec_bytes - c * L::kStage);
              mbar_arrive_expect_tx(&full[slot], bytes);
              bulk_load(smem + lay.ring + slot * L::kStage, pr + c * L::kStage, bytes, &full[slot]);
            }
          }
          __syncwarp();
        }
      }
      seg = nxt;
      have = have_nxt;
      if (have) have_nxt = iter.next(a, bsm, n, &nxt);
    }
    // the copies this warp started land before the CTA may exit
    if (lane == 0 && !(drain_ring(full, L::kStages, it) & drain_ring(qfull, 2, k))) {
      if (!*abort_flag) raise_error(a.err, PA_DEVERR_TIMEOUT);
      *abort_flag = 1;
    }
    return;
  }

  // ======================= consumer warps ==================================
  const int g = lane >> 2, t = lane & 3;  // mma fragment coordinates
  float *merge = reinterpret_cast<float *>(smem + lay.merge);
  const int mstride = a.group * (D + 4);
  const float sl2 = a.scale_log2;

  uint32_t it_base = 0, k = 0;
  SegIter iter;
  iter.init(a, bsm, n);
  Seg seg;
  for (; iter.next(a, bsm, n, &seg); ++k) {
    const Item &item = seg.it;
    const int nblocks = item.b1 - item.b0;

    // q as the B operand of S^T = K Q^T: b0 = Q[head][16ks+2t..], b1 = +8
    uint32_t qb[NT][KS][2];
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
      const uint16_t *qr = reinterpret_cast<const uint16_t *>(qbuf + qs * lay.qbytes);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int head = nt * 8 + g;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          if (head < a.group) {
            qb[nt][ks][0] = *reinterpret_cast<const uint32_t *>(qr + head * D + ks * 16 + 2 * t);
            qb[nt][ks][1] = *reinterpret_cast<const uint32_t *>(qr + head * D + ks * 16 + 8 + 2 * t);
          } else {
            qb[nt][ks][0] = qb[nt][ks][1] = 0u;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&qempty[qs]);
    }
    // Logit factor of heads 2t, 2t+1 of each n-tile: scale * log2(e) (times
    // k_scale for an FP8 cache), divided by the power of two that brought a
    // bf16 q row into fp16 range for the fp16 products.
    float qf[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) qf[nt][0] = qf[nt][1] = sl2;
    if constexpr (F8 && std::is_same<T, __nv_bfloat16>::value) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float mx = 0.f;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks)
#pragma unroll
          for (int j2 = 0; j2 < 2; ++j2) {
            const uint32_t u = qb[nt][ks][j2];
            mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(u << 16)), fabsf(__uint_as_float(u & 0xffff0000u))));
          }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        int e = 0;
        if (mx > 0.f && isfinite(mx)) frexpf(mx, &e);  // mx < 2^e
        const int sh = max(-100, min(100, 15 - e));     // |q| * 2^sh < 2^15 < fp16 max
        const float up = ldexpf(1.f, sh);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks)
#pragma unroll
          for (int j2 = 0; j2 < 2; ++j2) {
            const uint32_t u = qb[nt][ks][j2];
            __half2 h = __floats2half2_rn(__uint_as_float(u << 16) * up,
                                          __uint_as_float(u & 0xffff0000u) * up);
            qb[nt][ks][j2] = *reinterpret_cast<uint32_t *>(&h);
          }
        const float down = sl2 * ldexpf(1.f, -sh);
        qf[nt][0] = __shfl_sync(0xffffffffu, down, (2 * t) * 4);
        qf[nt][1] = __shfl_sync(0xffffffffu, down, (2 * t + 1) * 4);
      }
    }

    float o[NT][MT][4];
    float m[NT][2], l[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      m[nt][0] = m[nt][1] = -INFINITY;
      l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) o[nt][mt][0] = o[nt][mt][1] = o[nt][mt][2] = o[nt][mt][3] = 0.f;
    }
    bool item_bad = item.bad_bits != 0;
    if (item.bad_bits && tid == 0 && item.kvh == 0) raise_error(a.err, item.bad_bits);

    // Every consumer warp waits for and releases every stage in ring order
    // (no parity wait is ever more than one phase ahead of its barrier) but
    // computes only the blocks j = warp, warp + NCW, ... of the item.
    auto wait_stage = [&](uint32_t itn) -> bool {
      const uint32_t slot = itn % L::kStages;
      bool ok = !*abort_flag;
      if (ok) {
        ok = mbar_wait(&full[slot], (itn / L::kStages) & 1u);
        if (!ok && lane == 0) {
          if (!*abort_flag) raise_error(a.err, PA_DEVERR_TIMEOUT);
          *abort_flag = 1;
        }
      }
      return ok && !bad[slot];
    };
    auto release_stage = [&](uint32_t itn) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[itn % L::kStages]);
    };
    int next = 0;
    for (int j = warp; j < nblocks; j += NCW) {
      for (; next < j; ++next) {
        wait_stage(it_base + next);
        release_stage(it_base + next);
      }
      next = j + 1;
      const uint32_t itn = it_base + j;
      if (!wait_stage(itn)) {
        item_bad = true;
      } else {
        const int nvalid = min(BS, item.L - (item.b0 + j) * BS);
        const uint32_t ktile = ring + (itn % L::kStages) * L::kStage;
        const uint32_t vtile = ktile + L::kTile;
#pragma unroll
        for (int r0 = 0; r0 < BS; r0 += 16) {
          if (r0 < nvalid) {
            // ---- S^T = K Q^T over this 16-key sub-tile ----
            float s[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
            if constexpr (F8) {
              // E4M3 tile: the codes of this thread's fragment (rows g, g+8;
              // columns 2t, 2t+1, 2t+8, 2t+9 of four k-steps) are one 16-byte
              // chunk per row; each pair of codes converts to an fp16 pair.
              const int ra = r0 + g, rb = ra + 8;
#pragma unroll
              for (int j = 0; j < D / 64; ++j) {
                const uint4 wa = ld_shared_v4(ktile + ra * D + (((4 * j + t) ^ (ra & (D / 16 - 1))) << 4));
                const uint4 wb = ld_shared_v4(ktile + rb * D + (((4 * j + t) ^ (rb & (D / 16 - 1))) << 4));
                const uint32_t xa[4] = {wa.x, wa.y, wa.z, wa.w};
                const uint32_t xb[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
                for (int kq = 0; kq < 4; ++kq) {
                  uint32_t af[4];  // rows g / g+8 x columns 2t.. / 2t+8..
                  e4m3x4_to_f16x2x2(xa[kq], af[0], af[2]);
                  e4m3x4_to_f16x2x2(xb[kq], af[1], af[3]);
#pragma unroll
                  for (int nt = 0; nt < NT; ++nt)
                    MmaT<Tc>::mma(s[nt], af, qb[nt][4 * j + kq][0], qb[nt][4 * j + kq][1]);
                }
              }
            } else {
              const int mi = lane >> 3;
              const int kr = r0 + (lane & 7) + (mi & 1) * 8;
#pragma unroll
              for (int ks = 0; ks < KS; ++ks) {
                uint32_t af[4];
                ldsm_x4(af, swz<BS>(ktile, kr, ks * 2 + (mi >> 1)));
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) MmaT<Tc>::mma(s[nt], af, qb[nt][ks][0], qb[nt][ks][1]);
              }
            }
            // ---- online softmax: thread holds keys r0+g, r0+g+8 of heads 2t, 2t+1 ----
            const bool v0 = r0 + g < nvalid, v1 = r0 + g + 8 < nvalid;
            uint32_t pb_hi[NT][2], pb_lo[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              float p[4], alpha[2];
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                const float x0 = v0 ? s[nt][hh] * qf[nt][hh] : -INFINITY;
                const float x1 = v1 ? s[nt][2 + hh] * qf[nt][hh] : -INFINITY;
                float mx = fmaxf(x0, x1);
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                const float mn = fmaxf(m[nt][hh], mx);
                alpha[hh] = fast_exp2(m[nt][hh] - mn);
                m[nt][hh] = mn;
                p[hh] = fast_exp2(x0 - mn);
                p[2 + hh] = fast_exp2(x1 - mn);
                l[nt][hh] = l[nt][hh] * alpha[hh] + p[hh] + p[2 + hh];
              }
              // O^T columns of heads whose max moved; skipped when every
              // factor of the warp is exactly 1 (the product would be o)
              if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                  o[nt][mt][0] *= alpha[0];
                  o[nt][mt][1] *= alpha[1];
                  o[nt][mt][2] *= alpha[0];
                  o[nt][mt][3] *= alpha[1];
                }
              }
              // P^T as the B operand: the S^T accumulator holds, per 8-key
              // half, rows = keys g and columns = heads 2t, 2t+1, i.e. the
              // m8n8 16-bit fragment of P^T transposed; movmatrix turns it
              // into rows = head g, columns = keys 2t, 2t+1
              uint32_t hw[2], lw[2];
#pragma unroll
              for (int half = 0; half < 2; ++half) {
                const uint16_t h0 = MmaT<Tc>::bits(p[2 * half]), h1 = MmaT<Tc>::bits(p[2 * half + 1]);
                hw[half] = (uint32_t)h0 | ((uint32_t)h1 << 16);
                if constexpr (MmaT<Tc>::kSplitP)
                  lw[half] = (uint32_t)MmaT<Tc>::bits(p[2 * half] - MmaT<Tc>::back(h0)) |
                             ((uint32_t)MmaT<Tc>::bits(p[2 * half + 1] - MmaT<Tc>::back(h1)) << 16);
              }
              pb_hi[nt][0] = movmatrix_t(hw[0]);
              pb_hi[nt][1] = movmatrix_t(hw[1]);
              if constexpr (MmaT<Tc>::kSplitP) {
                pb_lo[nt][0] = movmatrix_t(lw[0]);
                pb_lo[nt][1] = movmatrix_t(lw[1]);
              }
            }
            // ---- rows past the context end may hold anything (even NaN):
            //      zero them in the staged V tile, as P is 0 there ----
            if (!F8 && r0 + 16 > nvalid) {
              const int z0 = nvalid;
              const int nz = (r0 + 16 - z0) * (D / 8);
              for (int c = lane; c < nz; c += 32) {
                const int r = z0 + c / (D / 8), ch = c % (D / 8);
                asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(swz<BS>(vtile, r, ch)),
                             "r"(0u)
                             : "memory");
              }
              fence_proxy_async_smem();  // before the next TMA write of this stage
              __syncwarp();
            }
            // ---- O^T += V^T P^T ----
            if constexpr (F8) {
              // E4M3 V tile is stored transposed: the thread's keys 2t, 2t+1,
              // 2t+8, 2t+9 of one head-dim row are one word; keys past the
              // context end are masked to zero (P is 0 there, codes may be NaN)
              const int kb = r0 + 2 * t;
              const bool partial = r0 + 16 > nvalid;  // warp-uniform
              const uint32_t mlo = (kb < nvalid ? 0xffffu : 0u) | (kb + 1 < nvalid ? 0xffff0000u : 0u);
              const uint32_t mhi = (kb + 8 < nvalid ? 0xffffu : 0u) | (kb + 9 < nvalid ? 0xffff0000u : 0u);
              const int voff = BS == 16 ? 4 * t : 8 * t + 4 * (r0 >> 4);
#pragma unroll
              for (int mt = 0; mt < MT; ++mt) {
                const uint32_t wa = ld_shared_u32(vtile + (16 * mt + g) * BS + voff);
                const uint32_t wb = ld_shared_u32(vtile + (16 * mt + g + 8) * BS + voff);
                uint32_t af[4];  // head-dim rows g / g+8 x keys 2t.. / 2t+8..
                e4m3x4_to_f16x2x2(wa, af[0], af[2]);
                e4m3x4_to_f16x2x2(wb, af[1], af[3]);
                if (partial) {
                  af[0] &= mlo;
                  af[1] &= mlo;
                  af[2] &= mhi;
                  af[3] &= mhi;
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                  MmaT<Tc>::mma(o[nt][mt], af, pb_hi[nt][0], pb_hi[nt][1]);
                  if constexpr (MmaT<Tc>::kSplitP) MmaT<Tc>::mma(o[nt][mt], af, pb_lo[nt][0], pb_lo[nt][1]);
                }
              }
            } else {
              const int mi = lane >> 3;
              const int vr = r0 + (lane & 7) + (mi >> 1) * 8;
#pragma unroll
              for (int mt = 0; mt < MT; ++mt) {
                uint32_t af[4];
                ldsm_x4_t(af, swz<BS>(vtile, vr, mt * 2 + (mi & 1)));
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                  MmaT<Tc>::mma(o[nt][mt], af, pb_hi[nt][0], pb_hi[nt][1]);
                  if constexpr (MmaT<Tc>::kSplitP) MmaT<Tc>::mma(o[nt][mt], af, pb_lo[nt][0], pb_lo[nt][1]);
                }
              }
            }
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

    // ---- warp totals -> merge area [warp][head][D + 4] ----
    float *mw = merge + warp * mstride;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float lt = l[nt][hh];
        lt += __shfl_xor_sync(0xffffffffu, lt, 4);
        lt += __shfl_xor_sync(0xffffffffu, lt, 8);
        lt += __shfl_xor_sync(0xffffffffu, lt, 16);
        const int head = nt * 8 + 2 * t + hh;
        if (head < a.group) {
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            mw[head * (D + 4) + mt * 16 + g] = o[nt][mt][hh];
            mw[head * (D + 4) + mt * 16 + g + 8] = o[nt][mt][2 + hh];
          }
          if (g == 0) {
            mw[head * (D + 4) + D] = m[nt][hh];
            // an FP8 cache's values are codes * v_scale: the sum is stored
            // divided by v_scale, so that every later o / l carries it
            mw[head * (D + 4) + D + 1] = F8 ? lt * a.v_inv : lt;
            mw[head * (D + 4) + D + 2] = item_bad ? 1.f : 0.f;
          }
        }
      }
    }
    // the prefix partial of a shared-prefix item, from the ring stages the
    // producer loaded it into (a failed stage poisons the row: NaN sum)
    const int nrec = (seg.out == kOutDirect && item.boff > 0)
                         ? (a.group * (D + 4) * 4 + L::kStage - 1) / L::kStage : 0;
    bool rec_ok = true;
    for (int c = 0; c < nrec; ++c) rec_ok &= wait_stage(it_base + c);
    const unsigned char *ring_g = smem + lay.ring;
    const uint32_t rec_first = it_base;
    auto pre = [&](int hg, int d4, float4 *x, float *pm, float *pl) {
      const int f = (hg * (D + 4) + d4 * 4) * 4;  // byte offsets inside the record:
      const int fm = (hg * (D + 4) + D) * 4;      // each 16-byte run lies in one stage
      const unsigned char *px = ring_g + ((rec_first + f / L::kStage) % L::kStages) * L::kStage + f % L::kStage;
      const unsigned char *pmp = ring_g + ((rec_first + fm / L::kStage) % L::kStages) * L::kStage + fm % L::kStage;
      *x = *reinterpret_cast<const float4 *>(px);
      *pm = reinterpret_cast<const float *>(pmp)[0];
      *pl = rec_ok ? reinterpret_cast<const float *>(pmp)[1] : __int_as_float(0x7fc00000);
    };
    named_sync(1, NCW * 32);
    merge_store<T, D>(a, seg, merge, mstride, a.group, 1, NCW, NCW, tid, pre);
    for (int c = 0; c < nrec; ++c) release_stage(it_base + c);
    it_base += nrec;
    if (seg.out == kOutRecord && item.b0 == 0 && tid == 0) {
      // This CTA holds the first piece of a pair cut at its range end: leave
      // the merge kernel a descriptor {record slot, kv head, last covering
      // CTA, query row}.
      const int nu = ceil_div(item.L, a.block_size) + a.item_units;  // the pair's units
      const int64_t W = (int64_t)bsm.prefix[n] * a.num_kv_heads;
      const int64_t ps = (int64_t)bsm.prefix[item.seq - a.seq_begin] * a.num_kv_heads +
                         (int64_t)item.kvh * nu;
      int *d = a.bal_desc + 4 * blockIdx.x;
      d[1] = item.kvh;
      d[2] = bal_owner(ps + nu - 1, W, gridDim.x);
      d[3] = item.qrow;
      d[0] = seg.index;  // record slot of this piece in this CTA
    }
    named_sync(1, NCW * 32);
  }
}

// Merge the partial records of the (sequence, KV head) pairs that the
// balanced partition cut.  The decode kernel leaves, for every CTA holding
// the first piece of a cut pair, a descriptor {sequence, kv head, last
// covering CTA, query row}; one warp per (CTA, group head) merges that
// pair's head from the records of CTAs first .. last.  Launched as a programmatic
// dependent of the decode grid: griddepcontrol.wait returns once that grid
// has finished and its writes are visible.
template <typename T, int D>
__global__ void __launch_bounds__(256) balanced_merge_kernel(const AttnArgs a) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int w = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);  // (CTA, group head)
  const int lane = threadIdx.x & 31;
  const int G = a.grid, grp = a.group;
  const int first = w / grp, hg = w - first * grp;
  if (first >= G) return;
  const int4 d = *reinterpret_cast<const int4 *>(a.bal_desc + 4 * first);
  const int64_t W = (int64_t)a.bal_prefix[a.num_seqs] * a.num_kv_heads;
  if (d.x < 0) return;  // no cut pair starts in this CTA
  const int slot0 = d.x, kvh = d.y, last = d.z, qrow = d.w;
  constexpr int PER = D / 32;
  float M = -INFINITY, Lsum = 0.f;
  bool poisoned = false;
  float o[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) o[e] = 0.f;
  for (int c = first; c <= last; ++c) {
    if (c > first && bal_start(c + 1, W, G) == bal_start(c, W, G)) continue;  // empty range
    // the pair's piece is record slot0 of CTA `first` and the first segment
    // (slot 0) of every later CTA
    const float *r = a.part_o + (((int64_t)c * 2 + (c == first ? slot0 : 0)) * grp + hg) * (D + 4);
    float x[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) x[e] = r[lane * PER + e];
    const float m = r[D], l = r[D + 1];
    poisoned |= isnan(l);
    const float Mn = fmaxf(M, m);
    const float sa = M == -INFINITY ? 0.f : fast_exp2(M - Mn);
    const float sb = m == -INFINITY ? 0.f : fast_exp2(m - Mn);
    Lsum = Lsum * sa + l * sb;
#pragma unroll
    for (int e = 0; e < PER; ++e) o[e] = o[e] * sa + x[e] * sb;
    M = Mn;
  }
  if (a.seq_pre && a.seq_pre[qrow] > 0) {
    // the sequence's shared prefix: fold in the prefix kernel's partial
    // (one decode row per sequence here, so the query row is the sequence)
    const float *r = a.pre_rec + ((int64_t)qrow * a.num_heads + kvh * grp + hg) * (D + 4);
    const float m = r[D], l = r[D + 1];
    if (isnan(l)) {
      poisoned = true;
    } else {
      const float Mn = fmaxf(M, m);
      if (Mn != -INFINITY) {
        const float sa = M == -INFINITY ? 0.f : fast_exp2(M - Mn);
        const float sb = m == -INFINITY ? 0.f : fast_exp2(m - Mn);
        Lsum = Lsum * sa + l * sb;
#pragma unroll
        for (int e = 0; e < PER; ++e) o[e] = o[e] * sa + r[lane * PER + e] * sb;
        M = Mn;
      }
    }
  }
  const float inv = (Lsum > 0.f && !poisoned) ? 1.f / Lsum : 0.f;
  T *dst = static_cast<T *>(a.out) + ((int64_t)qrow * a.num_heads + kvh * grp + hg) * D + lane * PER;
#pragma unroll
  for (int e = 0; e < PER; ++e) dst[e] = Elem<T>::from_f(o[e] * inv);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  // looked up once; a function-local static is initialised thread-safely
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    cudaDriverEntryPointQueryResult q;
    void *p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return nullptr;
  }();
  return fn;
}

// 2-D view of a cache: rows = num_blocks * num_kv_heads * block_size, columns
// = head_dim; boxes of 64 columns x block_size rows, 128-byte swizzle.
template <typename T, int D, int BS>
bool make_map(CUtensorMap *map, const void *base, int num_blocks, int num_kv_heads) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)num_blocks * num_kv_heads * BS};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)BS};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, MmaT<T>::kTmaType, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool make_cache_map(CUtensorMap *map, const void *base, int num_blocks, int num_kv_heads,
                    int head_dim, int block_size, int dtype) {
  if (dtype != PA_F16 && dtype != PA_BF16) return false;
  const bool bf = dtype == PA_BF16;
  if (head_dim == 64)
    return block_size == 16
               ? (bf ? make_map<__nv_bfloat16, 64, 16>(map, base, num_blocks, num_kv_heads)
                     : make_map<__half, 64, 16>(map, base, num_blocks, num_kv_heads))
               : (bf ? make_map<__nv_bfloat16, 64, 32>(map, base, num_blocks, num_kv_heads)
                     : make_map<__half, 64, 32>(map, base, num_blocks, num_kv_heads));
  return block_size == 16
             ? (bf ? make_map<__nv_bfloat16, 128, 16>(map, base, num_blocks, num_kv_heads)
                   : make_map<__half, 128, 16>(map, base, num_blocks, num_kv_heads))
             : (bf ? make_map<__nv_bfloat16, 128, 32>(map, base, num_blocks, num_kv_heads)
                   : make_map<__half, 128, 32>(map, base, num_blocks, num_kv_heads));
}

namespace {

template <typename T, int D, int BS, int NT, bool F8>
cudaError_t launch_mma_t(const AttnArgs &a, int sm_count, cudaStream_t stream) {
  constexpr int NCW = PA_MMA_WARPS;
  using L = MmaLayout<D, BS, NT, NCW, F8>;
  auto kern = paged_decode_mma_kernel<T, D, BS, NT, NCW, F8>;
  CUtensorMap tmk{}, tmv{};  // E4M3 tiles are moved with plain bulk copies
  if (!F8 && !(make_map<T, D, BS>(&tmk, a.k_cache, a.num_blocks, a.num_kv_heads) &&
               make_map<T, D, BS>(&tmv, a.v_cache, a.num_blocks, a.num_kv_heads)))
    return cudaErrorInvalidValue;
  const L lay(a.num_seqs, a.group);
  const L big(kMaxSeqsPerLaunch, 8 * NT);
  cudaError_t e = set_smem_limit_once(reinterpret_cast<const void *>(kern), big.bytes, true);
  if (e != cudaSuccess) return e;
  int occ = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, 32 * (NCW + 1), lay.bytes);
  if (e != cudaSuccess) return e;
  if (occ < 1) occ = 1;
  int64_t grid = (int64_t)sm_count * occ;
  if (a.balanced) {
    grid = a.grid;  // fixed by the host (records are per CTA)
  } else {
    const int64_t max_items = (int64_t)a.num_seqs * a.num_kv_heads * a.max_splits;
    if (grid > max_items) grid = max_items;
  }
  if (grid < 1) grid = 1;
  // programmatic dependent launch: the grid may be scheduled while the
  // previous kernel in the stream finishes; it waits (griddepcontrol.wait)
  // before touching global memory.  Not beside a mixed batch's chunk rows
  // forked to another stream: there the decode CTAs, all resident at once,
  // would take every SM before the chunk kernel placed its CTAs.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(32 * (NCW + 1));
  cfg.dynamicSmemBytes = lay.bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.no_pdl ? 0 : 1;
  return cudaLaunchKernelEx(&cfg, kern, a, tmk, tmv);
}

template <typename T, int D, int BS, int NT, bool F8>
int grid_mma_t(const AttnArgs &a, int sm_count) {
  constexpr int NCW = PA_MMA_WARPS;
  using L = MmaLayout<D, BS, NT, NCW, F8>;
  auto kern = paged_decode_mma_kernel<T, D, BS, NT, NCW, F8>;
  const L big(kMaxSeqsPerLaunch, 8 * NT);
  if (set_smem_limit_once(reinterpret_cast<const void *>(kern), big.bytes, true) != cudaSuccess) return 0;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, 32 * (NCW + 1),
                                                    L(a.num_seqs, a.group).bytes) != cudaSuccess)
    return 0;
  return sm_count * (occ < 1 ? 1 : occ);
}

template <typename T, bool F8 = false>
int grid_mma_d(const AttnArgs &a, int sm_count) {
  if (a.head_dim == 64)
    return a.block_size == 16 ? (a.group <= 8 ? grid_mma_t<T, 64, 16, 1, F8>(a, sm_count) : grid_mma_t<T, 64, 16, 2, F8>(a, sm_count))
                              : (a.group <= 8 ? grid_mma_t<T, 64, 32, 1, F8>(a, sm_count) : grid_mma_t<T, 64, 32, 2, F8>(a, sm_count));
  return a.block_size == 16 ? (a.group <= 8 ? grid_mma_t<T, 128, 16, 1, F8>(a, sm_count) : grid_mma_t<T, 128, 16, 2, F8>(a, sm_count))
                            : (a.group <= 8 ? grid_mma_t<T, 128, 32, 1, F8>(a, sm_count) : grid_mma_t<T, 128, 32, 2, F8>(a, sm_count));
}

template <typename T>
cudaError_t launch_bal_reduce_t(const AttnArgs &a, cudaStream_t stream) {
  const int warps = a.grid * a.group;  // one per (CTA descriptor, group head)
  if (warps <= 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((warps * 32 + 255) / 256));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.no_pdl ? 0 : 1;
  if (a.head_dim == 64) return cudaLaunchKernelEx(&cfg, balanced_merge_kernel<T, 64>, a);
  return cudaLaunchKernelEx(&cfg, balanced_merge_kernel<T, 128>, a);
}

template <typename T, int D, int BS, bool F8>
cudaError_t mma_nt(const AttnArgs &a, int sm_count, cudaStream_t s) {
  return a.group <= 8 ? launch_mma_t<T, D, BS, 1, F8>(a, sm_count, s)
                      : launch_mma_t<T, D, BS, 2, F8>(a, sm_count, s);
}

template <typename T, int D, bool F8>
cudaError_t mma_bs(const AttnArgs &a, int sm_count, cudaStream_t s) {
  return a.block_size == 16 ? mma_nt<T, D, 16, F8>(a, sm_count, s) : mma_nt<T, D, 32, F8>(a, sm_count, s);
}

template <typename T, bool F8 = false>
cudaError_t mma_d(const AttnArgs &a, int sm_count, cudaStream_t s) {
  return a.head_dim == 64 ? mma_bs<T, 64, F8>(a, sm_count, s) : mma_bs<T, 128, F8>(a, sm_count, s);
}

}  // namespace

int decode_mma_grid(const AttnArgs &a, int dtype, int sm_count) {
  return dtype == PA_F16 ? grid_mma_d<__half>(a, sm_count) : grid_mma_d<__nv_bfloat16>(a, sm_count);
}

cudaError_t launch_balanced_reduce(const AttnArgs &a, int dtype, cudaStream_t stream) {
  return dtype == PA_F16 ? launch_bal_reduce_t<__half>(a, stream)
                         : launch_bal_reduce_t<__nv_bfloat16>(a, stream);
}

bool decode_mma_supported(const AttnArgs &a, int dtype) {
  return (dtype == PA_F16 || dtype == PA_BF16) && a.group >= 1 && a.group <= 16 &&
         encode_fn() != nullptr;
}

cudaError_t launch_decode_mma(const AttnArgs &a, int dtype, int sm_count, cudaStream_t stream) {
  if (dtype == PA_F16) return mma_d<__half>(a, sm_count, stream);
  return mma_d<__nv_bfloat16>(a, sm_count, stream);
}

int decode_mma_grid_fp8(const AttnArgs &a, int q_dtype, int sm_count) {
  return q_dtype == PA_F16 ? grid_mma_d<__half, true>(a, sm_count)
                           : grid_mma_d<__nv_bfloat16, true>(a, sm_count);
}

cudaError_t launch_decode_mma_fp8(const AttnArgs &a, int q_dtype, int sm_count,
                                  cudaStream_t stream) {
  if (q_dtype == PA_F16) return mma_d<__half, true>(a, sm_count, stream);
  return mma_d<__nv_bfloat16, true>(a, sm_count, stream);
}

}  // namespace pa
