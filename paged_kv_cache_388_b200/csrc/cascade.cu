// cascade.cu -- shared-prefix decode: attention over the KV blocks that a
// group of sequences shares, computed once for the whole group.
//
// Sequences forked from one prompt (parallel sampling, beam search) map the
// prompt's logical blocks to the same physical blocks and own only what they
// write after the fork ("理解 vLLM PagedAttention", section 六; "核心概念",
// section 内存共享).  Plain decode reads a shared block once per sequence that
// uses it.  Here the query rows of all members of a group that read one KV
// head -- members x GROUP heads, up to 64 rows -- form one tile, so each
// shared K/V block is read once per group and the products are real matrix
// products.  The rest of each sequence, its private tail, is attended by the
// decode kernel, which folds in this kernel's partial softmax result (running
// max, running sum, unnormalised accumulator) the way it merges split-KV
// pieces; the result equals plain decode up to fp32 rounding.
//
// Work layout: one thread-block cluster of C CTAs per (group, member chunk,
// KV head).  CTA r of the cluster takes the r-th of C contiguous ranges of
// the shared blocks; the C partial results are merged through distributed
// shared memory, so the prefix leaves exactly one record (o, m, l) per
// (sequence, head) in global memory.
//
// Per CTA: one producer warp issues the Q gather (one bulk copy per member)
// and, per stage of 64 keys, tensor-map TMA loads of the stage's K and V
// block tiles (128-byte swizzle); it also checks that every member's block
// table holds the group's block ids over the shared range.  Four consumer
// warps own 16 query rows each: S = Q K^T and O += P V with mma.sync
// m16n8k16 (rows on M, fp32 accumulate), online softmax in base 2, and for
// bf16 the P operand split into hi + lo parts.
#include <stdlib.h>

#include "mma_sync.cuh"
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kRows = kPrefixRows;  // query rows per CTA
constexpr int kKeys = 64;           // keys per pipeline stage
constexpr int kCW = 4;              // consumer warps, 16 rows each
constexpr int kThreads = 32 * (kCW + 1);

template <int D, int BS>
struct PxLayout {
  static constexpr int kBlk = kKeys / BS;            // KV blocks per stage
  static constexpr int kTile = BS * D * 2;           // one block's K (or V) tile, bytes
  static constexpr int kStage = 2 * kBlk * kTile;    // the stage's K tiles, then its V tiles
  static constexpr int kStages = (64 * 1024) / kStage;
  static constexpr int kRing = 0;                    // 1024-byte aligned (128-byte swizzle)
  static constexpr int kQ = kRing + kStages * kStage;  // [kRows][D] 16-bit, dense rows
  static constexpr int kFull = kQ + kRows * D * 2;
  static constexpr int kEmpty = kFull + 8 * kStages;
  static constexpr int kQBar = kEmpty + 8 * kStages;
  static constexpr int kBad = kQBar + 8;
  static constexpr int kMisc = kBad + 4 * kStages;   // abort flag (int), member mask (u64 at +8)
  static constexpr int kBytes = kMisc + 16 + 1024;   // + alignment slack
  // merge area [kRows][D + 4] floats: accumulator, max, sum, bad flag; it
  // reuses the ring once every stage has been consumed
  static constexpr int kMS = D + 4;
  static_assert(kStages >= 2, "the ring needs two stages");
  static_assert(kRows * kMS * 4 <= kStages * kStage, "merge area must fit in the ring");
  static_assert(kMisc % 8 == 0, "member mask alignment");
};

// Byte address of the 8-element group (r, c8 * 8) of a staged block tile:
// D/64 boxes of BS rows x 128 bytes written by TMA with the 128-byte swizzle
// (16-byte chunk c of row r at chunk position c ^ (r % 8)).
template <int BS>
__device__ __forceinline__ uint32_t swz(uint32_t tile, int r, int c8) {
  const int box = c8 >> 3, chunk = c8 & 7;
  return tile + box * (BS * 128) + r * 128 + ((chunk ^ (r & 7)) << 4);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

// ---- thread-block cluster: barrier and distributed shared memory ------------
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_map(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ float4 ld_cluster_v4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ unsigned long long ld_cluster_u64(uint32_t addr) {
  unsigned long long v;
  asm volatile("ld.shared::cluster.u64 %0, [%1];" : "=l"(v) : "r"(addr) : "memory");
  return v;
}

template <typename T, int D, int BS>
__global__ void __launch_bounds__(kThreads, 2)
    shared_prefix_kernel(const AttnArgs a, const __grid_constant__ CUtensorMap tmk,
                         const __grid_constant__ CUtensorMap tmv) {
  using Lay = PxLayout<D, BS>;
  constexpr int KS = D / 16;
  constexpr int MS = Lay::kMS;
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + Lay::kFull);
  uint64_t *empty = reinterpret_cast<uint64_t *>(smem + Lay::kEmpty);
  uint64_t *qbar = reinterpret_cast<uint64_t *>(smem + Lay::kQBar);
  int *bad = reinterpret_cast<int *>(smem + Lay::kBad);
  volatile int *abort_flag = reinterpret_cast<int *>(smem + Lay::kMisc);
  unsigned long long *mbad = reinterpret_cast<unsigned long long *>(smem + Lay::kMisc + 8);
  const uint32_t ring = smem_addr(smem + Lay::kRing);
  const uint32_t sq = smem_addr(smem + Lay::kQ);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  uint32_t crank, csize;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(crank));
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(csize));

  if (tid == 0) {
    for (int s = 0; s < Lay::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCW);
    }
    mbar_init(qbar, 1);
    *abort_flag = 0;
    *mbad = 0ull;
    mbar_init_fence();
  }
  __syncthreads();
  // Launched as a programmatic dependent of the previous kernel (the cache
  // write): nothing is read from global memory before its writes are visible.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // The cluster's unit: (group j, member chunk, KV head).  Every CTA of the
  // cluster reads the same values, so a cluster leaves here as a whole.
  const int Hk = a.num_kv_heads, G = a.group;
  const int unit = (int)(blockIdx.x / csize);
  const int kvh = unit % Hk;
  const int chunk = (unit / Hk) % a.grp_chunks;
  const int j = unit / Hk / a.grp_chunks;
  const int n = a.num_seqs;
  const int s0 = a.grp_start[j], s1 = a.grp_start[j + 1], P = a.grp_blocks[j];
  const int mpc = kRows / G;  // members per chunk
  const int m0 = s0 + chunk * mpc;
  if (!(0 <= s0 && s0 <= s1 && s1 <= n && 0 < P && P <= a.max_blocks_per_seq && m0 < s1)) return;
  const int nmem = min(mpc, s1 - m0);
  const int b_lo = (int)((int64_t)crank * P / csize);
  const int b_hi = (int)((int64_t)(crank + 1) * P / csize);
  const int nstage = (b_hi - b_lo + Lay::kBlk - 1) / Lay::kBlk;
  const int32_t *lead = a.block_tables + (int64_t)s0 * a.max_blocks_per_seq;
  float *mrg = reinterpret_cast<float *>(smem + Lay::kRing);

  if (warp == kCW) {
    // ============================ producer warp ============================
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmk)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmv)) : "memory");
      // Q rows of the chunk: member i's GROUP heads of this KV head are g*D
      // contiguous elements of q, staged as rows i*G .. i*G+G-1.
      const uint32_t qbytes = (uint32_t)G * D * 2;
      mbar_arrive_expect_tx(qbar, (uint32_t)nmem * qbytes);
      for (int i = 0; i < nmem; ++i)
        bulk_load(smem + Lay::kQ + i * qbytes,
                  static_cast<const T *>(a.q) + ((int64_t)(m0 + i) * a.num_heads + kvh * G) * D,
                  qbytes, qbar);
    }
    // Block ids of the next stage are loaded while the current stage's loads
    // are issued; the member-table check runs after the issue, off the path.
    int cnt = nstage > 0 ? min(Lay::kBlk, b_hi - b_lo) : 0;
    int id = lane < cnt ? lead[b_lo + lane] : 0;
    for (int st = 0; st < nstage; ++st) {
      const int slot = st % Lay::kStages;
      const uint32_t par = ((st / Lay::kStages) & 1u) ^ 1u;
      const int bb = b_lo + st * Lay::kBlk;
      const bool anybad = __any_sync(0xffffffffu, lane < cnt && (id < 0 || id >= a.num_blocks));
      int ids[Lay::kBlk];
#pragma unroll
      for (int t = 0; t < Lay::kBlk; ++t) ids[t] = __shfl_sync(0xffffffffu, id, t);
      bool ok = !*abort_flag;
      if (ok) ok = mbar_wait(&empty[slot], par);
      if (lane == 0) {
        if (!ok) {
          if (!*abort_flag) raise_error(a.err, PA_DEVERR_TIMEOUT);
          *abort_flag = 1;
          bad[slot] = 1;
          mbar_arrive(&full[slot]);
        } else if (anybad) {
          raise_error(a.err, PA_DEVERR_BLOCK_ID);
          bad[slot] = 1;
          mbar_arrive(&full[slot]);
        } else {
          bad[slot] = 0;
          mbar_arrive_expect_tx(&full[slot], (uint32_t)(cnt * 2 * Lay::kTile));
          const uint32_t kdst = ring + slot * Lay::kStage;
          const uint32_t vdst = kdst + Lay::kBlk * Lay::kTile;
#pragma unroll
          for (int t = 0; t < Lay::kBlk; ++t) {
            if (t < cnt) {
              const int row = (ids[t] * Hk + kvh) * BS;
#pragma unroll
              for (int bx = 0; bx < D / 64; ++bx) {
                tma_load_2d(kdst + t * Lay::kTile + bx * (BS * 128), &tmk, bx * 64, row, &full[slot]);
                tma_load_2d(vdst + t * Lay::kTile + bx * (BS * 128), &tmv, bx * 64, row, &full[slot]);
              }
            }
          }
        }
      }
      __syncwarp();
      const int bn = bb + Lay::kBlk;
      const int cnt_n = st + 1 < nstage ? min(Lay::kBlk, b_hi - bn) : 0;
      const int id_n = lane < cnt_n ? lead[bn + lane] : 0;
      // every member's table must hold the group's ids over the shared range
      for (int x = lane; x < nmem * cnt; x += 32) {
        const int i = x / cnt, t = x - i * cnt;
        if (a.block_tables[(int64_t)(m0 + i) * a.max_blocks_per_seq + bb + t] != lead[bb + t])
          atomicOr(mbad, 1ull << i);
      }
      id = id_n;
      cnt = cnt_n;
    }
    __syncwarp();
    if (lane == 0 && *mbad) raise_error(a.err, PA_DEVERR_PREFIX);
    // the copies this warp started land before the CTA may exit
    if (lane == 0 && !(drain_ring(full, Lay::kStages, nstage) & drain_ring(qbar, 1, 1))) {
      if (!*abort_flag) raise_error(a.err, PA_DEVERR_TIMEOUT);
      *abort_flag = 1;
    }
  } else {
    // ============================ consumer warps ===========================
    const int g8 = lane >> 2, tig = lane & 3;
    bool tbad = false;
    {
      bool ok = !*abort_flag;
      if (ok) {
        ok = mbar_wait(qbar, 0);
        if (!ok && lane == 0) {
          if (!*abort_flag) raise_error(a.err, PA_DEVERR_TIMEOUT);
          *abort_flag = 1;
        }
      }
      tbad = !ok;
    }
    uint32_t qa[KS][4];
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      const int c = ks * 16 + (lane >> 4) * 8;
      ldsm_x4_a(qa[ks], sq + (uint32_t)(r * D + c) * 2u);
    }
    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
    const float sl2 = a.scale_log2;

    for (int st = 0; st < nstage; ++st) {
      const int slot = st % Lay::kStages;
      const uint32_t par = (st / Lay::kStages) & 1u;
      bool sok = !*abort_flag;
      if (sok) {
        sok = mbar_wait(&full[slot], par);
        if (!sok && lane == 0) {
          if (!*abort_flag) raise_error(a.err, PA_DEVERR_TIMEOUT);
          *abort_flag = 1;
        }
      }
      if (!sok || bad[slot]) {
        tbad = true;
      } else {
        const int nkeys = min(Lay::kBlk, b_hi - (b_lo + st * Lay::kBlk)) * BS;  // multiple of 16
        const uint32_t kt = ring + slot * Lay::kStage;
        const uint32_t vt = kt + Lay::kBlk * Lay::kTile;

        // ---- S = Q K^T: 16 rows x 64 keys per warp ----
        float s[kKeys / 8][4];
#pragma unroll
        for (int i = 0; i < kKeys / 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
        for (int np = 0; np < kKeys / 16; ++np) {
          if (np * 16 < nkeys) {
            const int key = np * 16 + (lane & 7) + (lane >> 4) * 8;
            const uint32_t tile = kt + (key / BS) * Lay::kTile;
            const int r = key % BS;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
              uint32_t b[4];
              ldsm_x4_a(b, swz<BS>(tile, r, ks * 2 + ((lane >> 3) & 1)));
              Mma<T>::run(s[2 * np], qa[ks], b[0], b[1]);
              Mma<T>::run(s[2 * np + 1], qa[ks], b[2], b[3]);
            }
          }
        }

        // ---- online softmax (base 2); keys past the stage's blocks masked ----
        float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
        for (int i = 0; i < kKeys / 8; ++i) {
          const bool kv = i * 8 < nkeys;
#pragma unroll
          for (int c = 0; c < 4; ++c) s[i][c] = kv ? s[i][c] * sl2 : -INFINITY;
          mx_a = fmaxf(mx_a, fmaxf(s[i][0], s[i][1]));
          mx_b = fmaxf(mx_b, fmaxf(s[i][2], s[i][3]));
        }
        mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
        mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
        mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
        mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
        const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
        const float al_a = fast_exp2(m_a - mn_a), al_b = fast_exp2(m_b - mn_b);
        m_a = mn_a;
        m_b = mn_b;
        float rs_a = 0.f, rs_b = 0.f;
        uint32_t pa[kKeys / 16][4];
        uint32_t pr[Mma<T>::kSplitP ? kKeys / 16 : 1][4];
#pragma unroll
        for (int i = 0; i < kKeys / 8; ++i) {
          const float p0 = fast_exp2(s[i][0] - mn_a), p1 = fast_exp2(s[i][1] - mn_a);
          const float p2 = fast_exp2(s[i][2] - mn_b), p3 = fast_exp2(s[i][3] - mn_b);
          rs_a += p0 + p1;
          rs_b += p2 + p3;
          pa[i / 2][(i & 1) * 2 + 0] = Mma<T>::pack(p0, p1);
          pa[i / 2][(i & 1) * 2 + 1] = Mma<T>::pack(p2, p3);
          if constexpr (Mma<T>::kSplitP) {
            pr[i / 2][(i & 1) * 2 + 0] = Mma<T>::pack_residual(p0, p1);
            pr[i / 2][(i & 1) * 2 + 1] = Mma<T>::pack_residual(p2, p3);
          }
        }
        l_a = l_a * al_a + rs_a;
        l_b = l_b * al_b + rs_b;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
          o[i][0] *= al_a;
          o[i][1] *= al_a;
          o[i][2] *= al_b;
          o[i][3] *= al_b;
        }

        // ---- O += P V ----
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk) {
          if (kk * 16 < nkeys) {
            const int key = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
            const uint32_t tile = vt + (key / BS) * Lay::kTile;
            const int r = key % BS;
#pragma unroll
            for (int dp = 0; dp < D / 16; ++dp) {
              uint32_t b[4];
              ldsm_x4_ta(b, swz<BS>(tile, r, dp * 2 + (lane >> 4)));
              Mma<T>::run(o[2 * dp], pa[kk], b[0], b[1]);
              Mma<T>::run(o[2 * dp + 1], pa[kk], b[2], b[3]);
              if constexpr (Mma<T>::kSplitP) {
                Mma<T>::run(o[2 * dp], pr[kk], b[0], b[1]);
                Mma<T>::run(o[2 * dp + 1], pr[kk], b[2], b[3]);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }

    // ---- this CTA's partial rows -> merge area (reuses the drained ring) ----
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
    tbad = __any_sync(0xffffffffu, tbad) || *abort_flag;
    named_sync(1, kCW * 32);  // every consumer warp is done reading the ring
    const int ra = warp * 16 + g8, rb = ra + 8;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      *reinterpret_cast<float2 *>(mrg + ra * MS + i * 8 + tig * 2) = make_float2(o[i][0], o[i][1]);
      *reinterpret_cast<float2 *>(mrg + rb * MS + i * 8 + tig * 2) = make_float2(o[i][2], o[i][3]);
    }
    if (tig == 0) {
      mrg[ra * MS + D] = m_a;
      mrg[ra * MS + D + 1] = l_a;
      mrg[ra * MS + D + 2] = tbad ? 1.f : 0.f;
      mrg[rb * MS + D] = m_b;
      mrg[rb * MS + D + 1] = l_b;
      mrg[rb * MS + D + 2] = tbad ? 1.f : 0.f;
    }
  }
  __syncwarp();
  cluster_sync_all();  // every CTA's merge area and member mask are written

  // ---- merge rows [crank*rpc, (crank+1)*rpc) over the cluster's CTAs ----
  // Task = (row, eighth of the row): every remote value a task needs is
  // requested before the first is used, so the reads overlap.
  {
    constexpr int kParts = 8;
    constexpr int NV = D / 4 / kParts;  // float4s of the accumulator per task
    constexpr int kMaxC = 8;
    const int rpc = kRows / (int)csize;
    const uint32_t mrg_local = smem_addr(mrg);
    unsigned long long mb_all = 0ull;
#pragma unroll
    for (int c = 0; c < kMaxC; ++c)
      if (c < (int)csize) mb_all |= ld_cluster_u64(cluster_map(smem_addr(mbad), c));
    for (int task = tid; task < rpc * kParts; task += kThreads) {
      const int r = (int)crank * rpc + task / kParts, part = task % kParts;
      const int i = r / G, hg = r - i * G;
      if (i >= nmem) continue;
      const uint32_t row = mrg_local + (uint32_t)(r * MS) * 4u;
      uint32_t base[kMaxC];
      float mc[kMaxC], lc[kMaxC], bc[kMaxC];
#pragma unroll
      for (int c = 0; c < kMaxC; ++c) {
        if (c < (int)csize) {
          base[c] = cluster_map(row, c);
          mc[c] = ld_cluster_f32(base[c] + D * 4);
          lc[c] = ld_cluster_f32(base[c] + (D + 1) * 4);
          bc[c] = ld_cluster_f32(base[c] + (D + 2) * 4);
        }
      }
      float M = -INFINITY;
#pragma unroll
      for (int c = 0; c < kMaxC; ++c)
        if (c < (int)csize) M = fmaxf(M, mc[c]);
      float w[kMaxC];
      float l = 0.f;
      bool rbad = ((mb_all >> i) & 1ull) != 0;
#pragma unroll
      for (int c = 0; c < kMaxC; ++c) {
        if (c < (int)csize) {
          w[c] = mc[c] == -INFINITY ? 0.f : fast_exp2(mc[c] - M);
          l += w[c] * lc[c];
          rbad |= bc[c] != 0.f;
        }
      }
      float *rec = a.pre_rec + ((int64_t)(m0 + i) * a.num_heads + kvh * G + hg) * (D + 4);
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        const int d4 = part * NV + v;
        float4 x[kMaxC];
#pragma unroll
        for (int c = 0; c < kMaxC; ++c)
          if (c < (int)csize) x[c] = ld_cluster_v4(base[c] + d4 * 16);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int c = 0; c < kMaxC; ++c) {
          if (c < (int)csize) {
            acc.x += w[c] * x[c].x;
            acc.y += w[c] * x[c].y;
            acc.z += w[c] * x[c].z;
            acc.w += w[c] * x[c].w;
          }
        }
        *reinterpret_cast<float4 *>(rec + d4 * 4) = acc;
      }
      if (part == 0) {
        rec[D] = M;
        rec[D + 1] = rbad ? __int_as_float(0x7fc00000) : l / a.o_scale;
      }
    }
  }
  __syncwarp();
  cluster_sync_all();  // no CTA leaves while a peer may still read its merge area
}

template <typename T, int D, int BS>
cudaError_t launch_prefix_t(const AttnArgs &a, int dtype, int cluster, cudaStream_t stream) {
  using Lay = PxLayout<D, BS>;
  auto kern = shared_prefix_kernel<T, D, BS>;
  CUtensorMap tmk, tmv;
  if (!make_cache_map(&tmk, a.k_cache, a.num_blocks, a.num_kv_heads, D, BS, dtype) ||
      !make_cache_map(&tmv, a.v_cache, a.num_blocks, a.num_kv_heads, D, BS, dtype))
    return cudaErrorInvalidValue;
  {
    cudaError_t e = set_smem_limit_once(reinterpret_cast<const void *>(kern), Lay::kBytes);
    if (e != cudaSuccess) return e;
  }
  const int64_t grid = (int64_t)a.num_groups * a.grp_chunks * a.num_kv_heads * cluster;
  if (grid == 0) return cudaSuccess;
  if (grid > 0x7fffffff) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Lay::kBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, a, tmk, tmv);
}

template <typename T, int D>
cudaError_t prefix_bs(const AttnArgs &a, int dtype, int cluster, cudaStream_t s) {
  return a.block_size == 16 ? launch_prefix_t<T, D, 16>(a, dtype, cluster, s)
                            : launch_prefix_t<T, D, 32>(a, dtype, cluster, s);
}

template <typename T>
cudaError_t prefix_d(const AttnArgs &a, int dtype, int cluster, cudaStream_t s) {
  return a.head_dim == 64 ? prefix_bs<T, 64>(a, dtype, cluster, s)
                          : prefix_bs<T, 128>(a, dtype, cluster, s);
}

}  // namespace

bool prefix_supported(const AttnArgs &a, int dtype) {
  return (dtype == PA_F16 || dtype == PA_BF16) && (a.head_dim == 64 || a.head_dim == 128) &&
         (a.block_size == 16 || a.block_size == 32) && a.group >= 1 && a.group <= kRows;
}

cudaError_t launch_prefix(const AttnArgs &a, int dtype, int cluster, cudaStream_t stream) {
  if (cluster != 1 && cluster != 2 && cluster != 4 && cluster != 8) return cudaErrorInvalidValue;
  if (dtype == PA_F16) return prefix_d<__half>(a, dtype, cluster, stream);
  return prefix_d<__nv_bfloat16>(a, dtype, cluster, stream);
}

}  // namespace pa
