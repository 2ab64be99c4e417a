// chunk_pp.cu -- chunked-prefill attention on the 5th-generation tensor cores:
// two query tiles in ping-pong over 128-key K/V tiles.
//
// A chunk of Q > 1 query tokens of one sequence attends causally over the
// sequence's paged KV: row t sees keys 0 .. L-Q+t ("PagedAttention 实战",
// section Chunked Prefill).  The GROUP query heads of a token read the same
// K/V, so 128 rows (128/GROUP tokens x GROUP heads) against a tile of keys
// form a dense contraction.
//
// CTA = (sequence, KV head, 256 query rows held as two Q tiles of 128).  Per
// 128-key tile j and Q tile t the tensor cores compute S_t = Q_t K_j^T
// (M 128, N 128, K = head_dim 128) and O_t += P_t V_j (M 128, N 128, K 128)
// with fp32 accumulators in tensor memory: S_t in 128 columns, O_t in the next
// 128 -- the four regions fill the SM's 512 columns.  P_t overwrites S_t in
// place (bf16 hi + lo words, or one fp16 word, two keys a word) and is read
// from there as the A operand of P V.
//
// Ping-pong: the MMA issue order per tile is PV_0(j), S_0(j+1), PV_1(j),
// S_1(j+1), so the softmax of one Q tile runs while the tensor cores work on
// the other's products.  S_t(j+1) overwrites P_t(j): the MMA thread waits for
// P V of tile j to complete before issuing it.
//
// K/V tiles arrive by TMA through the block table, one box per (block, KV
// head) and K or V: a 5-D tensor map splits every block's rows into groups of
// 8 and each row into two 64-column halves, so a box lands as [row group]
// [half][8 rows][64 columns] -- the 128-byte-swizzle atom layout the UMMA
// descriptors want, with a uniform 2 KB stride per 8 keys across the blocks
// of a tile.  One 4 KB (block size 16) or 8 KB (32) box per block instead of
// two 2 KB boxes halves the boxes the SM's TMA unit issues per key.
//
// Warps: 8 softmax (4 per Q tile; thread = row = TMEM lane), 1 TMA producer,
// 1 MMA issuer (one elected thread) that also owns the TMEM allocation.
//
// PREFIX: the shared-prefix pass of pa_decode_shared_prefix.  The CTA is
// (group, up to 256 member rows, KV head): its rows are the decode rows of
// the group's members (one query row per sequence, 128/GROUP members per Q
// tile), its keys the group's shared blocks read through the group's first
// table, with no causal mask; the softmax warps check every member's table
// over the shared range while the first tile loads, and the epilogue writes
// one record (o unnormalised, reference max in base 2, sum; NaN sum for a
// member whose table differs) per (member, head) for the decode kernel to
// fold in.
#include <stdlib.h>
#include <string.h>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "tc_common.cuh"

namespace pa {
namespace {

constexpr int kRows = 128;   // rows per Q tile (MMA M)
constexpr int kKeys = 128;   // keys per K/V tile (N of S = Q K^T, K of P V)
constexpr int kD = 128;      // head_dim
constexpr int kQTiles = 2;
#ifndef PA_CHUNK_PP_STAGES
#define PA_CHUNK_PP_STAGES 2
#endif
constexpr int kStages = PA_CHUNK_PP_STAGES;  // K/V tiles in flight
constexpr float kRescaleThreshold = 8.0f;    // log2 units: P stays <= 2^8 between rescales
constexpr int kSoftmaxWarps = 4 * kQTiles;
constexpr int kProducerWarp = kSoftmaxWarps, kMmaWarp = kSoftmaxWarps + 1;
constexpr int kThreads = 32 * (kSoftmaxWarps + 2);

// shared memory (offsets from a 1024-byte aligned base)
constexpr int kQBytes = kRows * kD * 2;           // one Q tile: 2 halves x [128 rows][128 B]
constexpr int kOffQ = 0;
constexpr int kHalfStage = kKeys * kD * 2;        // K (or V) of one tile: 32 KB
constexpr int kStageBytes = 2 * kHalfStage;
constexpr int kOffKV = kOffQ + kQTiles * kQBytes;
constexpr int kOffMemBad = kOffKV + kStages * kStageBytes;  // prefix mode: [256] member flags
// Barriers follow the member flags, which only the prefix mode has: without
// them a chunk-row CTA (~193 KB) leaves room on its SM for a decode CTA of a
// mixed batch (~33 KB), both with 1 KB reserved, within the SM's 228 KB.
template <bool PREFIX>
constexpr int off_bar() { return kOffMemBad + (PREFIX ? 256 : 0); }
enum {
  kQFull = 0,
  kKFull = 1,                      // [kStages] the K half of a stage landed
  kVFull = kKFull + kStages,       // [kStages] the V half landed
  kKvEmpty = kVFull + kStages,     // [kStages] both Q tiles' products of the stage done
  kSFull = kKvEmpty + kStages,     // [Q tile] S in TMEM
  kPFull = kSFull + kQTiles,       // [Q tile] P written over S (4 softmax warps)
  kPvDone = kPFull + kQTiles,      // [Q tile] P V complete
  kDone = kPvDone + kQTiles,
  kNumBars = kDone + 1
};
template <bool PREFIX>
constexpr int smem_bytes() { return off_bar<PREFIX>() + 8 * kNumBars + 64 + 1024; }  // + TMEM slot, flags, alignment
static_assert(smem_bytes<true>() <= 227 * 1024, "shared memory per CTA");

// TMEM columns: Q tile t's S/P at t*256, its O at t*256 + 128.
__device__ __forceinline__ uint32_t tmem_s_col(int t) { return (uint32_t)t * 256u; }
__device__ __forceinline__ uint32_t tmem_o_col(int t) { return (uint32_t)t * 256u + 128u; }

template <typename T, int BS, bool PREFIX>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_pp_kernel(const AttnArgs a, const __grid_constant__ CUtensorMap tmq,
                    const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                    int tiles_per_seq, int five_d) {
  using TT = TcType<T>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  constexpr int kOffBar = off_bar<PREFIX>();
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffBar + 8 * kNumBars);
  volatile int *flags = reinterpret_cast<volatile int *>(tmem_slot + 1);  // [0] abort, [1] bad block
  const uint32_t sbase = smem_addr(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // K/V stage layout: key k, 64-column half h at (k / 8) * GS + h * HS + (k % 8) * 128.
  // 5-D boxes: [8-key group][half][8 rows] (GS 2 KB, HS 1 KB); 2-D boxes (one
  // per block and half): [half][key] (GS 1 KB, HS 16 KB).
  const uint32_t GS = five_d ? 2048u : 1024u;
  const uint32_t HS = five_d ? 1024u : (uint32_t)(kKeys * 128);
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // ---- the CTA's rows: tokens t0 .. t0 + ntok - 1 of the sequence's chunk --
  // (prefix mode: members q0 .. q0 + ntok - 1 of the group, one row each)
  const int G = a.group;
  const int TPT = kRows / G;  // tokens (members) per Q tile
  const int tile = blockIdx.x % tiles_per_seq;
  const int rest = blockIdx.x / tiles_per_seq;
  const int kvh = rest % a.num_kv_heads;
  int seq, q0, Q, t0, ntok, L;
  if constexpr (PREFIX) {
    const int jg = rest / a.num_kv_heads;
    const int s0 = a.grp_start[jg], s1 = a.grp_start[jg + 1], P = a.grp_blocks[jg];
    const int m0 = s0 + tile * kQTiles * TPT;
    // CTA-uniform exits, before any barrier (malformed groups are reported by the decode kernel)
    if (!(0 <= s0 && s0 <= s1 && s1 <= a.num_seqs && 0 < P && P <= a.max_blocks_per_seq && m0 < s1))
      return;
    seq = s0;  // the group's first sequence: its table holds the shared blocks
    q0 = m0;   // one decode row per member: q row = sequence index
    Q = 1;     // with t0 = 0 every row sees keys 0 .. L-1 (no causal mask)
    t0 = 0;
    ntok = min(kQTiles * TPT, s1 - m0);
    L = P * BS;
  } else {
    seq = a.seq_begin + rest / a.num_kv_heads;
    q0 = a.query_start_loc[seq];
    Q = a.query_start_loc[seq + 1] - q0;
    if (Q <= 1 || q0 < 0 || q0 + Q > a.num_q_tokens) return;  // CTA-uniform exits, before any barrier
    if (Q > a.max_query_len) {
      if (tid == 0 && tile == 0) raise_error(a.err, PA_DEVERR_QUERY_LEN);
      return;
    }
    t0 = tile * kQTiles * TPT;
    if (t0 >= Q) return;
    ntok = min(kQTiles * TPT, Q - t0);
    L = a.context_lens[seq];
    if (L < Q || L > a.max_context_len) {
      if (tid == 0 && tile == 0 && kvh == 0)
        raise_error(a.err, (L < 0 || L > a.max_context_len) ? PA_DEVERR_CONTEXT_LEN : PA_DEVERR_QUERY_LEN);
      for (int idx = tid; idx < ntok * G * kD; idx += blockDim.x) {
        const int r = idx / kD, dd = idx - r * kD;
        static_cast<T *>(a.out)[((int64_t)(q0 + t0 + r / G) * a.num_heads + kvh * G + r % G) * kD + dd] =
            Elem<T>::from_f(0.f);
      }
      return;
    }
  }
  const int nq = ntok > TPT ? 2 : 1;   // Q tiles holding rows of this CTA
  const int kend = L - Q + t0 + ntok;  // keys [0, kend) are visible to some row
  volatile unsigned char *bad_member = smem + kOffMemBad;
  const int ntiles = (kend + kKeys - 1) / kKeys;
  const int nblk = (L + BS - 1) / BS;

  // ---- set-up: barriers, TMEM ---------------------------------------------
  if (tid == 0) {
    mbar_init(&bars[kQFull], 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars[kKFull + s], 1);
      mbar_init(&bars[kVFull + s], 1);
      mbar_init(&bars[kKvEmpty + s], 1);
    }
    for (int t = 0; t < kQTiles; ++t) {
      mbar_init(&bars[kSFull + t], 1);
      mbar_init(&bars[kPFull + t], 4);
      mbar_init(&bars[kPvDone + t], 1);
    }
    mbar_init(&bars[kDone], 1);
    flags[0] = 0;
    flags[1] = 0;
    if constexpr (PREFIX)
      for (int i = 0; i < kQTiles * kRows; ++i) bad_member[i] = 0;
    mbar_init_fence();
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&](void) {
    if (!flags[0]) raise_error(a.err, PA_DEVERR_TIMEOUT);
    flags[0] = 1;
  };

  if (warp == kProducerWarp) {
    // ======================= producer =======================================
    // The warp reads the block table 32 ids at a time (one coalesced load, the
    // next group fetched while the current one is issued); lane 0 issues the
    // TMA loads: Q once, then per tile one K box and one V box per block.
    const int32_t *table = a.block_tables + (int64_t)seq * a.max_blocks_per_seq;
    if (lane == 0) {
      mbar_arrive_expect_tx(&bars[kQFull], nq * kQBytes);
      for (int t = 0; t < nq; ++t)
        for (int h = 0; h < 2; ++h)
          tma_load_4d(sbase + kOffQ + t * kQBytes + h * (kQBytes / 2), &tmq, h * 64, 0, kvh,
                      q0 + t0 + t * TPT, &bars[kQFull]);
    }
    constexpr int kBpt = kKeys / BS;  // blocks per tile (8 or 4; divides 32)
    int grp = 0;
    int ids = lane < nblk ? table[lane] : 0;
    int ids_next = 32 + lane < nblk ? table[32 + lane] : 0;
    int last_issued[kStages];
#pragma unroll
    for (int s = 0; s < kStages; ++s) last_issued[s] = -1;
    bool aborted = false;
    for (int j = 0; j < ntiles && !aborted; ++j) {
      const int st = j % kStages;
      const int b0 = j * kBpt;
      if (b0 >= grp + 32) {
        grp += 32;
        ids = ids_next;
        ids_next = grp + 32 + lane < nblk ? table[grp + 32 + lane] : 0;
      }
      const int nb = min(kBpt, nblk - b0);  // blocks of this tile inside the sequence
      int pbs[kBpt];
#pragma unroll
      for (int b = 0; b < kBpt; ++b) pbs[b] = __shfl_sync(0xffffffffu, ids, (b0 - grp + b) & 31);
      bool ok = !flags[0] && mbar_wait(&bars[kKvEmpty + st], ((j / kStages) & 1) ^ 1);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) fail();
        aborted = true;
        continue;
      }
      if (lane == 0) {
        const uint32_t kdst = sbase + kOffKV + st * kStageBytes;
        const uint32_t vdst = kdst + kHalfStage;
        const uint32_t bytes = nb * BS * kD * 2;
        mbar_arrive_expect_tx(&bars[kKFull + st], bytes);
        mbar_arrive_expect_tx(&bars[kVFull + st], bytes);
#pragma unroll
        for (int b = 0; b < kBpt; ++b) {
          if (b < nb && (pbs[b] < 0 || pbs[b] >= a.num_blocks)) {
            raise_error(a.err, PA_DEVERR_BLOCK_ID);
            flags[1] = 1;
            pbs[b] = 0;  // load a valid block; the CTA's rows are written as zeros
          }
        }
        if (five_d) {
#pragma unroll
          for (int b = 0; b < kBpt; ++b)
            if (b < nb)
              tma_load_5d(kdst + b * BS * kD * 2, &tmk, 0, 0, 0, 0, pbs[b] * a.num_kv_heads + kvh,
                          &bars[kKFull + st]);
#pragma unroll
          for (int b = 0; b < kBpt; ++b)
            if (b < nb)
              tma_load_5d(vdst + b * BS * kD * 2, &tmv, 0, 0, 0, 0, pbs[b] * a.num_kv_heads + kvh,
                          &bars[kVFull + st]);
        } else {
#pragma unroll
          for (int b = 0; b < kBpt; ++b)
            if (b < nb) {
              const int row = (pbs[b] * a.num_kv_heads + kvh) * BS;
              for (int h = 0; h < 2; ++h)
                tma_load_2d(kdst + h * HS + b * BS * 128, &tmk, h * 64, row, &bars[kKFull + st]);
            }
#pragma unroll
          for (int b = 0; b < kBpt; ++b)
            if (b < nb) {
              const int row = (pbs[b] * a.num_kv_heads + kvh) * BS;
              for (int h = 0; h < 2; ++h)
                tma_load_2d(vdst + h * HS + b * BS * 128, &tmv, h * 64, row, &bars[kVFull + st]);
            }
        }
#pragma unroll
        for (int s2 = 0; s2 < kStages; ++s2)
          if (s2 == st) last_issued[s2] = j;
      }
      __syncwarp();
    }
    // Before the CTA can exit, every copy this warp started must have landed
    // (an unwinding CTA's shared memory may be handed to the next CTA).
    if (lane == 0) {
      mbar_wait(&bars[kQFull], 0);
#pragma unroll
      for (int s = 0; s < kStages; ++s) {
        if (last_issued[s] < 0) continue;
        const uint32_t par = (last_issued[s] / kStages) & 1;
        if (!mbar_wait(&bars[kKFull + s], par) || !mbar_wait(&bars[kVFull + s], par)) fail();
      }
    }
  } else if (warp == kMmaWarp) {
    // ======================= MMA issue ======================================
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc(TT::kFmt, 0, 0, kRows, kKeys);
      constexpr uint32_t idesc_pv = umma_idesc(TT::kFmt, 0, 1, kRows, kD);
      // S_t(j) = Q_t K_j^T: both operands K-major; K rows of 8-key group g at
      // GS steps (SBO), the two 64-column halves HS apart
      auto issue_s = [&](int t, int j) {
        const uint32_t kst = sbase + kOffKV + (j % kStages) * kStageBytes;
        const uint32_t qst = sbase + kOffQ + t * kQBytes;
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
          const int h = ks >> 2, kk = ks & 3;
          const uint64_t da = umma_desc(qst + h * (kQBytes / 2) + kk * 32, 16, 1024);
          const uint64_t db = umma_desc(kst + h * HS + kk * 32, 16, GS);
          umma(tmem + tmem_s_col(t), da, db, idesc_s, ks > 0 ? 1u : 0u);
        }
        umma_commit(&bars[kSFull + t]);
      };
      // O_t += P_t(j) V_j: A = P from tensor memory (16 keys in 8 columns per
      // word kind), B = V MN-major (64-column atoms HS apart, 8-key groups GS)
      auto issue_pv = [&](int t, int j) {
        const uint32_t vst = sbase + kOffKV + (j % kStages) * kStageBytes + kHalfStage;
#pragma unroll
        for (int ks = 0; ks < kKeys / 16; ++ks) {
          const uint64_t db = umma_desc(vst + ks * 2 * GS, HS, GS);
          if constexpr (TT::kSplitP) {
            umma_ts(tmem + tmem_o_col(t), tmem + tmem_s_col(t) + ks * 16, db, idesc_pv,
                    (j > 0 || ks > 0) ? 1u : 0u);
            umma_ts(tmem + tmem_o_col(t), tmem + tmem_s_col(t) + ks * 16 + 8, db, idesc_pv, 1u);
          } else {
            umma_ts(tmem + tmem_o_col(t), tmem + tmem_s_col(t) + ks * 8, db, idesc_pv,
                    (j > 0 || ks > 0) ? 1u : 0u);
          }
        }
        umma_commit(&bars[kPvDone + t]);
      };
      bool ok = mbar_wait(&bars[kQFull], 0) && mbar_wait(&bars[kKFull], 0);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        if (nq > 1) issue_s(1, 0);
      } else {
        fail();
      }
      for (int j = 0; ok && j < ntiles && !flags[0]; ++j) {
        const int st = j % kStages;
        const uint32_t par = (uint32_t)(j & 1);
        const int jn = j + 1;
        const bool more = jn < ntiles;
        for (int t = 0; t < nq && ok; ++t) {
          // P V of this Q tile (V of the stage must have landed)
          ok = mbar_wait(&bars[kPFull + t], par) && (t > 0 || mbar_wait(&bars[kVFull + st], (j / kStages) & 1));
          if (!ok) break;
          tc_fence_after();
          issue_pv(t, j);
          if (t == nq - 1) umma_commit(&bars[kKvEmpty + st]);  // the stage is free once these finish
          if (more) {
            // S(j+1) overwrites P(j) of this Q tile: its P V must be complete
            ok = mbar_wait(&bars[kPvDone + t], par) &&
                 (t > 0 || mbar_wait(&bars[kKFull + (jn % kStages)], (jn / kStages) & 1));
            if (!ok) break;
            tc_fence_after();
            issue_s(t, jn);
          }
        }
        if (!ok) fail();
      }
      umma_commit(&bars[kDone]);  // completes when every MMA above has finished
      if (!mbar_wait(&bars[kDone], 0)) fail();
    }
  } else {
    // ======================= softmax warps =================================
    const int qt = warp >> 2, qd = warp & 3;
    const int r = qd * 32 + lane;  // row of the Q tile = TMEM lane
    if (qt < nq) {
      const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
      const uint32_t ts = tmem + tmem_s_col(qt) + lane_off;
      const uint32_t to = tmem + tmem_o_col(qt) + lane_off;
      const int tok = qt * TPT + r / G;                     // token among the CTA's rows
      const int limit = min(L - Q + t0 + tok, L - 1);       // last key this row may see
      const int limit_lo = L - Q + t0 + qt * TPT;           // the tile's smallest limit
      const float sl2 = a.scale_log2;
      if constexpr (PREFIX) {
        // Every member's table must hold the group's ids over the shared
        // range.  All of the checks' loads are issued together here, while the
        // first tile is in flight, instead of one dependent round trip per tile.
        const int32_t *table = a.block_tables + (int64_t)seq * a.max_blocks_per_seq;
        const int sid = qt * kRows + r;  // 0 .. nq*128 - 1
        const int nth = nq * kRows;
        for (int x0 = sid; x0 < ntok * nblk; x0 += nth * 8) {
          int mine[8], ref[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int x = x0 + u * nth;
            const int i = x / nblk, b = x - i * nblk;
            mine[u] = x < ntok * nblk ? a.block_tables[(int64_t)(q0 + i) * a.max_blocks_per_seq + b] : 0;
            ref[u] = x < ntok * nblk ? table[b] : 0;
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int x = x0 + u * nth;
            if (x < ntok * nblk && mine[u] != ref[u]) {
              const int i = x / nblk;
              if (!bad_member[i]) raise_error(a.err, PA_DEVERR_PREFIX);
              bad_member[i] = 1;
            }
          }
        }
      }
      float m_used = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = 0; j < ntiles; ++j) {
        ok = !flags[0] && mbar_wait(&bars[kSFull + qt], (uint32_t)(j & 1));
        if (!__all_sync(0xffffffffu, ok)) { ok = false; fail(); break; }  // tcgen05.ld is collective
        tc_fence_after();
        // Pass 1: row max over the tile's S columns, 32 at a time (the next
        // chunk's load is in flight while this one is reduced).  Keys past
        // the row's causal limit are masked, in the tiles that reach past the
        // Q tile's smallest limit only (warp-uniform branch).
        const int k0 = j * kKeys;
        const bool masked = k0 + kKeys - 1 > limit_lo;
        float mx = -INFINITY;
        {
          uint32_t ca[32], cb[32];
          tmem_ld32(ts, ca);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < kKeys / 32; ++c) {
            uint32_t (&cur)[32] = (c & 1) ? cb : ca;
            uint32_t (&nxt)[32] = (c & 1) ? ca : cb;
            if (c + 1 < kKeys / 32) tmem_ld32(ts + 32 * (c + 1), nxt);
            if (masked) {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (k0 + 32 * c + i > limit) cur[i] = __float_as_uint(-INFINITY);
            }
#pragma unroll
            for (int i = 0; i < 32; i += 2) mx = fmax3(mx, __uint_as_float(cur[i]), __uint_as_float(cur[i + 1]));
            tmem_wait_ld();
          }
        }
        mx *= sl2;
        // lazy rescale: move the reference max only when the tile max exceeds
        // it by more than 2^8 (first tile: always).  O_t is quiescent here: S_t(j)
        // was issued after P V of tile j-1 completed.
        const bool need = mx > m_used + kRescaleThreshold;
        float alpha = 1.f;
        if (need) {
          alpha = m_used == -INFINITY ? 0.f : fast_exp2(m_used - mx);
          m_used = mx;
          l *= alpha;
        }
        if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll 1
          for (int c = 0; c < kD / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(to + 32 * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(to + 32 * c, o);
          }
        }
        // Pass 2: P = 2^(s*scale*log2e - m), chunk by chunk over the same
        // columns (next chunk prefetched); chunk c's P words go over S columns
        // the pass has already read (bf16: [32c, 32c+32), fp16: [16c, 16c+16)).
        // Key pairs are computed with packed f32x2 arithmetic.
        const float2 sl2x2 = make_float2(sl2, sl2);
        const float2 negx2 = make_float2(-m_used, -m_used);
        float2 psum2 = make_float2(0.f, 0.f);
#pragma unroll 1
        for (int cp = 0; cp < kKeys / 64; ++cp) {  // pairs of 32-column chunks
          uint32_t ca[32], cb[32];
          tmem_ld32(ts + 64 * cp, ca);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int c = 2 * cp + h;
            uint32_t (&cur)[32] = h ? cb : ca;
            if (h == 0) tmem_ld32(ts + 64 * cp + 32, cb);  // lands while chunk 2cp is computed
            if (masked) {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (k0 + 32 * c + i > limit) cur[i] = __float_as_uint(-INFINITY);
            }
            uint32_t w[16];
#pragma unroll
            for (int g2 = 0; g2 < 2; ++g2) {
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int kk = 16 * g2 + 2 * i;  // key within the chunk
                const float2 x = make_float2(__uint_as_float(cur[kk]), __uint_as_float(cur[kk + 1]));
                const float2 t = __ffma2_rn(x, sl2x2, negx2);
                const float2 pp = make_float2(fast_exp2(t.x), fast_exp2(t.y));
                psum2 = __fadd2_rn(psum2, pp);
                const uint32_t hi = TT::pack(pp.x, pp.y);
                if constexpr (TT::kSplitP) {
                  // 16 keys: 8 hi words then 8 lo words (columns 16g .. 16g+15)
                  const float2 hv = TT::unpack(hi);
                  const float2 rv = __ffma2_rn(hv, make_float2(-1.f, -1.f), pp);  // p - hi
                  w[i] = hi;
                  w[8 + i] = TT::pack(rv.x, rv.y);
                } else {
                  w[8 * g2 + i] = hi;  // 16 keys: 8 words (columns 8g .. 8g+7)
                }
              }
              if constexpr (TT::kSplitP) tmem_st16(ts + 32 * c + 16 * g2, w);
            }
            if constexpr (!TT::kSplitP) tmem_st16(ts + 16 * c, w);
            tmem_wait_ld();
          }
        }
        const float psum = psum2.x + psum2.y;
        tmem_wait_st();
        l += psum;
        // keys past the context end in the sequence's last tile: zero their V
        // rows (P is 0 there, but the slots may hold anything and 0 * NaN is
        // NaN).  Q tile 0's warps do it before P V of either tile is issued;
        // the stage's bytes have all landed (S(j) waited for K, and V is
        // waited for below).
        if (qt == 0 && (j + 1) * kKeys > L) {
          const int st = j % kStages;
          if (mbar_wait(&bars[kVFull + st], (uint32_t)((j / kStages) & 1))) {
            const uint32_t vst = sbase + kOffKV + st * kStageBytes + kHalfStage;
            const int z0 = L - j * kKeys;       // first stale key of the tile
            const int nz = (kKeys - z0) * 16;   // 16-byte chunks over both halves
            for (int c = r; c < nz; c += 128) {
              const int key = z0 + c / 16, ch = c % 16;
              const int h = ch >> 3, cc = ch & 7, kr = key & 7;
              st_shared_v4(vst + (key >> 3) * GS + h * HS + kr * 128 + ((cc ^ kr) << 4), 0, 0, 0, 0);
            }
          } else {
            fail();
          }
          fence_proxy_async_smem();  // generic-proxy writes -> tensor-core reads
        }
        tc_fence_before();  // the tcgen05.st of P -> the MMA thread
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kPFull + qt]);
      }
      // ---- epilogue: O / l -> out ----
      const uint32_t lastp = (uint32_t)((ntiles - 1) & 1);
      bool fin = ok && !flags[0] && ntiles > 0 && mbar_wait(&bars[kPvDone + qt], lastp);
      fin = __all_sync(0xffffffffu, fin);
      if (!fin && ntiles > 0) fail();
      tc_fence_after();
      const bool write = tok < ntok;
      if constexpr (PREFIX) {
        // the member flags of every active softmax warp (named barrier 1)
        named_sync(1, nq * kRows);
        // record of (member q0 + tok, head): o unnormalised, the reference max
        // (base 2) o and l are relative to, l; NaN l marks a poisoned record
        const bool poison = !fin || flags[1] || (write && bad_member[tok]);
        float *rec = a.pre_rec + ((int64_t)(q0 + tok) * a.num_heads + kvh * G + r % G) * (kD + 4);
#pragma unroll 1
        for (int c = 0; c < kD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(to + 32 * c, o);
          tmem_wait_ld();
          if (write) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4 *>(rec + 32 * c + i) =
                  make_float4(__uint_as_float(o[i]), __uint_as_float(o[i + 1]), __uint_as_float(o[i + 2]),
                              __uint_as_float(o[i + 3]));
          }
        }
        if (write) {
          rec[kD] = m_used;
          rec[kD + 1] = poison ? __int_as_float(0x7fc00000) : l / a.o_scale;
        }
        tc_fence_before();
      } else {
      const float inv = (fin && l > 0.f && !flags[1]) ? (1.f / l) * a.o_scale : 0.f;
      T *dst = static_cast<T *>(a.out) + ((int64_t)(q0 + t0 + tok) * a.num_heads + kvh * G + r % G) * kD;
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(to + 32 * c, o);
        tmem_wait_ld();
        if (write) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 v;
            v.x = TT::pack(__uint_as_float(o[i + 0]) * inv, __uint_as_float(o[i + 1]) * inv);
            v.y = TT::pack(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
            v.z = TT::pack(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv);
            v.w = TT::pack(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv);
            *reinterpret_cast<uint4 *>(dst + 32 * c + i) = v;
          }
        }
      }
      tc_fence_before();
      }
    }
  }
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512)
                 : "memory");
  }
}

template <typename T, int BS, bool PREFIX>
cudaError_t launch_pp_t(const AttnArgs &a, cudaStream_t stream) {
  auto fn = encode_fn_tc();
  if (!fn) return cudaErrorNotSupported;
  const int G = a.group;
  const int TPT = kRows / G;
  CUtensorMap tmq, tmk, tmv;
  {  // q viewed as [tokens][Hk][G][D]; box = TPT tokens x G heads x 64 columns
    cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)G, (cuuint64_t)a.num_kv_heads,
                          (cuuint64_t)a.num_q_tokens};
    cuuint64_t strides[3] = {(cuuint64_t)kD * 2, (cuuint64_t)G * kD * 2, (cuuint64_t)a.num_heads * kD * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)G, 1, (cuuint32_t)TPT};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(&tmq, TcType<T>::kTma, 4, const_cast<void *>(a.q), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
      debug_log("chunk_pp: Q tensor map refused (CUresult %d)", (int)r);
      return cudaErrorInvalidValue;
    }
  }
  // K/V: one box per (block, KV head) through a 5-D view whose half-of-row
  // dimension sits between the rows and the 8-row groups (when asked for and
  // the driver accepts the view), else two 2-D boxes per block (one per
  // 64-column half).
  // Two 2-D boxes per block unless PA_CHUNK_PP_BOXES=5d: on the long mixed
  // batch the whole call measured 1.382 ms with two boxes and 1.393 ms with
  // one -- the box rate does not bound this kernel.
  const char *boxes = getenv("PA_CHUNK_PP_BOXES");
  int five_d = (boxes && strcmp(boxes, "5d") == 0) ? 1 : 0;
  for (int i = 0; i < 2 && five_d; ++i) {
    // a cache viewed as [block x kv head][row group][half][8 rows][64 columns]
    // (innermost first below): one box = one (block, kv head) tile, landing
    // as [row group][half][8 rows][128 B]
    cuuint64_t dims[5] = {64, 8, 2, (cuuint64_t)(BS / 8), (cuuint64_t)a.num_blocks * a.num_kv_heads};
    cuuint64_t strides[4] = {(cuuint64_t)kD * 2, 128, (cuuint64_t)8 * kD * 2, (cuuint64_t)BS * kD * 2};
    cuuint32_t box[5] = {64, 8, 2, (cuuint32_t)(BS / 8), 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    const CUresult r = fn(i ? &tmv : &tmk, TcType<T>::kTma, 5, const_cast<void *>(i ? a.v_cache : a.k_cache),
                          dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
      debug_log("chunk_pp: 5-D K/V tensor map refused (CUresult %d); two 2-D boxes per block", (int)r);
      five_d = 0;
    }
  }
  if (!five_d) {
    for (int i = 0; i < 2; ++i) {
      cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)a.num_blocks * a.num_kv_heads * BS};
      cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
      cuuint32_t box[2] = {64, (cuuint32_t)BS};
      cuuint32_t estr[2] = {1, 1};
      const CUresult r = fn(i ? &tmv : &tmk, TcType<T>::kTma, 2, const_cast<void *>(i ? a.v_cache : a.k_cache),
                            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r != CUDA_SUCCESS) {
        debug_log("chunk_pp: 2-D K/V tensor map refused (CUresult %d)", (int)r);
        return cudaErrorInvalidValue;
      }
    }
  }
  auto kern = chunk_pp_kernel<T, BS, PREFIX>;
  constexpr int kSmemBytes = smem_bytes<PREFIX>();
  {
    cudaError_t e = set_smem_limit_once(reinterpret_cast<const void *>(kern), kSmemBytes, true);
    if (e != cudaSuccess) {
      debug_log("chunk_pp: shared-memory limit %d refused: %s", kSmemBytes, cudaGetErrorString(e));
      return e;
    }
  }
  // chunk rows: (sequence, KV head, pair of Q tiles); prefix: (group, KV
  // head, pair of member tiles)
  const int rows = PREFIX ? a.max_group : a.max_query_len;
  const int tiles = (rows + kQTiles * TPT - 1) / (kQTiles * TPT);
  const int64_t grid = (int64_t)(PREFIX ? a.num_groups : a.num_seqs) * a.num_kv_heads * tiles;
  if (grid == 0) return cudaSuccess;
  if (grid > 0x7fffffff) return cudaErrorInvalidValue;
  kern<<<(unsigned)grid, kThreads, kSmemBytes, stream>>>(a, tmq, tmk, tmv, tiles, five_d);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) debug_log("chunk_pp: launch failed: %s", cudaGetErrorString(e));
  return e;
}

}  // namespace

bool chunk_pp_supported(const AttnArgs &a, int dtype) {
  return (dtype == PA_BF16 || dtype == PA_F16) && a.head_dim == kD && a.group >= 1 &&
         a.group <= kRows && kRows % a.group == 0 && (a.block_size == 16 || a.block_size == 32) &&
         encode_fn_tc() != nullptr;
}

cudaError_t launch_chunk_pp(const AttnArgs &a, int dtype, cudaStream_t stream) {
  if (dtype == PA_BF16)
    return a.block_size == 16 ? launch_pp_t<__nv_bfloat16, 16, false>(a, stream)
                              : launch_pp_t<__nv_bfloat16, 32, false>(a, stream);
  return a.block_size == 16 ? launch_pp_t<__half, 16, false>(a, stream)
                            : launch_pp_t<__half, 32, false>(a, stream);
}

cudaError_t launch_prefix_pp(const AttnArgs &a, int dtype, cudaStream_t stream) {
  if (dtype == PA_BF16)
    return a.block_size == 16 ? launch_pp_t<__nv_bfloat16, 16, true>(a, stream)
                              : launch_pp_t<__nv_bfloat16, 32, true>(a, stream);
  return a.block_size == 16 ? launch_pp_t<__half, 16, true>(a, stream)
                            : launch_pp_t<__half, 32, true>(a, stream);
}

}  // namespace pa
