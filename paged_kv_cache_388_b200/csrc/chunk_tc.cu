// chunk_tc.cu -- chunked-prefill attention on the 5th-generation tensor cores.
//
// A chunk of Q > 1 query tokens of one sequence attends causally over the
// sequence's paged KV (row t sees keys 0 .. L-Q+t; "PagedAttention 实战",
// section Chunked Prefill).  Per (sequence, KV head) the GROUP query heads of
// every token read the same K/V, so a 128-row tile (128/GROUP tokens x GROUP
// heads) against 64-key tiles is a dense contraction: S = Q K^T
// (128x64x128) and O += P V (128x128x64) run as tcgen05.mma with fp32
// accumulators in tensor memory.
//
// CTA = (sequence, KV head, NQ tiles of 128 query rows); 4 * kHalves * NQ + 2
// warps (NQ = 2 for chunk rows: the two Q tiles share every K/V tile, which
// halves the TMA boxes per row -- a B200 SM's TMA unit spends ~100 cycles per
// 2 KB box, and a 64-key bs-16 tile is 16 of them):
//   softmax    warps of Q tile t (and w + 4 when kHalves = 2) own rows 32w ..
//              32w+31 of the tile (TMEM lane quadrant w), each taking
//              64 / kHalves of every K tile's keys and 128 / kHalves of O's
//              columns.  Reads S from TMEM, masks, exchanges the tile row max
//              with its partner (two halves), keeps a running max that is
//              only moved (and O rescaled in TMEM) when the tile max exceeds
//              it by more than 2^8, writes P = 2^(s - m) as bf16 hi + lo (or
//              fp16) over its S columns in TMEM, and at the end writes O / l.
//   producer   TMA loads of Q (once) and of each 64-key K/V tile, block by
//              block through the block table (128-byte swizzle).
//   MMA        (the last warp) MMA issue (one elected thread) and TMEM
//              allocation.
// TMEM per Q tile: S/P buffers of 64 columns (3 with one Q tile, 2 with two)
// and O (128 columns).  Shared memory: Q 32 KB per tile, kStagesTC K/V stages
// of 32 KB.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "tc_common.cuh"

namespace pa {
namespace {

constexpr int kRowsTC = 128;   // query rows per CTA (MMA M)
constexpr int kKeysTC = 64;    // keys per tile (MMA N of S, K of P.V)
constexpr int kHeadDim = 128;
// P in tensor memory: the softmax writes P (bf16 hi + lo, or fp16) over its
// tile's S columns and P V reads it from there as the A operand, instead of
// P going through shared memory (generic stores, a proxy fence, and the
// tensor core reading it back).  Three S/P buffers in TMEM then let S(j) be
// issued while P(j-1) and P(j-2) are still to be consumed.
#ifndef PA_CHUNK_TC_PTMEM
#define PA_CHUNK_TC_PTMEM 1
#endif
constexpr bool kPTmem = PA_CHUNK_TC_PTMEM != 0;
#ifndef PA_CHUNK_TC_STAGES
#define PA_CHUNK_TC_STAGES (PA_CHUNK_TC_PTMEM ? 4 : 3)
#endif
constexpr int kStagesTC = PA_CHUNK_TC_STAGES;  // K/V tiles in flight
// Softmax warps per row quadrant: each of the kHalves warps that share 32 rows
// (TMEM lanes) takes kKeysTC / kHalves keys of every tile and kHeadDim /
// kHalves columns of O; with two, the pair exchanges its tile row maxima and,
// at the end, its row sums through shared memory.  Measured on B200 (long
// mixed batch, 4 chunks of 512 rows over 16K-token prefixes): 2.06 ms with
// one warp per quadrant, 2.10 ms with two -- the softmax warps are not what
// bounds the kernel -- so one is the default.
#ifndef PA_CHUNK_TC_HALVES
#define PA_CHUNK_TC_HALVES 1
#endif
constexpr int kHalves = PA_CHUNK_TC_HALVES;
// Warps of a CTA (see chunk_tc_kernel): 4 * kHalves softmax warps per Q tile,
// then one TMA producer warp and one MMA-issue / TMEM-allocation warp.
// Q tiles of 128 rows per chunk-row CTA (1 or 2; see chunk_tc_kernel)
#ifndef PA_CHUNK_TC_NQ
#define PA_CHUNK_TC_NQ 2
#endif
constexpr int kChunkQTiles = PA_CHUNK_TC_NQ;
constexpr int kKeysPerHalf = kKeysTC / kHalves;
constexpr int kOColsPerHalf = kHeadDim / kHalves;
static_assert(kHalves == 1 || kHalves == 2, "one or two softmax warps per row quadrant");
// P buffers in shared memory (PA_CHUNK_TC_PTMEM=0): tile j's softmax writes
// buffer j % kPBufs once tile j - kPBufs's P.V has read it.  Measured on B200
// (long mixed batch, whole call): P in TMEM 1.717 ms vs 1.742 ms through
// shared memory; 3 / 4 / 5 K/V stages 1.729 / 1.717 / 1.717 ms; a second
// softmax warp per row quadrant 1.735 ms; separate K and V rings (V trailing
// K by a tile) 2.05-2.18 ms.  A tile takes about 2300 cycles, of which the
// MMA thread spends about 1550 issuing its 16 tcgen05.mma (the tensor pipe
// runs these M=128, N=64/128, K=16 shapes at about half its peak rate) and
// the softmax warps about 1700: the chain S -> softmax -> P V, not the
// loads, sets the pace.
#ifndef PA_CHUNK_TC_PBUFS
#define PA_CHUNK_TC_PBUFS 2
#endif
#ifndef PA_CHUNK_TC_SBUFS
#define PA_CHUNK_TC_SBUFS (PA_CHUNK_TC_PTMEM ? 3 : 2)
#endif
constexpr int kSBufs = PA_CHUNK_TC_SBUFS;                // S (and with kPTmem P) buffers in TMEM
#ifndef PA_CHUNK_TC_MIN_CTAS
#define PA_CHUNK_TC_MIN_CTAS 1
#endif
constexpr int kPBufs = kPTmem ? kSBufs : PA_CHUNK_TC_PBUFS;
constexpr uint32_t kTmemO = kSBufs * 64 <= 128 ? 128 : 256;  // O's first column
constexpr uint32_t kTmemCols = kTmemO + 128 <= 256 ? 256 : 512;  // allocation: a power of two
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P stays <= 2^8 between rescales

// ---- shared-memory layout (offsets from a 1024-byte aligned base) ---------
template <int NQ>
struct TcLayoutT {
  static constexpr int kQ = 0;                                   // NQ tiles x 2 halves x [128 rows x 128 B]
  static constexpr int kKV = kQ + NQ * kRowsTC * kHeadDim * 2;   // stages: K (2x8 KB) + V (2x8 KB)
  static constexpr int kStageBytes = 2 * kKeysTC * kHeadDim * 2;
  static constexpr int kP = kKV + kStagesTC * kStageBytes;       // 2 buffers x (hi, lo) x [128 x 128 B]
  static constexpr int kPBuf = 2 * kRowsTC * kKeysTC * 2;
  // row-max exchange [2 buffers][kHalves][128] and row-sum exchange [kHalves][128] floats
  static constexpr int kX = kP + (kPTmem ? 0 : kPBufs * kPBuf);
  static constexpr int kXBytes = 3 * kHalves * kRowsTC * 4;
  static constexpr int kMemBad = kX + kXBytes;   // prefix mode: [128] member-table mismatch flags
  static constexpr int kBar = kMemBad + 128;
  static_assert(kBar + 512 + 1024 <= 227 * 1024, "shared memory per CTA");
  static constexpr int kBytes = kBar + 512 + 1024;               // barriers etc. + alignment slack
};

// barrier indices within the barrier block; per-(Q tile, buffer) arrays hold
// up to two Q tiles of kSBufs buffers
constexpr int kSlots = 2 * (kSBufs > kPBufs ? kSBufs : kPBufs);
enum {
  kQFull = 0,
  kKvFull = 1,                       // [kStagesTC]
  kKvEmpty = kKvFull + kStagesTC,    // [kStagesTC]
  kSFull = kKvEmpty + kStagesTC,     // [Q tile][buffer] (kSlots)
  kSFree = kSFull + kSlots,          // (P in shared memory only)
  kPFull = kSFree + kSlots,          // [Q tile][buffer]
  kPvDone = kPFull + kSlots,         // [Q tile][buffer]
  kDone = kPvDone + kSlots,
  kXFull = kDone + 1,                // [4 quadrants][2 buffers] row maxima written
  kLFull = kXFull + 8,               // [4 quadrants] row sums written
  kNumBars = kLFull + 4
};

// PREFIX: the shared-prefix pass of pa_decode_shared_prefix.  The CTA is
// (group, chunk of 128/GROUP members, KV head); its rows are the members'
// decode rows (consecutive sequences, so the same 4-D view of q serves), its
// keys the group's shared blocks read through the group's first table, with
// no causal mask; the softmax warps check every member's table against those
// ids while the first tile loads; the
// output is one record (o unnormalised, reference max in base 2, sum) per
// (member, head) for the decode kernel to fold in.
//
// NQ = 2 (chunk rows): the CTA holds two 128-row Q tiles of the same
// (sequence, KV head) against one stream of K/V tiles, so every K/V box the
// TMA unit moves serves 256 rows; each Q tile has its own 4 softmax warps,
// its own 2 S/P buffers and O in TMEM (2 x 128 + 2 x 128 = 512 columns).
template <typename T, int BS, bool PREFIX = false, int NQ = 1>
__global__ void __launch_bounds__(32 * (4 * kHalves * NQ + 2), PA_CHUNK_TC_MIN_CTAS)
    chunk_tc_kernel(const AttnArgs a, const __grid_constant__ CUtensorMap tmq,
                    const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                    int tiles_per_seq) {
  using TT = TcType<T>;
  using LY = TcLayoutT<NQ>;
  static_assert(NQ == 1 || (NQ == 2 && kHalves == 1 && kPTmem && !PREFIX),
                "two Q tiles: chunk rows, P in TMEM, one softmax warp per lane quadrant");
  constexpr int SWT = 4 * kHalves;                      // softmax warps per Q tile
  constexpr int SW = SWT * NQ;                          // softmax warps
  constexpr int PW = SW, MW = SW + 1;                   // producer, MMA warps
  constexpr int SB = NQ == 1 ? kSBufs : 2;              // S (/P) buffers per Q tile
  constexpr int PB = kPTmem ? SB : kPBufs;              // P buffers per Q tile
  constexpr uint32_t OB = NQ == 1 ? kTmemO : 256;       // first O column (tile t: OB + 128 t)
  constexpr uint32_t TCOLS = NQ == 1 ? kTmemCols : 512;
  static_assert(NQ * SB <= kSlots && NQ * PB <= kSlots, "barrier slots");
  constexpr int D = kHeadDim;
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + LY::kBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + LY::kBar + 8 * kNumBars);
  volatile int *flags = reinterpret_cast<volatile int *>(tmem_slot + 1);  // [0] abort, [1] bad block
  const uint32_t sbase = smem_addr(smem);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  asm volatile("griddepcontrol.wait;" ::: "memory");

  const int G = a.group;
  const int TPT = kRowsTC / G;
  // The CTA's work: rows (query token or member, head) q0 + t0 .., the
  // sequence whose table holds the keys, the keys [0, kend) some row sees.
  int kvh, seq, q0, Q, t0, ntok, L, kend;
  if constexpr (PREFIX) {
    const int chunk = blockIdx.x % tiles_per_seq;  // member chunk
    const int rest = blockIdx.x / tiles_per_seq;
    kvh = rest % a.num_kv_heads;
    const int jg = rest / a.num_kv_heads;
    const int s0 = a.grp_start[jg], s1 = a.grp_start[jg + 1], P = a.grp_blocks[jg];
    const int m0 = s0 + chunk * TPT;
    // CTA-uniform exits, before any barrier
    if (!(0 <= s0 && s0 <= s1 && s1 <= a.num_seqs && 0 < P && P <= a.max_blocks_per_seq && m0 < s1))
      return;
    seq = s0;        // the group's first sequence: its table holds the shared blocks
    q0 = m0;         // one decode row per member: q row = sequence index
    Q = 1;
    t0 = 0;
    ntok = min(TPT, s1 - m0);
    L = P * BS;      // every row sees every shared key
    kend = L;
  } else {
    const int tile = blockIdx.x % tiles_per_seq;
    const int rest = blockIdx.x / tiles_per_seq;
    kvh = rest % a.num_kv_heads;
    seq = a.seq_begin + rest / a.num_kv_heads;
    q0 = a.query_start_loc[seq];
    Q = a.query_start_loc[seq + 1] - q0;
    if (Q <= 1 || q0 < 0 || q0 + Q > a.num_q_tokens) return;  // CTA-uniform exits, before any barrier
    if (Q > a.max_query_len) {
      if (tid == 0 && tile == 0) raise_error(a.err, PA_DEVERR_QUERY_LEN);
      return;
    }
    t0 = tile * NQ * TPT;
    if (t0 >= Q) return;
    ntok = min(NQ * TPT, Q - t0);  // rows of all Q tiles
    L = a.context_lens[seq];
    if (L < Q || L > a.max_context_len) {
      if (tid == 0 && tile == 0 && kvh == 0)
        raise_error(a.err, (L < 0 || L > a.max_context_len) ? PA_DEVERR_CONTEXT_LEN : PA_DEVERR_QUERY_LEN);
      for (int idx = tid; idx < ntok * G * D; idx += blockDim.x) {
        const int r = idx / D, dd = idx - r * D;
        static_cast<T *>(a.out)[((int64_t)(q0 + t0 + r / G) * a.num_heads + kvh * G + r % G) * D + dd] =
            Elem<T>::from_f(0.f);
      }
      return;
    }
    kend = L - Q + t0 + ntok;                      // keys [0, kend) visible to some row
  }
  const int ntiles = (kend + kKeysTC - 1) / kKeysTC;
  const int nblk = (L + BS - 1) / BS;              // blocks that hold the keys
  volatile unsigned char *bad_member = smem + LY::kMemBad;

  // ---- set-up: barriers, TMEM ------------------------------------------------
  if (tid == 0) {
    mbar_init(&bars[kQFull], 1);
    for (int s = 0; s < kStagesTC; ++s) {
      mbar_init(&bars[kKvFull + s], 1);
      mbar_init(&bars[kKvEmpty + s], 1);
    }
    for (int b = 0; b < NQ * SB; ++b) {
      mbar_init(&bars[kSFull + b], 1);
      mbar_init(&bars[kSFree + b], SWT);
    }
    for (int b = 0; b < NQ * PB; ++b) {
      mbar_init(&bars[kPFull + b], SWT);
      mbar_init(&bars[kPvDone + b], 1);
    }
    mbar_init(&bars[kDone], 1);
    for (int b = 0; b < 8; ++b) mbar_init(&bars[kXFull + b], 32 * kHalves);
    for (int b = 0; b < 4; ++b) mbar_init(&bars[kLFull + b], 32 * kHalves);
    flags[0] = 0;
    for (int i = 0; i < 128; ++i) bad_member[i] = 0;
    flags[1] = 0;
    mbar_init_fence();
  }
  if (warp == MW) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(TCOLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM: Q tile t's S/P buffers at columns t*SB*64 .., its O at OB + 128 t

  auto fail = [&](void) {
    if (!flags[0]) raise_error(a.err, PA_DEVERR_TIMEOUT);
    flags[0] = 1;
  };

  if (warp == PW) {
    // ======================= producer =======================================
    // The whole warp reads the block table 32 ids at a time (one coalesced
    // load, the next group fetched while the current one is issued); lane 0
    // issues the TMA loads.
    const int32_t *table = a.block_tables + (int64_t)seq * a.max_blocks_per_seq;
    if (lane == 0) {
      // Q: 128 rows (token, head) per Q tile, two 64-column boxes each
      mbar_arrive_expect_tx(&bars[kQFull], NQ * kRowsTC * D * 2);
      for (int t = 0; t < NQ; ++t)
        for (int h = 0; h < 2; ++h)
          tma_load_4d(sbase + LY::kQ + t * kRowsTC * D * 2 + h * kRowsTC * 128, &tmq, h * 64, 0, kvh,
                      q0 + t0 + t * TPT, &bars[kQFull]);
    }
    constexpr int kBpt = kKeysTC / BS;  // blocks per tile
    int grp = 0;                        // first block of the group held in `ids`
    int ids = lane < nblk ? table[lane] : 0;
    int ids_next = 32 + lane < nblk ? table[32 + lane] : 0;
    bool aborted = false;
    uint32_t issued = 0;  // tiles whose loads were issued
    for (int j = 0; j < ntiles && !aborted; ++j) {
      const int st = j % kStagesTC;
      const int b0 = j * kBpt;
      if (b0 >= grp + 32) {  // next group of 32 block ids
        grp += 32;
        ids = ids_next;
        ids_next = grp + 32 + lane < nblk ? table[grp + 32 + lane] : 0;
      }
      const int nb = min(kBpt, nblk - b0);  // blocks of this tile inside the sequence
      int pbs[kBpt];
#pragma unroll
      for (int b = 0; b < kBpt; ++b) pbs[b] = __shfl_sync(0xffffffffu, ids, (b0 - grp + b) & 31);
      bool ok = !flags[0] && mbar_wait(&bars[kKvEmpty + st], ((j / kStagesTC) & 1) ^ 1);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) fail();
        aborted = true;
        continue;
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(&bars[kKvFull + st], nb * 2 * BS * D * 2);
        const uint32_t kdst = sbase + LY::kKV + st * LY::kStageBytes;
        const uint32_t vdst = kdst + LY::kStageBytes / 2;
        for (int b = 0; b < nb; ++b) {
          int pb = pbs[b];
          if (pb < 0 || pb >= a.num_blocks) {
            raise_error(a.err, PA_DEVERR_BLOCK_ID);
            flags[1] = 1;
            pb = 0;  // load a valid block; the tile's rows are written as zeros
          }
          const int row = (pb * a.num_kv_heads + kvh) * BS;
          for (int h = 0; h < 2; ++h) {
            tma_load_2d(kdst + h * kKeysTC * 128 + b * BS * 128, &tmk, h * 64, row, &bars[kKvFull + st]);
            tma_load_2d(vdst + h * kKeysTC * 128 + b * BS * 128, &tmv, h * 64, row, &bars[kKvFull + st]);
          }
        }
      }
      issued = j + 1;
      __syncwarp();
    }
    // the copies this warp started land before the CTA may exit
    if (lane == 0 && !(drain_ring(&bars[kKvFull], kStagesTC, issued) & drain_ring(&bars[kQFull], 1, 1)))
      fail();
  } else if (warp == MW) {
    // ======================= MMA issue ======================================
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc(TT::kFmt, 0, 0, kRowsTC, kKeysTC);
      constexpr uint32_t idesc_pv = umma_idesc(TT::kFmt, 0, 1, kRowsTC, D);
      bool ok = mbar_wait(&bars[kQFull], 0);
      if (!ok) fail();
      auto issue_pv = [&](int jj) {
        const int pbuf = jj % PB;
        const uint32_t vst = sbase + LY::kKV + (jj % kStagesTC) * LY::kStageBytes +
                             LY::kStageBytes / 2;
        for (int t = 0; t < NQ; ++t) {
          if (!mbar_wait(&bars[kPFull + t * PB + pbuf], (jj / PB) & 1)) { fail(); return false; }
          tc_fence_after();
          const uint32_t tmem_o = tmem + OB + t * 128;
          const int nparts = TT::kSplitP ? 2 : 1;
          for (int part = 0; part < nparts; ++part) {
            for (int ks = 0; ks < kKeysTC / 16; ++ks) {
              const uint64_t db = umma_desc(vst + ks * 16 * 128, kKeysTC * 128, 1024);
              const uint32_t acc = (jj > 0 || part > 0 || ks > 0) ? 1u : 0u;
              if constexpr (kPTmem) {
                // P of tile jj: hi in the first half of its S columns, lo in the second
                const uint32_t pa =
                    tmem + (t * SB + jj % SB) * kKeysTC + part * (kKeysTC / 2) + ks * 8;
                umma_ts(tmem_o, pa, db, idesc_pv, acc);
              } else {
                const uint32_t pbase = sbase + LY::kP + pbuf * LY::kPBuf;
                const uint64_t da = umma_desc(pbase + part * (kRowsTC * 128) + ks * 32, 16, 1024);
                umma(tmem_o, da, db, idesc_pv, acc);
              }
            }
          }
          umma_commit(&bars[kPvDone + t * PB + pbuf]);
        }
        umma_commit(&bars[kKvEmpty + (jj % kStagesTC)]);  // after every Q tile's P V
        return true;
      };
      for (int j = 0; ok && j < ntiles && !flags[0]; ++j) {
        const int st = j % kStagesTC, sb = j % SB;
        if (!mbar_wait(&bars[kKvFull + st], (j / kStagesTC) & 1)) { fail(); break; }
        const uint32_t kst = sbase + LY::kKV + st * LY::kStageBytes;
        bool go = true;
        for (int t = 0; t < NQ && go; ++t) {
          if constexpr (kPTmem) {
            // S(j) overwrites P(j - SB) of this Q tile: its P V must be done
            if (j >= SB && !mbar_wait(&bars[kPvDone + t * PB + sb], ((j / SB) - 1) & 1)) {
              fail();
              go = false;
              break;
            }
          } else {
            if (!mbar_wait(&bars[kSFree + sb], ((j / SB) & 1) ^ 1)) {
              fail();
              go = false;
              break;
            }
          }
          tc_fence_after();
          for (int ks = 0; ks < D / 16; ++ks) {
            const int h = ks >> 2, kk = ks & 3;
            const uint64_t da =
                umma_desc(sbase + LY::kQ + t * kRowsTC * D * 2 + h * kRowsTC * 128 + kk * 32, 16, 1024);
            const uint64_t db = umma_desc(kst + h * kKeysTC * 128 + kk * 32, 16, 1024);
            umma(tmem + (t * SB + sb) * kKeysTC, da, db, idesc_qk, ks > 0 ? 1u : 0u);
          }
          umma_commit(&bars[kSFull + t * SB + sb]);
        }
        if (!go) break;
        if (j > 0 && !issue_pv(j - 1)) break;
      }
      if (ok && !flags[0] && ntiles > 0) issue_pv(ntiles - 1);
      umma_commit(&bars[kDone]);  // completes when every MMA above has finished
      if (!mbar_wait(&bars[kDone], 0)) fail();
    }
  } else {
    // ======================= softmax warps =================================
    // Warp w: Q tile qt = w / SWT; within it rows 32 (w mod 4) .. +31 (its
    // TMEM lane quadrant), keys hf * kKeysPerHalf .. of every tile and O
    // columns hf * kOColsPerHalf ..
    const int qt = warp / SWT, wl = warp - qt * SWT;
    const int qd = wl & 3, hf = wl >> 2;
    const int r = qd * 32 + lane;              // query row of the Q tile = TMEM lane
    const int sid = hf * kRowsTC + r;          // 0 .. SWT * 32 - 1
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    const uint32_t tmem_s0 = tmem + qt * SB * kKeysTC;  // this Q tile's S/P buffers
    const uint32_t tmem_o = tmem + OB + qt * 128;       // and its O
    float *xmax = reinterpret_cast<float *>(smem + LY::kX);  // [2][kHalves][128]
    float *xl = xmax + 2 * kHalves * kRowsTC;                      // [kHalves][128]
    (void)xl;
    const int tok = qt * TPT + r / G;          // token (member) among the CTA's rows
    const int limit = PREFIX ? L - 1 : L - Q + t0 + tok;  // last key this row may see
    const float sl2 = a.scale_log2;
    if constexpr (PREFIX) {
      // Every member's table must hold the group's ids over the shared range.
      // All of the checks' loads are issued together here, while the first
      // tile is still in flight, instead of one dependent round trip per tile
      // on the producer's path.
      const int32_t *table = a.block_tables + (int64_t)seq * a.max_blocks_per_seq;
      for (int x0 = sid; x0 < ntok * nblk; x0 += SWT * 32 * 8) {
        int mine[8], ref[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int x = x0 + u * SWT * 32;
          const int i = x / nblk, b = x - i * nblk;
          mine[u] = x < ntok * nblk ? a.block_tables[(int64_t)(q0 + i) * a.max_blocks_per_seq + b] : 0;
          ref[u] = x < ntok * nblk ? table[b] : 0;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int x = x0 + u * SWT * 32;
          if (x < ntok * nblk && mine[u] != ref[u]) {
            const int i = x / nblk;
            if (!bad_member[i]) raise_error(a.err, PA_DEVERR_PREFIX);
            bad_member[i] = 1;
          }
        }
      }
    }
    float m_used = -INFINITY, l = 0.f;
    for (int j = 0; j < ntiles; ++j) {
      const int sb = j % SB;
      bool ok = !flags[0] && mbar_wait(&bars[kSFull + qt * SB + sb], (j / SB) & 1);
      if (!__all_sync(0xffffffffu, ok)) { fail(); break; }  // warp-uniform: tcgen05.ld is collective
      tc_fence_after();
      uint32_t sr[kKeysPerHalf];
      {
        uint32_t part[32];
#pragma unroll
        for (int q32 = 0; q32 < kKeysPerHalf / 32; ++q32) {
          tmem_ld32(tmem_s0 + lane_off + sb * kKeysTC + hf * kKeysPerHalf + q32 * 32, part);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) sr[q32 * 32 + i] = part[i];
        }
      }
      if constexpr (!kPTmem) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kSFree + sb]);
      }
      // scale and causal mask in place (as float bits), max over this warp's keys
      float mx = -INFINITY;
      const int k0 = j * kKeysTC + hf * kKeysPerHalf;
#pragma unroll
      for (int c = 0; c < kKeysPerHalf; ++c) {
        const float v = (k0 + c <= limit) ? __uint_as_float(sr[c]) * sl2 : -INFINITY;
        sr[c] = __float_as_uint(v);
        mx = fmaxf(mx, v);
      }
      if constexpr (kHalves > 1) {
        // the tile max of the row: exchange with the other warp of the quadrant
        const int xb = j & 1;
        xmax[(xb * kHalves + hf) * kRowsTC + r] = mx;
        mbar_arrive(&bars[kXFull + qd * 2 + xb]);
        const bool got = mbar_wait(&bars[kXFull + qd * 2 + xb], (j >> 1) & 1);
        if (!__all_sync(0xffffffffu, got)) { fail(); break; }
#pragma unroll
        for (int h2 = 0; h2 < kHalves; ++h2) mx = fmaxf(mx, xmax[(xb * kHalves + h2) * kRowsTC + r]);
      }
      // lazy rescale: move the reference max only when the tile max exceeds it
      // by more than 2^8 (first tile: always); both warps of a row decide alike
      const bool need = mx > m_used + kRescaleThreshold;
      float alpha = 1.f;
      if (need) {
        alpha = m_used == -INFINITY ? 0.f : fast_exp2(m_used - mx);
        m_used = mx;
        l *= alpha;
      }
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // O (in TMEM) is complete up to tile j-1 once that tile's P.V is done
        const bool done = mbar_wait(&bars[kPvDone + qt * PB + ((j - 1) % PB)], ((j - 1) / PB) & 1);
        if (!__all_sync(0xffffffffu, done)) { fail(); break; }
        tc_fence_after();
#pragma unroll 1
        for (int cblk = 0; cblk < kOColsPerHalf / 32; ++cblk) {
          const uint32_t col = hf * kOColsPerHalf + cblk * 32;
          uint32_t o[32];
          tmem_ld32(tmem_o + lane_off + col, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tmem_o + lane_off + col, o);
        }
        tmem_wait_st();
        tc_fence_before();
      }
      const int pb = j % PB;
      float psum = 0.f;
      if constexpr (kPTmem) {
        // P = 2^(x - m_used) over this tile's S columns: hi words at
        // columns [0, 32), lo words at [32, 64) of the buffer, two keys a word
        constexpr int W = kKeysPerHalf / 2;  // words of this warp per part
        uint32_t hi[W], lo[W];
#pragma unroll
        for (int i = 0; i < W; ++i) {
          const float p0 = fast_exp2(__uint_as_float(sr[2 * i]) - m_used);
          const float p1 = fast_exp2(__uint_as_float(sr[2 * i + 1]) - m_used);
          psum += p0 + p1;
          hi[i] = TT::pack(p0, p1);
          if constexpr (TT::kSplitP) {
            const float2 h = TT::unpack(hi[i]);
            lo[i] = TT::pack(p0 - h.x, p1 - h.y);
          }
        }
        const uint32_t pcol = tmem_s0 + lane_off + sb * kKeysTC + hf * W;
#pragma unroll
        for (int w16 = 0; w16 < W / 16; ++w16) {
          tmem_st16(pcol + w16 * 16, hi + w16 * 16);
          if constexpr (TT::kSplitP) tmem_st16(pcol + kKeysTC / 2 + w16 * 16, lo + w16 * 16);
        }
        tmem_wait_st();
      } else {
        // the P buffer of tile j was last read by tile j - PB's P.V
        if (j >= PB && !mbar_wait(&bars[kPvDone + qt * PB + pb], ((j - PB) / PB) & 1)) { fail(); break; }
        // P = 2^(x - m_used) -> shared memory (K-major, 128-byte swizzle), hi and lo
        const uint32_t prow = sbase + LY::kP + pb * LY::kPBuf + r * 128;
#pragma unroll
        for (int c8 = 0; c8 < kKeysPerHalf / 8; ++c8) {
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int c = c8 * 8 + 2 * i;
            const float p0 = fast_exp2(__uint_as_float(sr[c]) - m_used);
            const float p1 = fast_exp2(__uint_as_float(sr[c + 1]) - m_used);
            psum += p0 + p1;
            hi[i] = TT::pack(p0, p1);
            if constexpr (TT::kSplitP) {
              const float2 h = TT::unpack(hi[i]);
              lo[i] = TT::pack(p0 - h.x, p1 - h.y);
            }
          }
          const int cg = hf * (kKeysPerHalf / 8) + c8;  // 16-byte chunk of the row
          const uint32_t addr = prow + ((cg ^ (r & 7)) << 4);
          st_shared_v4(addr, hi[0], hi[1], hi[2], hi[3]);
          if constexpr (TT::kSplitP) st_shared_v4(addr + kRowsTC * 128, lo[0], lo[1], lo[2], lo[3]);
        }
      }
      l += psum;
      // keys past the context end in the last tile: zero their V rows (P is 0
      // there, but the slots may hold anything and 0 * NaN is NaN)
      if (j == ntiles - 1 && (j + 1) * kKeysTC > L) {
        const uint32_t vst = sbase + LY::kKV + (j % kStagesTC) * LY::kStageBytes +
                             LY::kStageBytes / 2;
        const int z0 = L - j * kKeysTC;  // first stale row of the tile
        const int nz = (kKeysTC - z0) * 16;  // 16-byte chunks over both halves
        // all of the tile's K/V bytes must have landed before they are overwritten
        if (mbar_wait(&bars[kKvFull + (j % kStagesTC)], (j / kStagesTC) & 1)) {
          for (int c = sid; c < nz; c += SWT * 32) {  // each Q tile's warps zero all of them
            const int row = z0 + c / 16, ch = c % 16;
            const int h = ch >> 3, cc = ch & 7;
            st_shared_v4(vst + h * kKeysTC * 128 + row * 128 + ((cc ^ (row & 7)) << 4), 0, 0, 0, 0);
          }
        } else {
          fail();
        }
      }
      fence_proxy_async_smem();  // generic-proxy writes -> tensor-core reads
      if constexpr (kPTmem) tc_fence_before();  // the tcgen05.st of P -> the MMA thread
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kPFull + qt * PB + pb]);
    }
    // ---- epilogue: O / l -> out ----
    bool ok = !flags[0] && ntiles > 0 &&
              mbar_wait(&bars[kPvDone + qt * PB + ((ntiles - 1) % PB)], ((ntiles - 1) / PB) & 1);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && ntiles > 0) fail();
    if constexpr (kHalves > 1) {  // the row's sum over both warps' keys
      xl[hf * kRowsTC + r] = l;
      mbar_arrive(&bars[kLFull + qd]);
      if (mbar_wait(&bars[kLFull + qd], 0)) {
        l = 0.f;
#pragma unroll
        for (int h2 = 0; h2 < kHalves; ++h2) l += xl[h2 * kRowsTC + r];
      } else {
        fail();
        ok = false;
      }
      ok = __all_sync(0xffffffffu, ok);
    }
    tc_fence_after();
    const bool write = tok < ntok && r < TPT * G;
    if constexpr (PREFIX) {
      // the member flags of every softmax warp (named barrier 1)
      asm volatile("bar.sync 1, %0;" ::"n"(SW * 32) : "memory");
      // record of (member q0 + tok, head): o unnormalised, the reference max
      // (base 2) o and l are relative to, l; NaN l marks a poisoned record
      const bool poison = !ok || flags[1] || (write && bad_member[tok]);
      float *rec = a.pre_rec + ((int64_t)(q0 + tok) * a.num_heads + kvh * G + r % G) * (D + 4);
#pragma unroll 1
      for (int cblk = 0; cblk < kOColsPerHalf / 32; ++cblk) {
        const int col = hf * kOColsPerHalf + cblk * 32;
        uint32_t o[32];
        tmem_ld32(tmem_o + lane_off + col, o);
        tmem_wait_ld();
        if (write) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4 *>(rec + col + i) =
                make_float4(__uint_as_float(o[i]), __uint_as_float(o[i + 1]), __uint_as_float(o[i + 2]),
                            __uint_as_float(o[i + 3]));
        }
      }
      if (write && hf == 0) {
        rec[D] = m_used;
        rec[D + 1] = poison ? __int_as_float(0x7fc00000) : l / a.o_scale;
      }
    } else {
      const float inv = (ok && l > 0.f && !flags[1]) ? (1.f / l) * a.o_scale : 0.f;
      T *dst = static_cast<T *>(a.out) + ((int64_t)(q0 + t0 + tok) * a.num_heads + kvh * G + r % G) * D;
#pragma unroll 1
      for (int cblk = 0; cblk < kOColsPerHalf / 32; ++cblk) {
        const int col = hf * kOColsPerHalf + cblk * 32;
        uint32_t o[32];
        tmem_ld32(tmem_o + lane_off + col, o);
        tmem_wait_ld();
        if (write) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 v;
            v.x = TT::pack(__uint_as_float(o[i + 0]) * inv, __uint_as_float(o[i + 1]) * inv);
            v.y = TT::pack(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
            v.z = TT::pack(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv);
            v.w = TT::pack(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv);
            *reinterpret_cast<uint4 *>(dst + col + i) = v;
          }
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == MW) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TCOLS)
                 : "memory");
  }
}

template <typename T, int BS, bool PREFIX = false, int NQ = 1>
cudaError_t launch_tc_t(const AttnArgs &a, cudaStream_t stream) {
  auto fn = encode_fn_tc();
  if (!fn) return cudaErrorNotSupported;
  constexpr int D = kHeadDim;
  const int G = a.group;
  const int TPT = kRowsTC / G;
  CUtensorMap tmq, tmk, tmv;
  {  // q viewed as [tokens][Hk][G][D]; box = TPT tokens x G heads x 64 columns
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)G, (cuuint64_t)a.num_kv_heads,
                          (cuuint64_t)a.num_q_tokens};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)G * D * 2, (cuuint64_t)a.num_heads * D * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)G, 1, (cuuint32_t)TPT};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    if (fn(&tmq, TcType<T>::kTma, 4, const_cast<void *>(a.q), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  for (int i = 0; i < 2; ++i) {
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)a.num_blocks * a.num_kv_heads * BS};
    cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)BS};
    cuuint32_t estr[2] = {1, 1};
    if (fn(i ? &tmv : &tmk, TcType<T>::kTma, 2, const_cast<void *>(i ? a.v_cache : a.k_cache), dims,
           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  auto kern = chunk_tc_kernel<T, BS, PREFIX, NQ>;
  constexpr int kBytes = TcLayoutT<NQ>::kBytes;
  constexpr int kThreads = 32 * (4 * kHalves * NQ + 2);
  {
    cudaError_t e = set_smem_limit_once(reinterpret_cast<const void *>(kern), kBytes);
    if (e != cudaSuccess) return e;
  }
  // chunk rows: (sequence, KV head, tile of TPT tokens); prefix: (group, KV
  // head, chunk of TPT members)
  const int tiles = PREFIX ? (a.max_group + TPT - 1) / TPT : (a.max_query_len + NQ * TPT - 1) / (NQ * TPT);
  const int64_t grid = (int64_t)(PREFIX ? a.num_groups : a.num_seqs) * a.num_kv_heads * tiles;
  if (grid == 0) return cudaSuccess;
  kern<<<(unsigned)grid, kThreads, kBytes, stream>>>(a, tmq, tmk, tmv, tiles);
  return cudaGetLastError();
}

}  // namespace

bool chunk_tc_supported(const AttnArgs &a, int dtype) {
  return (dtype == PA_BF16 || dtype == PA_F16) && a.head_dim == kHeadDim && a.group >= 1 &&
         a.group <= kRowsTC && kRowsTC % a.group == 0 && encode_fn_tc() != nullptr;
}

cudaError_t launch_prefix_tc(const AttnArgs &a, int dtype, cudaStream_t stream) {
  if (dtype == PA_BF16)
    return a.block_size == 16 ? launch_tc_t<__nv_bfloat16, 16, true>(a, stream)
                              : launch_tc_t<__nv_bfloat16, 32, true>(a, stream);
  return a.block_size == 16 ? launch_tc_t<__half, 16, true>(a, stream)
                            : launch_tc_t<__half, 32, true>(a, stream);
}

cudaError_t launch_chunk_tc(const AttnArgs &a, int dtype, cudaStream_t stream) {
  if (dtype == PA_BF16)
    return a.block_size == 16 ? launch_tc_t<__nv_bfloat16, 16, false, kChunkQTiles>(a, stream)
                              : launch_tc_t<__nv_bfloat16, 32, false, kChunkQTiles>(a, stream);
  return a.block_size == 16 ? launch_tc_t<__half, 16, false, kChunkQTiles>(a, stream)
                            : launch_tc_t<__half, 32, false, kChunkQTiles>(a, stream);
}

}  // namespace pa
