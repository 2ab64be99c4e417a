// chunk.cu -- attention of a chunked-prefill query chunk over its paged KV.
//
// A long prompt is processed in chunks that share a batch with decode tokens
// ("PagedAttention 实战", section Chunked Prefill).  For a sequence with Q > 1
// query rows and context length L (chunk included), row t sees keys
// 0 .. L-Q+t.  Unlike decode this is a dense contraction: the Q-tile of one
// (sequence, KV head) is (tokens x GROUP heads) rows long and every K/V tile
// is reused by all of them, so the products run on the tensor cores.
//
// This kernel: one CTA = (sequence, KV head, tile of 64/GROUP query tokens),
// i.e. 64 query rows, 4 warps x 16 rows.  K/V tiles of 64 keys are gathered
// through the block table with 16-byte cp.async into padded shared-memory rows
// (row stride D+8 elements: conflict-free ldmatrix), double-buffered.
// S = Q K^T and O += P V use mma.sync m16n8k16 (bf16/f16 in, fp32 out); the
// softmax is the online (running max / running sum) form in base 2.
#include <stdlib.h>
#include <string.h>

#include "mma_sync.cuh"
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kRows = 64;  // query rows per CTA
constexpr int kKT = 64;    // keys per tile
constexpr int kPad = 8;    // elements of padding per smem row

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(smem)), "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <typename T, int D, int BS>
__global__ void __launch_bounds__(128) chunk_kernel(const AttnArgs a, int tiles_per_seq) {
  constexpr int LD = D + kPad;
  constexpr int CPR = D / 8;  // 16-byte chunks per row
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __shared__ int s_bad;
  T *sQ = reinterpret_cast<T *>(smem_raw);
  T *sK = sQ + kRows * LD;      // [2][kKT][LD]
  T *sV = sK + 2 * kKT * LD;    // [2][kKT][LD]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x % tiles_per_seq;
  const int rest = blockIdx.x / tiles_per_seq;
  const int kvh = rest % a.num_kv_heads;
  const int seq = a.seq_begin + rest / a.num_kv_heads;
  const int q0 = a.query_start_loc[seq];
  const int Q = a.query_start_loc[seq + 1] - q0;
  if (Q <= 1) return;  // decode rows are handled by the decode kernel
  if (q0 < 0 || q0 + Q > a.num_q_tokens) return;  // reported by the decode kernel's scan
  if (Q > a.max_query_len) {  // rows past the host bound would be left unwritten
    if (threadIdx.x == 0 && blockIdx.x % tiles_per_seq == 0) raise_error(a.err, PA_DEVERR_QUERY_LEN);
    return;
  }
  const int G = a.group;
  const int TPT = kRows / G;  // query tokens per tile
  const int t0 = tile * TPT;
  if (t0 >= Q) return;
  const int ntok = min(TPT, Q - t0);
  const int L = a.context_lens[seq];
  const bool valid = L >= Q && L <= a.max_context_len;
  if (!valid) {
    if (tid == 0 && tile == 0 && kvh == 0)
      raise_error(a.err, L > a.max_context_len || L < 0 ? PA_DEVERR_CONTEXT_LEN
                                                        : PA_DEVERR_QUERY_LEN);
    for (int idx = tid; idx < ntok * G * D; idx += blockDim.x) {
      const int r = idx / D, d = idx - r * D;
      const int t = t0 + r / G, g = r % G;
      static_cast<T *>(a.out)[((int64_t)(q0 + t) * a.num_heads + kvh * G + g) * D + d] =
          Elem<T>::from_f(0.f);
    }
    return;
  }
  if (tid == 0) s_bad = 0;
  __syncthreads();
  const int32_t *table = a.block_tables + (int64_t)seq * a.max_blocks_per_seq;
  const T *kc = static_cast<const T *>(a.k_cache);
  const T *vc = static_cast<const T *>(a.v_cache);
  const int kend = L - Q + t0 + ntok;  // keys [0, kend) are visible to some row
  const int ntiles = (kend + kKT - 1) / kKT;

  // ---- stage the Q tile (row r = token t0 + r/G, head kvh*G + r%G) --------
  for (int idx = tid; idx < kRows * CPR; idx += blockDim.x) {
    const int r = idx / CPR, c = idx - r * CPR;
    T *dst = sQ + r * LD + c * 8;
    const int t = r / G, g = r % G;
    if (r < TPT * G && t < ntok) {
      cp_async16(dst, static_cast<const T *>(a.q) +
                          ((int64_t)(q0 + t0 + t) * a.num_heads + kvh * G + g) * D + c * 8);
    } else {
      *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
    }
  }

  auto load_tile = [&](int kt, int buf) {
    T *dk = sK + buf * kKT * LD;
    T *dv = sV + buf * kKT * LD;
    for (int idx = tid; idx < kKT * CPR; idx += blockDim.x) {
      const int r = idx / CPR, c = idx - r * CPR;
      const int key = kt * kKT + r;
      if (key < kend) {
        int pb = table[key / BS];
        if (pb < 0 || pb >= a.num_blocks) {
          raise_error(a.err, PA_DEVERR_BLOCK_ID);
          s_bad = 1;
          pb = -1;
        }
        if (pb >= 0) {
          const int64_t off = (((int64_t)pb * a.num_kv_heads + kvh) * BS + (key % BS)) * D + c * 8;
          cp_async16(dk + r * LD + c * 8, kc + off);
          cp_async16(dv + r * LD + c * 8, vc + off);
          continue;
        }
      }
      *reinterpret_cast<uint4 *>(dk + r * LD + c * 8) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4 *>(dv + r * LD + c * 8) = make_uint4(0, 0, 0, 0);
    }
  };

  load_tile(0, 0);
  cp_async_commit();

  // per-thread fragment coordinates
  const int g8 = lane >> 2;   // row within the 8-row half
  const int tig = lane & 3;   // thread in quad
  const int row_a = warp * 16 + g8;       // rows of c0/c1
  const int row_b = row_a + 8;            // rows of c2/c3
  const int lim_a = L - Q + t0 + row_a / G;  // last visible key of row_a
  const int lim_b = L - Q + t0 + row_b / G;

  uint32_t qa[D / 16][4];
  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

  for (int kt = 0; kt < ntiles; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < ntiles) load_tile(kt + 1, buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (kt == 0) {
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = ks * 16 + (lane >> 4) * 8;
        ldsm_x4(qa[ks], sQ + r * LD + c);
      }
    }
    const T *tK = sK + buf * kKT * LD;
    const T *tV = sV + buf * kKT * LD;

    // ---- S = Q K^T (16 rows x 64 keys per warp) ----
    float s[kKT / 8][4];
#pragma unroll
    for (int i = 0; i < kKT / 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
      for (int np = 0; np < kKT / 16; ++np) {
        uint32_t b[4];
        const int key = np * 16 + (lane & 7) + (lane >> 4) * 8;
        const int c = ks * 16 + ((lane >> 3) & 1) * 8;
        ldsm_x4(b, tK + key * LD + c);
        Mma<T>::run(s[2 * np], qa[ks], b[0], b[1]);
        Mma<T>::run(s[2 * np + 1], qa[ks], b[2], b[3]);
      }
    }

    // ---- scale, causal mask, online softmax ----
    const int k0 = kt * kKT;
    const bool need_mask = k0 + kKT - 1 > L - Q + t0;
    float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
    for (int i = 0; i < kKT / 8; ++i) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v = s[i][c] * a.scale_log2;
        if (need_mask) {
          const int key = k0 + i * 8 + tig * 2 + (c & 1);
          if (key > (c < 2 ? lim_a : lim_b)) v = -INFINITY;
        }
        s[i][c] = v;
      }
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
    uint32_t pa[kKT / 16][4];
    uint32_t pr[Mma<T>::kSplitP ? kKT / 16 : 1][4];
#pragma unroll
    for (int i = 0; i < kKT / 8; ++i) {
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
    for (int kk = 0; kk < kKT / 16; ++kk) {
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        uint32_t b[4];
        const int key = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = dp * 16 + (lane >> 4) * 8;
        ldsm_x4_t(b, tV + key * LD + c);
        Mma<T>::run(o[2 * dp], pa[kk], b[0], b[1]);
        Mma<T>::run(o[2 * dp + 1], pa[kk], b[2], b[3]);
        if constexpr (Mma<T>::kSplitP) {
          Mma<T>::run(o[2 * dp], pr[kk], b[0], b[1]);
          Mma<T>::run(o[2 * dp + 1], pr[kk], b[2], b[3]);
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // ---- normalise and write rows that exist ----
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
  __syncthreads();
  const bool bad = s_bad != 0;  // a bad block id anywhere: the tile's rows are zeros
  const float inv_a = (l_a > 0.f && !bad) ? (1.f / l_a) * a.o_scale : 0.f;
  const float inv_b = (l_b > 0.f && !bad) ? (1.f / l_b) * a.o_scale : 0.f;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = half ? row_b : row_a;
    const int t = r / G, g = r % G;
    if (r >= TPT * G || t >= ntok) continue;
    const float inv = half ? inv_b : inv_a;
    T *dst = static_cast<T *>(a.out) + ((int64_t)(q0 + t0 + t) * a.num_heads + kvh * G + g) * D;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      const uint32_t v = Mma<T>::pack(o[i][half * 2] * inv, o[i][half * 2 + 1] * inv);
      *reinterpret_cast<uint32_t *>(dst + i * 8 + tig * 2) = v;
    }
  }
}

template <typename T, int D, int BS>
cudaError_t launch_chunk_t(const AttnArgs &a, cudaStream_t stream) {
  constexpr int LD = D + kPad;
  const int smem = (kRows * LD + 4 * kKT * LD) * (int)sizeof(T);
  auto kern = chunk_kernel<T, D, BS>;
  cudaError_t e = set_smem_limit_once(reinterpret_cast<const void *>(kern), smem);
  if (e != cudaSuccess) return e;
  const int tpt = kRows / a.group;
  const int tiles = (a.max_query_len + tpt - 1) / tpt;
  const int64_t grid = (int64_t)a.num_seqs * a.num_kv_heads * tiles;
  if (grid == 0) return cudaSuccess;
  kern<<<(unsigned)grid, 128, smem, stream>>>(a, tiles);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t chunk_bs(const AttnArgs &a, cudaStream_t s) {
  return a.block_size == 16 ? launch_chunk_t<T, D, 16>(a, s) : launch_chunk_t<T, D, 32>(a, s);
}

template <typename T>
cudaError_t chunk_d(const AttnArgs &a, cudaStream_t s) {
  return a.head_dim == 64 ? chunk_bs<T, 64>(a, s) : chunk_bs<T, 128>(a, s);
}

}  // namespace

cudaError_t launch_chunk(const AttnArgs &a, int dtype, int /*num_q_tokens*/, cudaStream_t stream) {
  // head_dim 128: the tcgen05 ping-pong kernel (chunk_pp.cu); PA_CHUNK_KERNEL=tc64
  // selects the earlier tcgen05 kernel over 64-key tiles (chunk_tc.cu) and
  // PA_CHUNK_KERNEL=mma this mma.sync kernel, which also serves head_dim 64.
  const char *sel = getenv("PA_CHUNK_KERNEL");
  const bool want_mma = sel && strcmp(sel, "mma") == 0;
  const bool want_tc64 = sel && strcmp(sel, "tc64") == 0;
  if (!want_mma && !want_tc64 && chunk_pp_supported(a, dtype)) return launch_chunk_pp(a, dtype, stream);
  if (!want_mma && chunk_tc_supported(a, dtype)) return launch_chunk_tc(a, dtype, stream);
  if (dtype == PA_F16) return chunk_d<__half>(a, stream);
  if (dtype == PA_BF16) return chunk_d<__nv_bfloat16>(a, stream);
  return cudaErrorNotSupported;  // fp32 chunks run through the decode kernel's row mode
}

}  // namespace pa
