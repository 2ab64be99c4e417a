// fp8.cu -- FP8 (E4M3) KV cache: quantising reshape_and_cache and decode over
// the quantised cache.
//
// KV-cache quantisation halves the bytes decode has to read ("理解 vLLM
// PagedAttention", 版本矩阵: 量化 FP8 ... 权重 KV cache 量化; decode is bound by
// the KV history it reads, "PagedAttention 实战", section 先理解 KV Cache).  One
// scale per cache tensor: an element x of a new key is stored as the E4M3
// code of x / k_scale (one IEEE binary32 division, round to nearest even,
// magnitudes beyond 448 saturated), values likewise with v_scale.  Decode
// reads the codes (one byte each) and computes with code * scale: k_scale is
// folded into the logit scale, v_scale into the softmax sum.
#include <cuda_fp8.h>

#include "../../include/pa.h"
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

template <typename T>
__device__ __forceinline__ void load8(const T *p, float (&x)[8]);

template <>
__device__ __forceinline__ void load8<float>(const float *p, float (&x)[8]) {
  const float4 a = __ldcs(reinterpret_cast<const float4 *>(p));
  const float4 b = __ldcs(reinterpret_cast<const float4 *>(p) + 1);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16 *p, float (&x)[8]) {
  const uint4 v = __ldcs(reinterpret_cast<const uint4 *>(p));
  float2 f[4];
  Elem<__nv_bfloat16>::to_f2(v, f);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = f[i].x;
    x[2 * i + 1] = f[i].y;
  }
}

template <>
__device__ __forceinline__ void load8<__half>(const __half *p, float (&x)[8]) {
  const uint4 v = __ldcs(reinterpret_cast<const uint4 *>(p));
  float2 f[4];
  Elem<__half>::to_f2(v, f);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = f[i].x;
    x[2 * i + 1] = f[i].y;
  }
}

// Two consecutive elements as floats.
template <typename T>
__device__ __forceinline__ void load2(const T *p, float &a, float &b);
template <>
__device__ __forceinline__ void load2<float>(const float *p, float &a, float &b) {
  const float2 v = __ldcs(reinterpret_cast<const float2 *>(p));
  a = v.x;
  b = v.y;
}
template <>
__device__ __forceinline__ void load2<__nv_bfloat16>(const __nv_bfloat16 *p, float &a, float &b) {
  const uint32_t u = __ldcs(reinterpret_cast<const unsigned int *>(p));
  a = __uint_as_float(u << 16);
  b = __uint_as_float(u & 0xffff0000u);
}
template <>
__device__ __forceinline__ void load2<__half>(const __half *p, float &a, float &b) {
  const uint32_t u = __ldcs(reinterpret_cast<const unsigned int *>(p));
  const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&u));
  a = f.x;
  b = f.y;
}

// Two elements -> two E4M3 codes of x / scale (the first in the low byte).
__device__ __forceinline__ uint32_t quant2(float a, float b, float scale) {
  const float2 q = make_float2(__fdiv_rn(a, scale), __fdiv_rn(b, scale));
  return (uint32_t)__nv_cvt_float2_to_fp8x2(q, __NV_SATFINITE, __NV_E4M3);
}

// K: one thread per (token, kv head, 16-byte chunk of the row), so that the
// lanes of a warp write whole rows; V: see below.  The cache tile of a
// (block, kv head) is laid out for the decode kernel's fragment loads:
//   K [BS][D]: column d = 64j + 16k + c of row r goes to byte
//     ((4j + t) ^ (r mod D/16)) * 16 + 4k + i of the row, t = (c mod 8) / 2,
//     i = c mod 2 + 2 (c / 8): the four codes a thread's mma fragment needs
//     for k-step 4j + k sit in one word, its four k-steps in one 16-byte
//     chunk, and the chunk swizzle keeps the warp's loads off shared banks.
//   V [D][BS] (transposed): key r = 16k + c of column d goes to byte
//     d * BS + (BS == 16 ? 4t + i : 8t + 4k + i).
template <typename T, int D, int BS>
__global__ void __launch_bounds__(256) reshape_and_cache_fp8_kernel(
    const T *__restrict__ key, const T *__restrict__ value, unsigned char *__restrict__ k_cache,
    unsigned char *__restrict__ v_cache, const int64_t *__restrict__ slot_mapping, int num_tokens,
    int num_kv_heads, int64_t num_slots, float k_scale, float v_scale, unsigned int *err) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int G16 = D / 16;
  const int64_t per_token = (int64_t)num_kv_heads * G16;
  const int64_t total = (int64_t)num_tokens * per_token;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t tok = i / per_token;
    const int64_t rest = i - tok * per_token;
    const int64_t slot = slot_mapping[tok];
    if (slot < 0) continue;  // padding token
    if (slot >= num_slots) {
      if (rest == 0) raise_error(err, PA_DEVERR_SLOT);
      continue;
    }
    // the row's 16-byte chunk of fragment column group jt = 4j + t: word k
    // holds columns 64j + 16k + 2t, +1 (low half) and +8, +9 (high half)
    const int h = (int)(rest / G16);
    const int jt = (int)(rest - (int64_t)h * G16);
    const int j = jt >> 2, t = jt & 3;
    const int64_t blk = slot / BS;
    const int r = (int)(slot - blk * BS);
    const int64_t tile = (blk * num_kv_heads + h) * (int64_t)(BS * D);
    const T *kp = key + (tok * num_kv_heads + h) * D + 64 * j + 2 * t;
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float a0, a1, b0, b1;
      load2<T>(kp + 16 * k, a0, a1);
      load2<T>(kp + 16 * k + 8, b0, b1);
      w[k] = quant2(a0, a1, k_scale) | (quant2(b0, b1, k_scale) << 16);
    }
    unsigned char *krow = k_cache + tile + (int64_t)r * D;
    *reinterpret_cast<uint4 *>(krow + ((jt ^ (r & (G16 - 1))) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  // V: a thread takes 8 columns of one token; the 16 lanes of a half-warp take
  // 16 consecutive tokens, so that when they fill consecutive slots of a
  // block their bytes of a column form whole 16-byte runs of the transposed
  // tile (one store transaction instead of sixteen)
  const int64_t vtotal = (int64_t)((num_tokens + 15) / 16) * num_kv_heads * G16 * 32;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < vtotal;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int lo = (int)(i & 15), half = (int)((i >> 4) & 1);
    int64_t rest = i >> 5;
    const int g16 = (int)(rest % G16);
    rest /= G16;
    const int h = (int)(rest % num_kv_heads);
    const int64_t tok = (rest / num_kv_heads) * 16 + lo;
    if (tok >= num_tokens) continue;
    const int64_t slot = slot_mapping[tok];
    if (slot < 0 || slot >= num_slots) continue;  // reported by the K loop
    const int64_t blk = slot / BS;
    const int r = (int)(slot - blk * BS);
    const int64_t tile = (blk * num_kv_heads + h) * (int64_t)(BS * D);
    float x[8];
    load8<T>(value + (tok * num_kv_heads + h) * D + g16 * 16 + half * 8, x);
    const int kk = r >> 4, c = r & 15;
    const int vpos = BS == 16 ? 4 * ((c & 7) >> 1) + (c & 1) + 2 * (c >> 3)
                              : 8 * ((c & 7) >> 1) + 4 * kk + (c & 1) + 2 * (c >> 3);
    unsigned char *vcol = v_cache + tile + (int64_t)(g16 * 16 + half * 8) * BS + vpos;
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      const uint32_t two = quant2(x[e], x[e + 1], v_scale);
      vcol[(int64_t)e * BS] = (unsigned char)(two & 0xffu);
      vcol[(int64_t)(e + 1) * BS] = (unsigned char)(two >> 8);
    }
  }
}

template <typename T, int D>
cudaError_t reshape_fp8_bs(int block_size, const cudaLaunchConfig_t &cfg, const void *key,
                           const void *value, void *kc, void *vc, const int64_t *slots,
                           int num_tokens, int num_kv_heads, int64_t num_slots, float ks,
                           float vs, unsigned int *err) {
  if (block_size == 16)
    return cudaLaunchKernelEx(&cfg, reshape_and_cache_fp8_kernel<T, D, 16>, (const T *)key,
                              (const T *)value, (unsigned char *)kc, (unsigned char *)vc, slots,
                              num_tokens, num_kv_heads, num_slots, ks, vs, err);
  return cudaLaunchKernelEx(&cfg, reshape_and_cache_fp8_kernel<T, D, 32>, (const T *)key,
                            (const T *)value, (unsigned char *)kc, (unsigned char *)vc, slots,
                            num_tokens, num_kv_heads, num_slots, ks, vs, err);
}

template <typename T>
cudaError_t reshape_fp8_d(int head_dim, int block_size, const cudaLaunchConfig_t &cfg,
                          const void *key, const void *value, void *kc, void *vc,
                          const int64_t *slots, int num_tokens, int num_kv_heads,
                          int64_t num_slots, float ks, float vs, unsigned int *err) {
  if (head_dim == 64)
    return reshape_fp8_bs<T, 64>(block_size, cfg, key, value, kc, vc, slots, num_tokens,
                                 num_kv_heads, num_slots, ks, vs, err);
  return reshape_fp8_bs<T, 128>(block_size, cfg, key, value, kc, vc, slots, num_tokens,
                                num_kv_heads, num_slots, ks, vs, err);
}

// ---- chunk rows over an FP8 cache -----------------------------------------
// The tensor-core chunk kernels read 16-bit K/V tiles through TMA.  For a
// mixed batch over an FP8 cache the blocks of the sequences with chunk rows
// are first staged into a 16-bit pool of their codes' values (every E4M3
// value is exact in fp16 and bf16), in the plain [block_size][head_dim] tile
// layout, with per-sequence tables into that pool; k_scale goes into the
// logit scale and v_scale onto O / l, as for the decode rows.

// A sequence has staged blocks when it has more than one query row and a
// context length the kernels accept.
__device__ __forceinline__ int staged_blocks_of(const AttnArgs &a, int s) {
  const int Q = a.query_start_loc[s + 1] - a.query_start_loc[s];
  const int L = a.context_lens[s];
  if (Q <= 1 || L <= 0 || L > a.max_context_len) return 0;
  return (L + a.block_size - 1) / a.block_size;
}

// base[s] = first staged block of sequence s, base[num_seqs] = their total.
// One CTA of 1024 threads; PA_DEVERR_STAGING if the total exceeds capacity.
__global__ void __launch_bounds__(1024) fp8_stage_plan_kernel(const AttnArgs a, int *base,
                                                             int capacity) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ int warp_tot[32];
  __shared__ int carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int s0 = 0; s0 < a.num_seqs; s0 += 1024) {
    const int s = s0 + tid;
    const int c = s < a.num_seqs ? staged_blocks_of(a, s) : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int w = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_tot[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int before = carry + (warp > 0 ? warp_tot[warp - 1] : 0);
    if (s < a.num_seqs) base[s] = before + incl - c;
    __syncthreads();
    if (tid == 0) carry += warp_tot[31];
    __syncthreads();
  }
  if (tid == 0) {
    base[a.num_seqs] = carry;
    if (carry > capacity) raise_error(a.err, PA_DEVERR_STAGING);
  }
}

template <typename T>
__device__ __forceinline__ uint32_t pack2_t(float lo, float hi);
template <>
__device__ __forceinline__ uint32_t pack2_t<__nv_bfloat16>(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}


// Blocks of chunk-row sequences -> the 16-bit pool (sk, sv) and the tables
// `tab` [num_seqs][max_blocks_per_seq] (-1 for a block not staged: an id
// outside the cache, or past the pool's capacity).  Grid (x: (block, group of
// up to kStageHeads KV heads), y: sequences).  The K (and V) tiles of
// consecutive KV heads of a block are one contiguous run in the cache and in
// the pool.  A thread loads 16-byte runs of codes (all in flight at once),
// converts each pair of codes with one cvt and stores the values at their
// places in a plain [head][row][column] tile in shared memory; the group then
// goes out with 16-byte stores.
//   K run at byte 16q of a tile: row r = q / (D/16), chunk p = q mod (D/16)
//     holds k-steps 0..3 of fragment column group 4j + t = p ^ (r mod D/16):
//     word k, bytes 0,1 -> columns 64j + 16k + 2t, +1; bytes 2,3 -> +8, +9.
//   V run at byte 16q: column d = 16q / BS, bytes b0 .. b0+15 (b0 = 16q mod
//     BS) of its transposed keys; byte b is key 16 kk + 2t + (i & 1) + 8 (i >> 1)
//     with i = b mod 4, and t = b / 4 (BS 16) or t = b / 8, kk = (b / 4) mod 2
//     (BS 32).
constexpr int kStageHeads = 4;

template <typename T>
__device__ __forceinline__ uint32_t e4m3x2_to(uint16_t two);
template <>
__device__ __forceinline__ uint32_t e4m3x2_to<__half>(uint16_t two) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(two, __NV_E4M3);  // low code -> .x
  return (uint32_t)h.x | ((uint32_t)h.y << 16);
}
template <>
__device__ __forceinline__ uint32_t e4m3x2_to<__nv_bfloat16>(uint16_t two) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(two, __NV_E4M3);
  const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h));
  return pack2_t<__nv_bfloat16>(f.x, f.y);
}

// Converts the K and V tiles of KV heads h0 .. h0+nh-1 of cache block `src`
// into pool block `id` (CTA-wide: every thread of the CTA calls it).
template <typename T, int D, int BS>
__device__ __forceinline__ void stage_group(const AttnArgs &a, int src, int id, int h0, int nh,
                                            T *sk, T *sv, unsigned char *stage_sm) {
  constexpr int kTile = BS * D;                 // elements (= code bytes) per tile
  constexpr int kQ = kTile / 16;                // 16-byte code runs per tile
  constexpr int kPer = kStageHeads * kQ / 256;  // runs per thread for K and for V
  constexpr int G16 = D / 16;
  uint16_t *ok_sm = reinterpret_cast<uint16_t *>(stage_sm);
  uint16_t *ov_sm = ok_sm + kStageHeads * kTile;
  const unsigned char *kcache = static_cast<const unsigned char *>(a.k_cache);
  const unsigned char *vcache = static_cast<const unsigned char *>(a.v_cache);
  const int64_t run = ((int64_t)src * a.num_kv_heads + h0) * kTile;
  const int n16 = nh * kQ;
  uint4 rk[kPer], rv[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int i = threadIdx.x + u * 256;
    if (i < n16) {
      rk[u] = reinterpret_cast<const uint4 *>(kcache + run)[i];
      rv[u] = reinterpret_cast<const uint4 *>(vcache + run)[i];
    }
  }
  __syncthreads();  // the previous group's tile has been copied out
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int i = threadIdx.x + u * 256;
    if (i < n16) {
      const int hh = i / kQ, q = i - hh * kQ;
      // K: four words, one per k-step, each two adjacent column pairs
      {
        const int r = q / G16, p = q - r * G16;
        const int jt = p ^ (r & (G16 - 1));
        const int col = 64 * (jt >> 2) + 2 * (jt & 3);
        uint16_t *row = ok_sm + hh * kTile + r * D;
        const uint32_t w[4] = {rk[u].x, rk[u].y, rk[u].z, rk[u].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          *reinterpret_cast<uint32_t *>(row + col + 16 * k) = e4m3x2_to<T>((uint16_t)(w[k] & 0xffffu));
          *reinterpret_cast<uint32_t *>(row + col + 16 * k + 8) = e4m3x2_to<T>((uint16_t)(w[k] >> 16));
        }
      }
      // V: sixteen keys of one column
      {
        const int d = (16 * q) / BS, b0 = (16 * q) % BS;
        uint16_t *tile = ov_sm + hh * kTile;
        const uint32_t w[4] = {rv[u].x, rv[u].y, rv[u].z, rv[u].w};
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const uint32_t two = e4m3x2_to<T>((uint16_t)(half ? w[wi] >> 16 : w[wi] & 0xffffu));
            const int bb = b0 + 4 * wi + 2 * half;  // byte of the first code of the pair
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int byte = bb + e, i4 = byte & 3;
              const int t = BS == 16 ? (byte >> 2) : (byte >> 3);
              const int kk = BS == 16 ? 0 : ((byte >> 2) & 1);
              const int key = 16 * kk + 2 * t + (i4 & 1) + 8 * (i4 >> 1);
              tile[key * D + d] = (uint16_t)(e ? two >> 16 : two & 0xffffu);
            }
          }
        }
      }
    }
  }
  __syncthreads();
  const int64_t dst = ((int64_t)id * a.num_kv_heads + h0) * kTile;
  for (int i = threadIdx.x; i < nh * kTile / 8; i += blockDim.x) {
    reinterpret_cast<uint4 *>(sk + dst)[i] = reinterpret_cast<const uint4 *>(ok_sm)[i];
    reinterpret_cast<uint4 *>(sv + dst)[i] = reinterpret_cast<const uint4 *>(ov_sm)[i];
  }
}

template <typename T, int D, int BS>
__global__ void __launch_bounds__(256) fp8_stage_kernel(const AttnArgs a, const int *base,
                                                       int32_t *tab, T *sk, T *sv, int capacity) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  extern __shared__ __align__(16) unsigned char stage_sm[];  // [K | V][kStageHeads][BS][D] of T
  const int s = blockIdx.y;
  const int nblk = staged_blocks_of(a, s);
  const int ngrp = (a.num_kv_heads + kStageHeads - 1) / kStageHeads;
  for (int bg = blockIdx.x; bg < nblk * ngrp; bg += gridDim.x) {
    const int b = bg / ngrp, h0 = (bg - b * ngrp) * kStageHeads;
    const int id = base[s] + b;
    const int src = a.block_tables[(int64_t)s * a.max_blocks_per_seq + b];
    const bool src_ok = src >= 0 && src < a.num_blocks;
    const bool ok = src_ok && id < capacity;
    if (threadIdx.x == 0 && h0 == 0) {
      tab[(int64_t)s * a.max_blocks_per_seq + b] = ok ? id : -1;
      if (!src_ok) raise_error(a.err, PA_DEVERR_BLOCK_ID);
    }
    if (!ok) continue;  // uniform over the CTA
    stage_group<T, D, BS>(a, src, id, h0, min(kStageHeads, a.num_kv_heads - h0), sk, sv, stage_sm);
  }
}

// Shared prefixes over an FP8 cache: group j (sequences grp_start[j] ..
// grp_start[j+1]-1 sharing grp_blocks[j] leading blocks) stages those blocks
// of its first sequence at pool blocks base[j] ..; gbase[num_groups] = total.
__device__ __forceinline__ int group_blocks_of(const AttnArgs &a, int j) {
  const int s0 = a.grp_start[j], s1 = a.grp_start[j + 1], P = a.grp_blocks[j];
  const bool valid = 0 <= s0 && s0 < s1 && s1 <= a.num_seqs && 0 < P && P <= a.max_blocks_per_seq;
  return valid ? P : 0;
}

__global__ void __launch_bounds__(1024) fp8_group_plan_kernel(const AttnArgs a, int *gbase,
                                                             int capacity) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ int warp_tot[32];
  __shared__ int carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int j0 = 0; j0 < a.num_groups; j0 += 1024) {
    const int j = j0 + tid;
    const int c = j < a.num_groups ? group_blocks_of(a, j) : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int w = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_tot[lane] = w;
    }
    __syncthreads();
    const int before = carry + (warp > 0 ? warp_tot[warp - 1] : 0);
    if (j < a.num_groups) gbase[j] = before + incl - c;
    __syncthreads();
    if (tid == 0) carry += warp_tot[31];
    __syncthreads();
  }
  if (tid == 0) {
    gbase[a.num_groups] = carry;
    if (carry > capacity) raise_error(a.err, PA_DEVERR_STAGING);
  }
}

// Grid (x: (shared block, group of KV heads), y: groups).  Every member's
// table row over the shared range gets the staged id where it holds the first
// sequence's block and -1 where it does not, so that the prefix kernel's
// member check still sees a member whose table differs.
template <typename T, int D, int BS>
__global__ void __launch_bounds__(256) fp8_group_stage_kernel(const AttnArgs a, const int *gbase,
                                                             int32_t *tab, T *sk, T *sv,
                                                             int capacity) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  extern __shared__ __align__(16) unsigned char stage_sm[];
  const int j = blockIdx.y;
  const int P = group_blocks_of(a, j);
  if (P == 0) return;
  const int s0 = a.grp_start[j], s1 = a.grp_start[j + 1];
  const int ngrp = (a.num_kv_heads + kStageHeads - 1) / kStageHeads;
  for (int bg = blockIdx.x; bg < P * ngrp; bg += gridDim.x) {
    const int b = bg / ngrp, h0 = (bg - b * ngrp) * kStageHeads;
    const int id = gbase[j] + b;
    const int src = a.block_tables[(int64_t)s0 * a.max_blocks_per_seq + b];
    const bool src_ok = src >= 0 && src < a.num_blocks;
    const bool ok = src_ok && id < capacity;
    if (h0 == 0) {
      for (int m = s0 + (int)threadIdx.x; m < s1; m += blockDim.x) {
        const int mine = a.block_tables[(int64_t)m * a.max_blocks_per_seq + b];
        tab[(int64_t)m * a.max_blocks_per_seq + b] = (ok && mine == src) ? id : -1;
      }
      if (threadIdx.x == 0 && !src_ok) raise_error(a.err, PA_DEVERR_BLOCK_ID);
    }
    if (!ok) continue;  // uniform over the CTA
    stage_group<T, D, BS>(a, src, id, h0, min(kStageHeads, a.num_kv_heads - h0), sk, sv, stage_sm);
  }
}

template <typename T, int D, int BS>
cudaError_t launch_group_stage_bs(const AttnArgs &a, const int *gbase, int32_t *tab, void *sk,
                                  void *sv, int capacity, cudaStream_t s) {
  auto kern = fp8_group_stage_kernel<T, D, BS>;
  constexpr int kSmem = 2 * kStageHeads * BS * D * 2;
  cudaError_t e = set_smem_limit_once(reinterpret_cast<const void *>(kern), kSmem);
  if (e != cudaSuccess) return e;
  const int ngrp = (a.num_kv_heads + kStageHeads - 1) / kStageHeads;
  const int64_t work = (int64_t)a.max_blocks_per_seq * ngrp;
  const dim3 grid((unsigned)(work < 1024 ? work : 1024), (unsigned)a.num_groups);
  kern<<<grid, 256, kSmem, s>>>(a, gbase, tab, static_cast<T *>(sk), static_cast<T *>(sv), capacity);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_group_stage_t(const AttnArgs &a, const int *gbase, int32_t *tab, void *sk,
                                 void *sv, int capacity, cudaStream_t s) {
  return a.block_size == 16 ? launch_group_stage_bs<T, D, 16>(a, gbase, tab, sk, sv, capacity, s)
                            : launch_group_stage_bs<T, D, 32>(a, gbase, tab, sk, sv, capacity, s);
}

template <typename T, int D, int BS>
cudaError_t launch_stage_bs(const AttnArgs &a, const int *base, int32_t *tab, void *sk, void *sv,
                            int capacity, cudaStream_t s) {
  auto kern = fp8_stage_kernel<T, D, BS>;
  constexpr int kSmem = 2 * kStageHeads * BS * D * 2;
  cudaError_t e = set_smem_limit_once(reinterpret_cast<const void *>(kern), kSmem);
  if (e != cudaSuccess) return e;
  const int ngrp = (a.num_kv_heads + kStageHeads - 1) / kStageHeads;
  const int64_t work = (int64_t)a.max_blocks_per_seq * ngrp;
  const dim3 grid((unsigned)(work < 1024 ? work : 1024), (unsigned)a.num_seqs);
  kern<<<grid, 256, kSmem, s>>>(a, base, tab, static_cast<T *>(sk), static_cast<T *>(sv), capacity);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_stage_t(const AttnArgs &a, const int *base, int32_t *tab, void *sk, void *sv,
                           int capacity, cudaStream_t s) {
  return a.block_size == 16 ? launch_stage_bs<T, D, 16>(a, base, tab, sk, sv, capacity, s)
                            : launch_stage_bs<T, D, 32>(a, base, tab, sk, sv, capacity, s);
}

// Workspace of pa_decode_fp8_rows: the decode rows' records (the bound of
// pa_decode_workspace_size), base [num_seqs + 1], the staged tables
// [num_seqs][max_blocks_per_seq] and the K and V pools of staged_blocks
// 16-bit blocks, each part 1 KiB aligned.
struct RowsWs {
  size_t base, tab, k, v, total;
};
RowsWs rows_ws(size_t dec, int num_seqs, int num_kv_heads, int head_dim, int block_size,
               int max_blocks_per_seq, int staged_blocks) {
  auto up = [](size_t x) { return (x + 1023) / 1024 * 1024; };
  RowsWs w;
  w.base = up(dec);
  w.tab = w.base + up((size_t)(num_seqs + 1) * sizeof(int));
  w.k = w.tab + up((size_t)num_seqs * max_blocks_per_seq * sizeof(int32_t));
  const size_t pool = up((size_t)staged_blocks * num_kv_heads * block_size * head_dim * 2);
  w.v = w.k + pool;
  w.total = w.v + pool;
  return w;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool scale_ok(float s) { return s > 0.f && s < 3.0e38f; }

}  // namespace

cudaError_t launch_fp8_group_stage(const AttnArgs &a, int q_dtype, int *gbase, int32_t *tab,
                                   void *sk, void *sv, int capacity, cudaStream_t s) {
  if (a.num_groups <= 0) return cudaSuccess;
  fp8_group_plan_kernel<<<1, 1024, 0, s>>>(a, gbase, capacity);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (q_dtype == PA_BF16)
    return a.head_dim == 64 ? launch_group_stage_t<__nv_bfloat16, 64>(a, gbase, tab, sk, sv, capacity, s)
                            : launch_group_stage_t<__nv_bfloat16, 128>(a, gbase, tab, sk, sv, capacity, s);
  return a.head_dim == 64 ? launch_group_stage_t<__half, 64>(a, gbase, tab, sk, sv, capacity, s)
                          : launch_group_stage_t<__half, 128>(a, gbase, tab, sk, sv, capacity, s);
}

size_t fp8_pool_bytes(int staged_blocks, int num_kv_heads, int head_dim, int block_size) {
  return ((size_t)staged_blocks * num_kv_heads * block_size * head_dim * 2 + 1023) / 1024 * 1024;
}

}  // namespace pa

using namespace pa;

namespace pa {
namespace {

int decode_fp8_call(void *out, const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *block_tables, int max_blocks_per_seq,
                    const int32_t *context_lens, const int32_t *query_start_loc, int num_seqs,
                    int num_q_tokens, int max_query_len, int num_heads, int num_kv_heads,
                    int head_dim, int block_size, int num_blocks, float scale, float k_scale,
                    float v_scale, int max_context_len, int staged_blocks, int q_dtype,
                    void *workspace, size_t workspace_bytes, struct CUstream_st *stream) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 ||
      max_blocks_per_seq <= 0)
    return PA_ERR_INVALID_ARG;
  if (!scale_ok(k_scale) || !scale_ok(v_scale)) return PA_ERR_INVALID_ARG;
  if (q_dtype != PA_F16 && q_dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  if (num_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
  const int group = num_heads / num_kv_heads;
  if (group > 16) return PA_ERR_UNSUPPORTED;
  if (num_seqs > decode_max_seqs_per_launch()) return PA_ERR_UNSUPPORTED;
  if (!query_start_loc) {
    if (num_q_tokens != num_seqs) return PA_ERR_INVALID_ARG;
    max_query_len = 1;
  } else if (max_query_len < 1 || num_q_tokens < num_seqs) {
    return PA_ERR_INVALID_ARG;
  }
  const bool chunk_rows = max_query_len > 1;
  if (staged_blocks < 0 || (chunk_rows && staged_blocks == 0)) return PA_ERR_INVALID_ARG;
  if (chunk_rows && group > 64) return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0 || num_q_tokens == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID_ARG;
  if (out == q) return PA_ERR_INVALID_ARG;
  if ((int64_t)max_blocks_per_seq * block_size > (int64_t)1 << 30) return PA_ERR_UNSUPPORTED;
  const int cap = max_blocks_per_seq * block_size;
  if (max_context_len <= 0 || max_context_len > cap) max_context_len = cap;

  DevInfo dev;
  if (device_info(&dev) != cudaSuccess) return PA_ERR_CUDA;
  AttnArgs a{};
  a.o_scale = 1.f;
  a.out = out;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.err = dev.err;
  a.num_seqs = num_seqs;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.group = group;
  a.head_dim = head_dim;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.split_blocks = 1;
  a.max_splits = 1;
  a.query_start_loc = query_start_loc;
  a.max_query_len = max_query_len;
  a.max_context_len = max_context_len;
  a.num_q_tokens = num_q_tokens;
  a.scale_log2 = scale * k_scale * 1.4426950408889634f;
  a.v_inv = 1.f / v_scale;
  a.balanced = 1;
  a.item_units = kItemUnitsFp8;
  a.grid = decode_mma_grid_fp8(a, q_dtype, dev.sm_count);
  if (a.grid <= 0) return PA_ERR_CUDA;
  const size_t rec = balanced_record_bytes(a.grid, group, head_dim);
  const size_t desc = balanced_desc_bytes(a.grid);
  const size_t need = rec + desc + (size_t)(num_seqs + 1) * sizeof(int);
  RowsWs w{};
  if (chunk_rows) {
    w = rows_ws(pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                         max_context_len, 0),
                num_seqs, num_kv_heads, head_dim, block_size, max_blocks_per_seq, staged_blocks);
    if (need > w.base) return PA_ERR_WORKSPACE;
  }
  if (!workspace || workspace_bytes < (chunk_rows ? w.total : need) || !aligned16(workspace))
    return PA_ERR_WORKSPACE;
  char *ws = static_cast<char *>(workspace);
  a.part_o = static_cast<float *>(workspace);
  a.bal_desc = reinterpret_cast<int *>(ws + rec);
  a.bal_prefix = reinterpret_cast<int *>(ws + rec + desc);
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaSuccess;
  // the chunk rows (staging + 16-bit chunk kernel) fork onto the library's
  // high-priority stream beside the decode rows, as in pa_decode
  SideStream *side = (chunk_rows && mixed_overlap_wanted()) ? side_fork(s) : nullptr;
  const cudaStream_t cs = side ? side->stream : s;
  a.no_pdl = side ? 1 : 0;
  if (chunk_rows) {
    int *base = reinterpret_cast<int *>(ws + w.base);
    int32_t *tab = reinterpret_cast<int32_t *>(ws + w.tab);
    fp8_stage_plan_kernel<<<1, 1024, 0, cs>>>(a, base, staged_blocks);
    e = cudaGetLastError();
    if (e == cudaSuccess)
      e = q_dtype == PA_BF16
              ? (head_dim == 64 ? launch_stage_t<__nv_bfloat16, 64>(a, base, tab, ws + w.k, ws + w.v, staged_blocks, cs)
                                : launch_stage_t<__nv_bfloat16, 128>(a, base, tab, ws + w.k, ws + w.v, staged_blocks, cs))
              : (head_dim == 64 ? launch_stage_t<__half, 64>(a, base, tab, ws + w.k, ws + w.v, staged_blocks, cs)
                                : launch_stage_t<__half, 128>(a, base, tab, ws + w.k, ws + w.v, staged_blocks, cs));
    if (e == cudaSuccess) {
      AttnArgs c = a;
      c.k_cache = ws + w.k;
      c.v_cache = ws + w.v;
      c.block_tables = tab;
      c.num_blocks = staged_blocks;
      c.o_scale = v_scale;
      c.seq_begin = 0;
      e = launch_chunk(c, q_dtype, num_q_tokens, cs);
    }
  }
  if (e == cudaSuccess) e = launch_decode_mma_fp8(a, q_dtype, dev.sm_count, s);
  if (e == cudaSuccess) e = launch_balanced_reduce(a, q_dtype, s);
  if (side) {
    const cudaError_t j = side_join(side, s);  // also after a failed launch
    if (e == cudaSuccess) e = j;
  }
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}


}  // namespace
}  // namespace pa

extern "C" {

int pa_reshape_and_cache_fp8(const void *key, const void *value, void *k_cache, void *v_cache,
                             const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                             int head_dim, int block_size, int num_blocks, int in_dtype,
                             float k_scale, float v_scale, struct CUstream_st *stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0) return PA_ERR_INVALID_ARG;
  if (in_dtype != PA_F32 && in_dtype != PA_F16 && in_dtype != PA_BF16) return PA_ERR_INVALID_ARG;
  if (!scale_ok(k_scale) || !scale_ok(v_scale)) return PA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
  if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID_ARG;
  DevInfo dev;
  if (device_info(&dev) != cudaSuccess) return PA_ERR_CUDA;
  const int64_t total = (int64_t)num_tokens * num_kv_heads * (head_dim / 16);
  int64_t blocks = (total + 255) / 256;
  if (blocks > (int64_t)dev.sm_count * 16) blocks = (int64_t)dev.sm_count * 16;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(256);
  cfg.stream = (cudaStream_t)stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int64_t slots = (int64_t)num_blocks * block_size;
  cudaError_t e;
  if (in_dtype == PA_F32)
    e = reshape_fp8_d<float>(head_dim, block_size, cfg, key, value, k_cache, v_cache, slot_mapping,
                             num_tokens, num_kv_heads, slots, k_scale, v_scale, dev.err);
  else if (in_dtype == PA_F16)
    e = reshape_fp8_d<__half>(head_dim, block_size, cfg, key, value, k_cache, v_cache,
                              slot_mapping, num_tokens, num_kv_heads, slots, k_scale, v_scale,
                              dev.err);
  else
    e = reshape_fp8_d<__nv_bfloat16>(head_dim, block_size, cfg, key, value, k_cache, v_cache,
                                     slot_mapping, num_tokens, num_kv_heads, slots, k_scale,
                                     v_scale, dev.err);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int pa_decode_fp8(void *out, const void *q, const void *k_cache, const void *v_cache,
                  const int32_t *block_tables, int max_blocks_per_seq,
                  const int32_t *context_lens, int num_seqs, int num_heads, int num_kv_heads,
                  int head_dim, int block_size, int num_blocks, float scale, float k_scale,
                  float v_scale, int max_context_len, int q_dtype, void *workspace,
                  size_t workspace_bytes, struct CUstream_st *stream) {
  return decode_fp8_call(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                         nullptr, num_seqs, num_seqs, 1, num_heads, num_kv_heads, head_dim,
                         block_size, num_blocks, scale, k_scale, v_scale, max_context_len, 0,
                         q_dtype, workspace, workspace_bytes, stream);
}

size_t pa_decode_fp8_rows_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                         int head_dim, int block_size, int max_context_len,
                                         int max_blocks_per_seq, int staged_blocks) {
  if (num_seqs <= 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      max_blocks_per_seq <= 0 || staged_blocks < 0 ||
      (int64_t)max_blocks_per_seq * block_size > (int64_t)1 << 30)
    return 0;
  const int cap = max_blocks_per_seq * block_size;
  if (max_context_len <= 0 || max_context_len > cap) max_context_len = cap;
  return rows_ws(pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                          max_context_len, 0),
                 num_seqs, num_kv_heads, head_dim, block_size, max_blocks_per_seq, staged_blocks)
      .total;
}

int pa_decode_fp8_rows(void *out, const void *q, const void *k_cache, const void *v_cache,
                       const int32_t *block_tables, int max_blocks_per_seq,
                       const int32_t *context_lens, const int32_t *query_start_loc, int num_seqs,
                       int num_q_tokens, int max_query_len, int num_heads, int num_kv_heads,
                       int head_dim, int block_size, int num_blocks, float scale, float k_scale,
                       float v_scale, int max_context_len, int staged_blocks, int q_dtype,
                       void *workspace, size_t workspace_bytes, struct CUstream_st *stream) {
  return decode_fp8_call(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                         query_start_loc, num_seqs, num_q_tokens, max_query_len, num_heads,
                         num_kv_heads, head_dim, block_size, num_blocks, scale, k_scale, v_scale,
                         max_context_len, staged_blocks, q_dtype, workspace, workspace_bytes, stream);
}

}  // extern "C"
