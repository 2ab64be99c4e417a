/*
 * pa_oracle.c -- plain, slow CPU oracle for paged KV-cache attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code, header, table or helper with the CUDA library; it reads host copies
 * of every input and computes in IEEE double precision.
 *
 * What it computes (each function cites the passage it follows):
 *
 *   Address translation.  A sequence's tokens are logically contiguous; token
 *   p of sequence i lives in physical block block_tables[i][p / bs] at offset
 *   p % bs of that block ("核心概念", section 逻辑视图与物理视图分离: the
 *   block table maps logical block index -> physical block index; worked
 *   table [5, 2, 8, 1] for tokens 0-63).
 *
 *   Attention.  The new token attends to every earlier token of its sequence
 *   and to itself; only the current token's Q/K/V are new, older K/V are read
 *   back from the cache ("核心概念", section KV Cache：推理的显存瓶颈 /
 *   为什么需要 KV Cache).  The pages give no formula, so the oracle takes the
 *   plain definition of scaled-dot-product attention:
 *       s_p = scale * sum_d q[d] * K[p][d]
 *       o   = sum_p exp(s_p - max s) * V[p] / sum_p exp(s_p - max s)
 *   For a chunk of Q query tokens of one sequence (chunked prefill,
 *   "PagedAttention 实战", section Chunked Prefill) row t (0-based) sees keys
 *   0 .. L - Q + t inclusive, L being the context length after the chunk was
 *   appended.  Decode is the case Q = 1.
 *
 *   GQA.  Query head h reads KV head h / (num_heads / num_kv_heads); the pages
 *   are silent on the head grouping and this is the plainest contiguous one.
 *
 *   reshape_and_cache.  New K/V of token t are written to slot
 *   slot_mapping[t] = block_table[pos / bs] * bs + pos % bs, i.e. block
 *   slot / bs, offset slot % bs; a negative slot means "no write".
 *
 *   copy_blocks.  Copy-on-write copy of whole blocks: every (src, dst) pair
 *   copies K and V of all KV heads; all reads happen before any write
 *   ("理解 vLLM PagedAttention", section 六: a shared block gets its own copy
 *   only when the sequences diverge, like copy-on-write).
 *
 * Cache layout, fixed by this project because the pages give none:
 *   k_cache, v_cache: [num_blocks][num_kv_heads][block_size][head_dim]
 *   key, value:       [num_tokens][num_kv_heads][head_dim]
 *   q, out:           [num_q_tokens][num_heads][head_dim]
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F32 = 0, ORACLE_F16 = 1, ORACLE_BF16 = 2, ORACLE_FP8_E4M3 = 3 };

enum {
  ORACLE_OK = 0,
  ORACLE_BAD_ARG = 1,
  ORACLE_BAD_BLOCK = 2,
  ORACLE_BAD_LEN = 3,
  ORACLE_BAD_SLOT = 4,
  ORACLE_NO_MEM = 5
};

/* IEEE binary16 bit pattern -> exact double. */
static double f16_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int expo = (h >> 10) & 0x1f;
  int mant = h & 0x3ff;
  double v;
  if (expo == 0)
    v = ldexp((double)mant, -24);                 /* subnormal: mant * 2^-24 */
  else if (expo == 31)
    v = mant ? NAN : INFINITY;
  else
    v = ldexp((double)(mant | 0x400), expo - 25); /* 1.mant * 2^(expo-15) */
  return sign ? -v : v;
}

/* bfloat16 is the top half of an IEEE binary32: exact via float. */
static double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/*
 * FP8 E4M3 (the "FN" variant: no infinities): 1 sign bit, 4 exponent bits
 * with bias 7, 3 mantissa bits.  Exponent field 0 holds subnormals
 * m * 2^-9; S.1111.111 is NaN; the largest finite magnitude is
 * 1.75 * 2^8 = 448.  Code -> exact double.
 */
static double e4m3_to_double(uint8_t c) {
  int sign = (c >> 7) & 1;
  int expo = (c >> 3) & 0xf;
  int mant = c & 7;
  double v;
  if (expo == 0xf && mant == 7)
    v = NAN;
  else if (expo == 0)
    v = ldexp((double)mant, -9);                /* subnormal: mant * 2^-9 */
  else
    v = ldexp((double)(8 + mant), expo - 10);   /* 1.mant * 2^(expo-7) */
  return sign ? -v : v;
}

/*
 * float -> E4M3 code: round to nearest, ties to the even code, magnitudes
 * beyond 448 saturated to +-448, NaN -> 0x7f.  Written as the plain
 * definition: of all finite non-negative codes (0x00 .. 0x7e, increasing in
 * value) take the one nearest |f|; on a tie the even one (its mantissa's low
 * bit is the code's low bit).  The sign bit is copied (so -0 -> 0x80).
 */
static uint8_t e4m3_from_float(float f) {
  uint8_t sign = signbit(f) ? 0x80 : 0x00;
  double a = fabs((double)f);
  int best = 0, c;
  double best_d;
  if (isnan(f)) return 0x7f;
  if (a >= 448.0) return (uint8_t)(sign | 0x7e);
  best_d = a;
  for (c = 1; c <= 0x7e; ++c) {
    double d = fabs(e4m3_to_double((uint8_t)c) - a);
    if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
      best = c;
      best_d = d;
    }
  }
  return (uint8_t)(sign | best);
}

static double elem(const void *base, int64_t idx, int dtype) {
  if (dtype == ORACLE_F32) return (double)((const float *)base)[idx];
  if (dtype == ORACLE_F16) return f16_to_double(((const uint16_t *)base)[idx]);
  if (dtype == ORACLE_FP8_E4M3) return e4m3_to_double(((const uint8_t *)base)[idx]);
  return bf16_to_double(((const uint16_t *)base)[idx]);
}

static int elem_bytes(int dtype) {
  return dtype == ORACLE_F32 ? 4 : (dtype == ORACLE_FP8_E4M3 ? 1 : 2);
}

/*
 * Layout of an FP8 cache tile (one block, one KV head), fixed by this project
 * (the pages give none) so that each thread of the device's products loads
 * its operands with one 16-byte (K) or 4/8-byte (V) read:
 *   K [block_size][head_dim] bytes: in every row r, column d = 64j + 16k + c
 *     (c < 16) is stored at byte (C ^ (r mod head_dim/16)) * 16 + 4k + i of
 *     the row, with t = (c mod 8) / 2, i = c mod 2 + 2 * (c / 8), C = 4j + t.
 *   V [head_dim][block_size] bytes (transposed): key r = 16k + c of column d
 *     is stored at byte d * block_size + 4t + i (block_size 16) or
 *     d * block_size + 8t + 4k + i (block_size 32), t and i from c as above.
 */
static int64_t fp8_k_pos(int r, int d, int head_dim) {
  int j = d / 64, w = d % 64, k = w / 16, c = w % 16;
  int t = (c % 8) / 2, i = c % 2 + 2 * (c / 8);
  int chunk = (4 * j + t) ^ (r % (head_dim / 16));
  return (int64_t)r * head_dim + chunk * 16 + 4 * k + i;
}

static int64_t fp8_v_pos(int r, int d, int block_size) {
  int k = r / 16, c = r % 16;
  int t = (c % 8) / 2, i = c % 2 + 2 * (c / 8);
  int pos = block_size == 16 ? 4 * t + i : 8 * t + 4 * k + i;
  return (int64_t)d * block_size + pos;
}

/* Exported for the pins: the codec alone. */
double oracle_e4m3_decode(uint8_t c) { return e4m3_to_double(c); }
uint8_t oracle_e4m3_encode(float f) { return e4m3_from_float(f); }

/*
 * One output row: query token `row` of sequence `seq`, query head `h`.
 * Writes head_dim doubles to out_row.  `kbuf`/`vbuf` are caller scratch of
 * n_vis * head_dim doubles and `sbuf` of n_vis doubles.
 */
static int attend_one(double *out_row, const void *q, int q_dtype, const void *k_cache,
                      const void *v_cache, int dtype, double k_scale, double v_scale,
                      const int32_t *table,
                      int n_vis, int64_t row, int h, int num_heads,
                      int num_kv_heads, int head_dim, int block_size,
                      int num_blocks, double scale, double *kbuf, double *vbuf,
                      double *sbuf) {
  int group = num_heads / num_kv_heads;
  int h_kv = h / group;
  int p, d;

  if (n_vis <= 0) { /* empty context: defined as a zero output */
    for (d = 0; d < head_dim; ++d) out_row[d] = 0.0;
    return ORACLE_OK;
  }

  /* Step 1: gather this sequence's visible K/V through its block table into
   * contiguous arrays (logical order). */
  for (p = 0; p < n_vis; ++p) {
    int32_t pb = table[p / block_size];
    int off = p % block_size;
    int64_t base;
    if (pb < 0 || pb >= num_blocks) return ORACLE_BAD_BLOCK;
    base = (((int64_t)pb * num_kv_heads + h_kv) * block_size + off) * head_dim;
    if (dtype == ORACLE_FP8_E4M3) { /* tile-internal layout above */
      int64_t tile = ((int64_t)pb * num_kv_heads + h_kv) * block_size * head_dim;
      for (d = 0; d < head_dim; ++d) {
        kbuf[(int64_t)p * head_dim + d] =
            elem(k_cache, tile + fp8_k_pos(off, d, head_dim), dtype) * k_scale;
        vbuf[(int64_t)p * head_dim + d] =
            elem(v_cache, tile + fp8_v_pos(off, d, block_size), dtype) * v_scale;
      }
      continue;
    }
    for (d = 0; d < head_dim; ++d) {
      kbuf[(int64_t)p * head_dim + d] = elem(k_cache, base + d, dtype) * k_scale;
      vbuf[(int64_t)p * head_dim + d] = elem(v_cache, base + d, dtype) * v_scale;
    }
  }

  /* Step 2: scores, max-shifted softmax, weighted sum of V. */
  {
    int64_t qbase = (row * num_heads + h) * (int64_t)head_dim;
    double m = -INFINITY, denom = 0.0;
    for (p = 0; p < n_vis; ++p) {
      double s = 0.0;
      for (d = 0; d < head_dim; ++d)
        s += elem(q, qbase + d, q_dtype) * kbuf[(int64_t)p * head_dim + d];
      s *= scale;
      sbuf[p] = s;
      if (s > m) m = s;
    }
    for (p = 0; p < n_vis; ++p) {
      sbuf[p] = exp(sbuf[p] - m);
      denom += sbuf[p];
    }
    for (d = 0; d < head_dim; ++d) {
      double acc = 0.0;
      for (p = 0; p < n_vis; ++p) acc += sbuf[p] * vbuf[(int64_t)p * head_dim + d];
      out_row[d] = acc / denom;
    }
  }
  return ORACLE_OK;
}

/*
 * Paged attention over the block-table cache.
 *
 *   out              [num_q_tokens][num_heads][head_dim] doubles
 *   query_start_loc  [num_seqs + 1] or NULL; NULL means one query token per
 *                    sequence (query row i belongs to sequence i)
 *   row_select       [num_q_tokens] or NULL; if given, rows with 0 are not
 *                    computed (their output is left untouched)
 *   num_threads      <= 0: library default
 */
static int decode_impl(double *out, const void *q, int q_dtype, const void *k_cache,
                       const void *v_cache, int dtype, double k_scale, double v_scale,
                       const int32_t *block_tables,
                       int max_blocks_per_seq, const int32_t *context_lens,
                       const int32_t *query_start_loc, int num_seqs, int num_heads,
                       int num_kv_heads, int head_dim, int block_size,
                       int num_blocks, double scale, const uint8_t *row_select,
                       int num_threads) {
  int64_t num_q_tokens;
  int64_t *task_row;
  int32_t *task_seq;
  int64_t ntasks = 0;
  int status = ORACLE_OK;
  int i;

  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      block_size <= 0 || num_heads % num_kv_heads != 0)
    return ORACLE_BAD_ARG;
  if (dtype != ORACLE_F32 && dtype != ORACLE_F16 && dtype != ORACLE_BF16 &&
      dtype != ORACLE_FP8_E4M3)
    return ORACLE_BAD_ARG;
  if (q_dtype != ORACLE_F32 && q_dtype != ORACLE_F16 && q_dtype != ORACLE_BF16)
    return ORACLE_BAD_ARG;

  num_q_tokens = query_start_loc ? query_start_loc[num_seqs] : num_seqs;
  for (i = 0; i < num_seqs; ++i) {
    int64_t q0 = query_start_loc ? query_start_loc[i] : i;
    int64_t q1 = query_start_loc ? query_start_loc[i + 1] : i + 1;
    if (q1 < q0) return ORACLE_BAD_LEN;
    if (context_lens[i] < 0 ||
        context_lens[i] > (int64_t)max_blocks_per_seq * block_size)
      return ORACLE_BAD_LEN;
    if (q1 - q0 > context_lens[i] && context_lens[i] > 0) return ORACLE_BAD_LEN;
  }

  task_row = (int64_t *)malloc(sizeof(int64_t) * (size_t)(num_q_tokens + 1));
  task_seq = (int32_t *)malloc(sizeof(int32_t) * (size_t)(num_q_tokens + 1));
  if (!task_row || !task_seq) {
    free(task_row);
    free(task_seq);
    return ORACLE_NO_MEM;
  }
  for (i = 0; i < num_seqs; ++i) {
    int64_t q0 = query_start_loc ? query_start_loc[i] : i;
    int64_t q1 = query_start_loc ? query_start_loc[i + 1] : i + 1;
    int64_t r;
    for (r = q0; r < q1; ++r) {
      if (row_select && !row_select[r]) continue;
      task_row[ntasks] = r;
      task_seq[ntasks] = i;
      ++ntasks;
    }
  }

#ifdef _OPENMP
  if (num_threads > 0) omp_set_num_threads(num_threads);
#endif

#pragma omp parallel
  {
    double *kbuf = NULL, *vbuf = NULL, *sbuf = NULL;
    int cap = -1;
    int64_t task;
#pragma omp for schedule(dynamic, 1)
    for (task = 0; task < ntasks * num_heads; ++task) {
      int64_t k = task / num_heads;
      int h = (int)(task % num_heads);
      int seq = task_seq[k];
      int64_t row = task_row[k];
      int64_t q0 = query_start_loc ? query_start_loc[seq] : seq;
      int64_t q1 = query_start_loc ? query_start_loc[seq + 1] : seq + 1;
      int64_t qlen = q1 - q0;
      int64_t tq = row - q0;
      /* visible keys: 0 .. L - Q + t inclusive */
      int n_vis = (int)(context_lens[seq] - qlen + tq + 1);
      int rc;
      if (context_lens[seq] == 0) n_vis = 0;
      if (n_vis > cap) {
        free(kbuf);
        free(vbuf);
        free(sbuf);
        cap = n_vis;
        kbuf = (double *)malloc(sizeof(double) * (size_t)(cap > 0 ? cap : 1) * head_dim);
        vbuf = (double *)malloc(sizeof(double) * (size_t)(cap > 0 ? cap : 1) * head_dim);
        sbuf = (double *)malloc(sizeof(double) * (size_t)(cap > 0 ? cap : 1));
      }
      if (!kbuf || !vbuf || !sbuf) {
#pragma omp atomic write
        status = ORACLE_NO_MEM;
        cap = -1;
        continue;
      }
      rc = attend_one(out + (row * num_heads + h) * (int64_t)head_dim, q, q_dtype, k_cache,
                      v_cache, dtype, k_scale, v_scale,
                      block_tables + (int64_t)seq * max_blocks_per_seq, n_vis,
                      row, h, num_heads, num_kv_heads, head_dim, block_size,
                      num_blocks, scale, kbuf, vbuf, sbuf);
      if (rc != ORACLE_OK) {
#pragma omp atomic write
        status = rc;
      }
    }
    free(kbuf);
    free(vbuf);
    free(sbuf);
  }
  free(task_row);
  free(task_seq);
  return status;
}

int oracle_decode(double *out, const void *q, const void *k_cache,
                  const void *v_cache, int dtype, const int32_t *block_tables,
                  int max_blocks_per_seq, const int32_t *context_lens,
                  const int32_t *query_start_loc, int num_seqs, int num_heads,
                  int num_kv_heads, int head_dim, int block_size,
                  int num_blocks, double scale, const uint8_t *row_select,
                  int num_threads) {
  return decode_impl(out, q, dtype, k_cache, v_cache, dtype, 1.0, 1.0, block_tables,
                     max_blocks_per_seq, context_lens, query_start_loc, num_seqs, num_heads,
                     num_kv_heads, head_dim, block_size, num_blocks, scale, row_select,
                     num_threads);
}

/*
 * Paged attention over an FP8 (E4M3) cache with one scale per cache tensor:
 * key element = code value * k_scale, value element = code value * v_scale
 * (KV-cache quantisation, "理解 vLLM PagedAttention", 版本矩阵: 量化 FP8 ...
 * 权重 KV cache 量化).  q (q_dtype) and everything else as oracle_decode.
 */
int oracle_decode_fp8(double *out, const void *q, int q_dtype, const uint8_t *k_codes,
                      const uint8_t *v_codes, double k_scale, double v_scale,
                      const int32_t *block_tables, int max_blocks_per_seq,
                      const int32_t *context_lens, const int32_t *query_start_loc,
                      int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                      int block_size, int num_blocks, double scale,
                      const uint8_t *row_select, int num_threads) {
  return decode_impl(out, q, q_dtype, k_codes, v_codes, ORACLE_FP8_E4M3, k_scale, v_scale,
                     block_tables, max_blocks_per_seq, context_lens, query_start_loc, num_seqs,
                     num_heads, num_kv_heads, head_dim, block_size, num_blocks, scale,
                     row_select, num_threads);
}

/*
 * reshape_and_cache: scatter each new token's K/V rows into its slot.
 * Byte copies; the result must match the GPU pool byte for byte.
 */
int oracle_reshape_and_cache(void *k_cache, void *v_cache, const void *key,
                             const void *value, const int64_t *slot_mapping,
                             int num_tokens, int num_kv_heads, int head_dim,
                             int block_size, int num_blocks, int dtype) {
  int e = elem_bytes(dtype);
  int64_t row_bytes = (int64_t)head_dim * e;
  int t, h;
  for (t = 0; t < num_tokens; ++t) {
    int64_t slot = slot_mapping[t];
    int64_t blk, off;
    if (slot < 0) continue; /* padding token: nothing to write */
    if (slot >= (int64_t)num_blocks * block_size) return ORACLE_BAD_SLOT;
    blk = slot / block_size;
    off = slot % block_size;
    for (h = 0; h < num_kv_heads; ++h) {
      int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * row_bytes;
      int64_t src = ((int64_t)t * num_kv_heads + h) * row_bytes;
      memcpy((char *)k_cache + dst, (const char *)key + src, (size_t)row_bytes);
      memcpy((char *)v_cache + dst, (const char *)value + src, (size_t)row_bytes);
    }
  }
  return ORACLE_OK;
}

/*
 * reshape_and_cache into an FP8 (E4M3) cache: the element x of key token t
 * (in_dtype) is stored as the code of x / k_scale, values likewise with
 * v_scale (KV-cache quantisation, "理解 vLLM PagedAttention", 版本矩阵).  The
 * division is one IEEE binary32 division (float / float) and the rounding to
 * E4M3 is done from that binary32 result, which is the precision the device
 * quantiser works in; slots as oracle_reshape_and_cache, positions inside the
 * (block, head) tile as fp8_k_pos / fp8_v_pos.
 */
int oracle_reshape_and_cache_fp8(uint8_t *k_codes, uint8_t *v_codes, const void *key,
                                 const void *value, int in_dtype, const int64_t *slot_mapping,
                                 int num_tokens, int num_kv_heads, int head_dim, int block_size,
                                 int num_blocks, float k_scale, float v_scale) {
  int t, h, d;
  if (in_dtype != ORACLE_F32 && in_dtype != ORACLE_F16 && in_dtype != ORACLE_BF16)
    return ORACLE_BAD_ARG;
  for (t = 0; t < num_tokens; ++t) {
    int64_t slot = slot_mapping[t];
    int64_t blk, off;
    if (slot < 0) continue;
    if (slot >= (int64_t)num_blocks * block_size) return ORACLE_BAD_SLOT;
    blk = slot / block_size;
    off = slot - blk * block_size;
    for (h = 0; h < num_kv_heads; ++h) {
      int64_t tile = (blk * num_kv_heads + h) * block_size * head_dim;
      int64_t src = ((int64_t)t * num_kv_heads + h) * head_dim;
      for (d = 0; d < head_dim; ++d) {
        float kx = (float)elem(key, src + d, in_dtype);
        float vx = (float)elem(value, src + d, in_dtype);
        k_codes[tile + fp8_k_pos((int)off, d, head_dim)] = e4m3_from_float(kx / k_scale);
        v_codes[tile + fp8_v_pos((int)off, d, block_size)] = e4m3_from_float(vx / v_scale);
      }
    }
  }
  return ORACLE_OK;
}

/*
 * copy_blocks: block_mapping holds num_pairs (src, dst) pairs.  All source
 * blocks are read into a staging buffer before any destination is written.
 */
int oracle_copy_blocks(void *k_cache, void *v_cache,
                       const int64_t *block_mapping, int num_pairs,
                       int num_kv_heads, int head_dim, int block_size,
                       int num_blocks, int dtype) {
  int64_t blk_bytes = (int64_t)num_kv_heads * block_size * head_dim * elem_bytes(dtype);
  char *stage_k, *stage_v;
  int i;
  for (i = 0; i < num_pairs; ++i) {
    int64_t s = block_mapping[2 * i], d = block_mapping[2 * i + 1];
    if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks) return ORACLE_BAD_BLOCK;
  }
  if (num_pairs == 0) return ORACLE_OK;
  stage_k = (char *)malloc((size_t)(blk_bytes * num_pairs));
  stage_v = (char *)malloc((size_t)(blk_bytes * num_pairs));
  if (!stage_k || !stage_v) {
    free(stage_k);
    free(stage_v);
    return ORACLE_NO_MEM;
  }
  for (i = 0; i < num_pairs; ++i) {
    int64_t s = block_mapping[2 * i];
    memcpy(stage_k + i * blk_bytes, (const char *)k_cache + s * blk_bytes, (size_t)blk_bytes);
    memcpy(stage_v + i * blk_bytes, (const char *)v_cache + s * blk_bytes, (size_t)blk_bytes);
  }
  for (i = 0; i < num_pairs; ++i) {
    int64_t d = block_mapping[2 * i + 1];
    memcpy((char *)k_cache + d * blk_bytes, stage_k + i * blk_bytes, (size_t)blk_bytes);
    memcpy((char *)v_cache + d * blk_bytes, stage_v + i * blk_bytes, (size_t)blk_bytes);
  }
  free(stage_k);
  free(stage_v);
  return ORACLE_OK;
}

/*
 * swap_blocks: move whole blocks from one pool to another (the GPU tier and
 * the CPU tier of a tiered KV cache, "核心概念", section 内存层次结构).  For
 * pair i, destination block dst_i of (dst_k, dst_v) receives the bytes of
 * source block src_i of (src_k, src_v).  Every pair is checked before anything
 * is written.  The two pools are distinct arrays, so the order of the pairs
 * does not matter.
 */
int oracle_swap_blocks(void *dst_k, void *dst_v, const void *src_k, const void *src_v,
                       const int64_t *block_mapping, int num_pairs, int num_kv_heads,
                       int head_dim, int block_size, int num_src_blocks, int num_dst_blocks,
                       int dtype) {
  int64_t blk_bytes = (int64_t)num_kv_heads * block_size * head_dim * elem_bytes(dtype);
  int i;
  for (i = 0; i < num_pairs; ++i) {
    int64_t s = block_mapping[2 * i], d = block_mapping[2 * i + 1];
    if (s < 0 || s >= num_src_blocks || d < 0 || d >= num_dst_blocks) return ORACLE_BAD_BLOCK;
  }
  for (i = 0; i < num_pairs; ++i) {
    int64_t s = block_mapping[2 * i], d = block_mapping[2 * i + 1];
    memcpy((char *)dst_k + d * blk_bytes, (const char *)src_k + s * blk_bytes, (size_t)blk_bytes);
    memcpy((char *)dst_v + d * blk_bytes, (const char *)src_v + s * blk_bytes, (size_t)blk_bytes);
  }
  return ORACLE_OK;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
