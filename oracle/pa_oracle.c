/*
 * pa_oracle.c -- the oracle for the paged KV-cache hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file; only the tests, the smoke check and the benchmark's CPU
 * baseline do.  It shares no code with the CUDA library: it has its own
 * 16-bit float decoders, its own slot arithmetic and its own attention.
 *
 * Plain C, fp64 arithmetic, no fast-math, no blocking, no fusion.  Each
 * function restates one step as the pages describe it:
 *
 *   orc_slot_mapping      "PagedAttention" (shubhamtatvamasi), "How attention
 *                         reads paged memory" + the block-size-4 figure:
 *                         entry i of a block table names the physical block
 *                         that holds the sequence's logical block i; token p
 *                         sits in logical block p / block_size at offset
 *                         p % block_size.
 *   orc_reshape_and_cache "How PagedAttention Works in vLLM to Maximize
 *                         Memory Efficiency", "write_to_paged_cache: Direct
 *                         In-Place Updates" and "Code Example": new K/V rows
 *                         [num_tokens, num_kv_heads, head_size] are scattered
 *                         into the pool at the flat slots of slot_mapping.
 *   orc_copy_blocks       "PagedAttention", "How does copy-on-write work for
 *                         parallel sampling?": allocate a block, copy the
 *                         shared block's contents into it.
 *   orc_decode            "PagedAttention", "How attention reads paged
 *                         memory": for each query token walk the sequence's
 *                         block table, gather every block's keys and values,
 *                         and run attention over them.  The oracle gathers
 *                         into one contiguous buffer and evaluates plain
 *                         softmax(scale * q K^T) V in double precision (the
 *                         exact quantity that an online softmax reaches up to
 *                         rounding order).
 *   orc_decode_multi      the same walk for several query tokens of one
 *                         sequence ("PagedAttention", "Sharing and
 *                         copy-on-write": a child request recomputes the
 *                         tokens of its partial last block over the shared
 *                         prompt blocks).  The causal rule is the decoder's,
 *                         not the pages': query token i of the last n attends
 *                         the first L - n + i + 1 tokens.
 *
 * Pool layout (one tensor for K, one for V):
 *   [num_blocks, block_size, num_kv_heads, head_dim]  -- "PagedAttention",
 *   "How attention reads paged memory"; the same as one half of the flash
 *   layout (2, num_blocks, block_size, num_kv_heads, head_size) on the vLLM
 *   page, "Flash Layout: The Canonical Storage Format".
 *
 * Readings where the pages are silent (grouped-query head mapping, empty
 * sequences) are stated at the function that takes them.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F16 0
#define ORC_BF16 1

/* ---------------------------------------------------------------------------
 * 16-bit float decoders, written from the IEEE 754 binary16 definition and
 * the bfloat16 definition (the upper half of an IEEE binary32).
 * ------------------------------------------------------------------------- */
double orc_half_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int m = h & 0x3ff;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -24); /* subnormal: m * 2^-14 * 2^-10 */
  } else if (e == 31) {
    v = (m == 0) ? INFINITY : NAN;
  } else {
    v = ldexp((double)(1024 + m), e - 25); /* (1 + m/2^10) * 2^(e-15) */
  }
  return sign ? -v : v;
}

double orc_bf16_to_double(uint16_t b) {
  int sign = (b >> 15) & 1;
  int e = (b >> 7) & 0xff;
  int m = b & 0x7f;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -133); /* subnormal: m * 2^-126 * 2^-7 */
  } else if (e == 255) {
    v = (m == 0) ? INFINITY : NAN;
  } else {
    v = ldexp((double)(128 + m), e - 134); /* (1 + m/2^7) * 2^(e-127) */
  }
  return sign ? -v : v;
}

/* ---------------------------------------------------------------------------
 * 8-bit float, E4M3 variant of the OCP 8-bit floating point formats: 1 sign
 * bit, 4 exponent bits (bias 7), 3 mantissa bits, no infinities, one NaN
 * pattern per sign (exponent and mantissa all ones); the largest finite value
 * is 448 and the smallest subnormal 2^-9.
 * ------------------------------------------------------------------------- */
double orc_e4m3_to_double(uint8_t c) {
  int sign = (c >> 7) & 1;
  int e = (c >> 3) & 0xf;
  int m = c & 0x7;
  double v;
  if (e == 15 && m == 7) {
    v = NAN;
  } else if (e == 0) {
    v = ldexp((double)m, -9); /* m/8 * 2^(1-7) */
  } else {
    v = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
  }
  return sign ? -v : v;
}

/* Nearest E4M3 code to the float x, ties to the even code, finite values
 * beyond 448 saturate to +-448; NaN gives the NaN code.  Written as a search
 * over the 127 non-negative finite codes, which are ordered by value. */
uint8_t orc_float_to_e4m3(float x) {
  if (x != x) return 0x7f;
  uint8_t sign = (x < 0.0f || (x == 0.0f && signbit(x))) ? 0x80 : 0x00;
  double a = fabs((double)x);
  if (a >= 448.0) return sign | 0x7e;
  uint8_t best = 0;
  double best_err = INFINITY;
  for (int c = 0; c <= 0x7e; ++c) {
    double err = fabs(orc_e4m3_to_double((uint8_t)c) - a);
    if (err < best_err || (err == best_err && (c & 1) == 0)) {
      best = (uint8_t)c;
      best_err = err;
    }
  }
  return sign | best;
}

/* reshape_and_cache into an fp8 cache: the code of key[t, h, d] / k_scale,
 * the quotient taken in float (single precision), as the cache stores it. */
void orc_reshape_and_cache_fp8(const uint16_t* key, const uint16_t* value,
                               int64_t key_stride_t, int64_t value_stride_t,
                               uint8_t* key_cache, uint8_t* value_cache,
                               const int32_t* slot_mapping, int64_t num_tokens,
                               int32_t block_size, int32_t num_kv_heads,
                               int32_t head_dim, int32_t dtype, float k_scale,
                               float v_scale);

static double orc_decode16(uint16_t bits, int dtype) {
  return dtype == ORC_BF16 ? orc_bf16_to_double(bits) : orc_half_to_double(bits);
}

/* ---------------------------------------------------------------------------
 * Slot of token position `pos` of a sequence whose block-table row is
 * `table_row`: the physical block holding logical block pos / block_size,
 * times block_size, plus the offset pos % block_size.
 * ------------------------------------------------------------------------- */
int64_t orc_slot_of(const int32_t* table_row, int64_t pos, int32_t block_size) {
  int64_t logical_block = pos / block_size;
  int64_t offset = pos % block_size;
  return (int64_t)table_row[logical_block] * block_size + offset;
}

/* slots[i] = slot of position pos[i] of sequence seq_idx[i]; the table is
 * row-major with `table_stride` entries per sequence. */
void orc_slot_mapping(const int32_t* block_tables, int64_t table_stride,
                      const int32_t* seq_idx, const int32_t* pos, int64_t n,
                      int32_t block_size, int64_t* slots) {
  for (int64_t i = 0; i < n; ++i) {
    const int32_t* row = block_tables + (int64_t)seq_idx[i] * table_stride;
    slots[i] = orc_slot_of(row, pos[i], block_size);
  }
}

/* ---------------------------------------------------------------------------
 * reshape_and_cache: for every new token t whose slot s = slot_mapping[t] is
 * non-negative, copy key[t, h, :] to key_cache[s / bs, s % bs, h, :] for every
 * KV head h, and the same for the values.  A negative slot is a padding token
 * and writes nothing.  The copy is of the raw 16-bit words, so the cache ends
 * up bit-identical to the input rows.
 * key/value rows are `key_stride_t` / `value_stride_t` elements apart.
 * ------------------------------------------------------------------------- */
void orc_reshape_and_cache(const uint16_t* key, const uint16_t* value,
                           int64_t key_stride_t, int64_t value_stride_t,
                           uint16_t* key_cache, uint16_t* value_cache,
                           const int32_t* slot_mapping, int64_t num_tokens,
                           int32_t block_size, int32_t num_kv_heads,
                           int32_t head_dim) {
  for (int64_t t = 0; t < num_tokens; ++t) {
    int64_t s = slot_mapping[t];
    if (s < 0) continue;
    int64_t block = s / block_size;
    int64_t offset = s % block_size;
    for (int32_t h = 0; h < num_kv_heads; ++h) {
      int64_t dst = ((block * block_size + offset) * num_kv_heads + h) * head_dim;
      for (int32_t d = 0; d < head_dim; ++d) {
        key_cache[dst + d] = key[t * key_stride_t + (int64_t)h * head_dim + d];
        value_cache[dst + d] = value[t * value_stride_t + (int64_t)h * head_dim + d];
      }
    }
  }
}

void orc_reshape_and_cache_fp8(const uint16_t* key, const uint16_t* value,
                               int64_t key_stride_t, int64_t value_stride_t,
                               uint8_t* key_cache, uint8_t* value_cache,
                               const int32_t* slot_mapping, int64_t num_tokens,
                               int32_t block_size, int32_t num_kv_heads,
                               int32_t head_dim, int32_t dtype, float k_scale,
                               float v_scale) {
  for (int64_t t = 0; t < num_tokens; ++t) {
    int64_t s = slot_mapping[t];
    if (s < 0) continue;
    int64_t block = s / block_size;
    int64_t offset = s % block_size;
    for (int32_t h = 0; h < num_kv_heads; ++h) {
      int64_t dst = ((block * block_size + offset) * num_kv_heads + h) * head_dim;
      for (int32_t d = 0; d < head_dim; ++d) {
        float k = (float)orc_decode16(key[t * key_stride_t + (int64_t)h * head_dim + d], dtype);
        float v = (float)orc_decode16(value[t * value_stride_t + (int64_t)h * head_dim + d], dtype);
        key_cache[dst + d] = orc_float_to_e4m3(k / k_scale);
        value_cache[dst + d] = orc_float_to_e4m3(v / v_scale);
      }
    }
  }
}

/* ---------------------------------------------------------------------------
 * copy_blocks (copy-on-write): for every (src, dst) pair, the whole physical
 * block dst of every layer's K and V pool becomes a byte copy of block src.
 * `caches` holds 2 * num_layers base pointers: K of layer 0, V of layer 0,
 * K of layer 1, ...
 * ------------------------------------------------------------------------- */
void orc_copy_blocks(uint8_t* const* caches, int32_t num_layers,
                     const int32_t* block_mapping, int64_t num_pairs,
                     int64_t block_bytes) {
  for (int64_t i = 0; i < num_pairs; ++i) {
    int64_t src = block_mapping[2 * i];
    int64_t dst = block_mapping[2 * i + 1];
    for (int32_t c = 0; c < 2 * num_layers; ++c) {
      memcpy(caches[c] + dst * block_bytes, caches[c] + src * block_bytes,
             (size_t)block_bytes);
    }
  }
}

/* ---------------------------------------------------------------------------
 * Decode attention, one query token per sequence.
 *
 *   out[b, h, :] = sum_t p_t V_b[t] / sum_t p_t,
 *   p_t = exp(s_t - max_u s_u),  s_t = scale * <q[b, h, :], K_b[t]>,
 *
 * where K_b, V_b are sequence b's first seq_lens[b] tokens gathered through
 * its block table into contiguous buffers.
 *
 * Readings where the pages are silent:
 *  - grouped-query attention: query head h reads KV head h / (Hq / Hkv)
 *    (consecutive query heads share one KV head);
 *  - a sequence with seq_len 0 attends to nothing: its output is all zeros.
 * Inputs q [B, Hq, D] and the pools hold 16-bit floats (`dtype`); the output
 * is double [B, Hq, D].  Sequences are independent, so `nthreads` worker
 * threads take whole sequences; the arithmetic per sequence is unchanged.
 * ------------------------------------------------------------------------- */
typedef struct {
  double* out;
  const uint16_t* q;
  const uint16_t* key_cache;
  const uint16_t* value_cache;
  const uint8_t* key_cache8;   /* fp8 cache (when not NULL, instead of the 16-bit ones) */
  const uint8_t* value_cache8;
  double k_scale, v_scale;
  const int32_t* block_tables;
  int64_t table_stride;
  const int32_t* seq_lens;
  const int32_t* q_start;      /* multi-query: rows q_start[b] .. q_start[b+1]-1, else NULL */
  int32_t num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, dtype;
  double scale;
  int32_t next_seq; /* work counter, guarded by mu */
  pthread_mutex_t mu;
  int32_t failed;
} orc_decode_job;

static int orc_decode_one(orc_decode_job* j, int32_t b) {
  const int32_t Hq = j->num_q_heads, Hkv = j->num_kv_heads, D = j->head_dim;
  const int32_t bs = j->block_size;
  const int32_t group = Hq / Hkv;
  const int64_t L = j->seq_lens[b];
  if (L <= 0) {  /* every query row of the sequence attends to nothing */
    const int64_t r0 = j->q_start ? j->q_start[b] : b;
    const int64_t nq = j->q_start ? (int64_t)j->q_start[b + 1] - j->q_start[b] : 1;
    for (int64_t i = 0; i < nq * Hq * D; ++i) j->out[r0 * Hq * D + i] = 0.0;
    return 0;
  }
  const int32_t* row = j->block_tables + (int64_t)b * j->table_stride;
  /* Gather this sequence's K and V into contiguous [L, Hkv, D] buffers. */
  double* Kc = (double*)malloc(sizeof(double) * (size_t)(L * Hkv * D));
  double* Vc = (double*)malloc(sizeof(double) * (size_t)(L * Hkv * D));
  double* s = (double*)malloc(sizeof(double) * (size_t)L);
  if (!Kc || !Vc || !s) {
    free(Kc); free(Vc); free(s);
    return 1;
  }
  for (int64_t t = 0; t < L; ++t) {
    int64_t slot = orc_slot_of(row, t, bs);
    for (int32_t g = 0; g < Hkv; ++g) {
      for (int32_t d = 0; d < D; ++d) {
        int64_t src = (slot * Hkv + g) * D + d;
        if (j->key_cache8) {
          Kc[(t * Hkv + g) * D + d] = orc_e4m3_to_double(j->key_cache8[src]) * j->k_scale;
          Vc[(t * Hkv + g) * D + d] = orc_e4m3_to_double(j->value_cache8[src]) * j->v_scale;
        } else {
          Kc[(t * Hkv + g) * D + d] = orc_decode16(j->key_cache[src], j->dtype);
          Vc[(t * Hkv + g) * D + d] = orc_decode16(j->value_cache[src], j->dtype);
        }
      }
    }
  }
  /* query rows of this sequence: one (row b) or q_start[b] .. q_start[b+1]-1;
   * query i of n attends the first L - n + i + 1 tokens (its own position and
   * everything before it) */
  const int64_t r0 = j->q_start ? j->q_start[b] : b;
  const int64_t nq = j->q_start ? (int64_t)j->q_start[b + 1] - j->q_start[b] : 1;
  for (int64_t i = 0; i < nq; ++i) {
    const int64_t r = r0 + i;
    int64_t n = j->q_start ? L - nq + i + 1 : L;
    if (n > L) n = L;
    double* outr = j->out + r * Hq * D;
    if (n <= 0) {
      for (int64_t e = 0; e < (int64_t)Hq * D; ++e) outr[e] = 0.0;
      continue;
    }
    for (int32_t h = 0; h < Hq; ++h) {
      const int32_t g = h / group;
      const uint16_t* qh = j->q + (r * Hq + h) * D;
      double m = -INFINITY;
      for (int64_t t = 0; t < n; ++t) {
        double dot = 0.0;
        for (int32_t d = 0; d < D; ++d)
          dot += orc_decode16(qh[d], j->dtype) * Kc[(t * Hkv + g) * D + d];
        s[t] = j->scale * dot;
        if (s[t] > m) m = s[t];
      }
      double denom = 0.0;
      for (int64_t t = 0; t < n; ++t) {
        s[t] = exp(s[t] - m);
        denom += s[t];
      }
      for (int32_t d = 0; d < D; ++d) {
        double acc = 0.0;
        for (int64_t t = 0; t < n; ++t) acc += s[t] * Vc[(t * Hkv + g) * D + d];
        outr[(int64_t)h * D + d] = acc / denom;
      }
    }
  }
  free(Kc); free(Vc); free(s);
  return 0;
}

static void* orc_decode_worker(void* arg) {
  orc_decode_job* j = (orc_decode_job*)arg;
  for (;;) {
    pthread_mutex_lock(&j->mu);
    int32_t b = j->next_seq++;
    pthread_mutex_unlock(&j->mu);
    if (b >= j->num_seqs) break;
    if (orc_decode_one(j, b)) {
      pthread_mutex_lock(&j->mu);
      j->failed = 1;
      pthread_mutex_unlock(&j->mu);
    }
  }
  return NULL;
}

/* Returns 0 on success, 1 on allocation failure, 2 on a bad argument.
 * With key_cache8 / value_cache8 not NULL the cache holds E4M3 codes and a
 * stored element reads as code * k_scale (keys) or code * v_scale (values);
 * the query keeps its 16-bit type (dtype). */
static int orc_decode_impl(double* out, const uint16_t* q, const int32_t* q_start,
                           const uint16_t* key_cache,
                           const uint16_t* value_cache, const uint8_t* key_cache8,
                           const uint8_t* value_cache8, double k_scale, double v_scale,
                           const int32_t* block_tables, int64_t table_stride,
                           const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                           int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                           double scale, int32_t dtype, int32_t nthreads) {
  if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 || block_size <= 0)
    return 2;
  orc_decode_job j;
  j.key_cache8 = key_cache8; j.value_cache8 = value_cache8;
  j.k_scale = k_scale; j.v_scale = v_scale;
  j.out = out; j.q = q; j.key_cache = key_cache; j.value_cache = value_cache;
  j.block_tables = block_tables; j.table_stride = table_stride;
  j.seq_lens = seq_lens; j.q_start = q_start;
  j.num_seqs = num_seqs; j.num_q_heads = num_q_heads;
  j.num_kv_heads = num_kv_heads; j.head_dim = head_dim;
  j.block_size = block_size; j.dtype = dtype; j.scale = scale;
  j.next_seq = 0; j.failed = 0;
  pthread_mutex_init(&j.mu, NULL);
  if (nthreads <= 1) {
    orc_decode_worker(&j);
  } else {
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!th) { pthread_mutex_destroy(&j.mu); return 1; }
    for (int32_t i = 0; i < nthreads; ++i)
      pthread_create(&th[i], NULL, orc_decode_worker, &j);
    for (int32_t i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
  }
  pthread_mutex_destroy(&j.mu);
  return j.failed ? 1 : 0;
}

int orc_decode(double* out, const uint16_t* q, const uint16_t* key_cache,
               const uint16_t* value_cache, const int32_t* block_tables,
               int64_t table_stride, const int32_t* seq_lens, int32_t num_seqs,
               int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
               int32_t block_size, double scale, int32_t dtype,
               int32_t nthreads) {
  return orc_decode_impl(out, q, NULL, key_cache, value_cache, NULL, NULL, 1.0, 1.0,
                         block_tables, table_stride, seq_lens, num_seqs, num_q_heads,
                         num_kv_heads, head_dim, block_size, scale, dtype, nthreads);
}

int orc_decode_fp8(double* out, const uint16_t* q, const uint8_t* key_cache,
                   const uint8_t* value_cache, double k_scale, double v_scale,
                   const int32_t* block_tables, int64_t table_stride,
                   const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                   int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                   double scale, int32_t q_dtype, int32_t nthreads) {
  return orc_decode_impl(out, q, NULL, NULL, NULL, key_cache, value_cache, k_scale, v_scale,
                         block_tables, table_stride, seq_lens, num_seqs, num_q_heads,
                         num_kv_heads, head_dim, block_size, scale, q_dtype, nthreads);
}

/* Multi-query paged attention (several new tokens per sequence, as in a chunk
 * of prefill or the verification of speculated tokens): sequence b owns query
 * rows q_start[b] .. q_start[b+1]-1 of q [T, Hq, D] (its last n = q_len tokens,
 * whose K and V are already in the cache), and query i of them attends, like
 * any token of a causal decoder, to the tokens at positions 0 .. L_b - n + i.
 * out is double [T, Hq, D].  A query that would attend nothing (q_len > L_b)
 * gets zeros.  Same pools and readings as orc_decode. */
int orc_decode_multi(double* out, const uint16_t* q, const int32_t* q_start,
                     const uint16_t* key_cache, const uint16_t* value_cache,
                     const int32_t* block_tables, int64_t table_stride,
                     const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                     int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                     double scale, int32_t dtype, int32_t nthreads) {
  if (!q_start) return 2;
  return orc_decode_impl(out, q, q_start, key_cache, value_cache, NULL, NULL, 1.0, 1.0,
                         block_tables, table_stride, seq_lens, num_seqs, num_q_heads,
                         num_kv_heads, head_dim, block_size, scale, dtype, nthreads);
}
