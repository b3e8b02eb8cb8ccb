/*
 * Test infrastructure only: the CPU oracle for paged decode attention and the
 * two cache-maintenance operations that feed it.  Nothing in the product path
 * may call, link or include this file; only the test suite, the smoke check
 * and the benchmark's CPU-baseline leg load the shared library built from it.
 *
 * It is deliberately plain and slow: no blocking, no fusion, no reordering
 * beyond what the definition states.  Floating point is fp64 throughout.
 *
 * Sources (web pages on PagedAttention):
 *   - "Atención paginada en modelos de lenguaje grandes (LLM)" (7minutos.es),
 *     section 2: PagePool is a flat array of equal pages of 16 tokens;
 *     PagedRequest's block_table maps logical page i to a physical page id.
 *   - "PagedAttention" (e-fortepiano.pl wiki mirror), "Formulació matemàtica":
 *     for one query token of causal self-attention the output is the softmax
 *     of the query-key scores (scaled by the attention dimension) weighting
 *     the value vectors; computing it block by block over KV blocks leaves
 *     the causal attention result unchanged, so the paged result equals the
 *     contiguous one.  The formula symbols were lost in extraction; the
 *     reading taken is softmax(q.K^T * scale).V with scale an argument.
 *
 * Layout of a pool (K and V alike): [num_blocks][heads][block_size][head_dim],
 * row-major, elements of the pool's dtype.  A token at logical position t of
 * sequence s lives in physical block block_tables[s][t / block_size] at
 * in-block offset t % block_size.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORACLE_F32 = 0, ORACLE_F16 = 1, ORACLE_BF16 = 2 };

/* IEEE 754 binary16 -> double, from the format's definition: 1 sign bit,
 * 5 exponent bits (bias 15), 10 fraction bits; exponent 0 is subnormal
 * (value = fraction * 2^-24), exponent 31 is infinity or NaN. */
double oracle_half_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int expo = (h >> 10) & 0x1f;
  int frac = h & 0x3ff;
  double v;
  if (expo == 0) {
    v = ldexp((double)frac, -24);
  } else if (expo == 31) {
    v = frac ? NAN : INFINITY;
  } else {
    v = ldexp((double)(frac | 0x400), expo - 25);
  }
  return sign ? -v : v;
}

/* bfloat16 -> double: bfloat16 is the upper 16 bits of an IEEE binary32. */
double oracle_bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static double load_elem(const void* base, int64_t idx, int dtype) {
  if (dtype == ORACLE_F32) return (double)((const float*)base)[idx];
  if (dtype == ORACLE_F16) return oracle_half_to_double(((const uint16_t*)base)[idx]);
  return oracle_bf16_to_double(((const uint16_t*)base)[idx]);
}

/*
 * Decode attention for every (sequence, query head):
 *   1. gather the sequence's cached tokens 0..L-1 through its block table
 *      into contiguous fp64 arrays K[L][D], V[L][D];
 *   2. x_t = scale * sum_d q[d] * K[t][d];
 *   3. m = max_t x_t, w_t = exp(x_t - m), Z = sum_t w_t;
 *   4. out[d] = sum_t w_t * V[t][d] / Z.
 * q:   [num_seqs][num_q_heads][head_dim], same dtype as the pools.
 * out: [num_seqs][num_q_heads][head_dim] in fp64.
 * Query head h reads KV head h / (num_q_heads / kv_heads) (equal counts: the
 * same head).  A sequence with L == 0 has no tokens to attend to; its output
 * is defined as zeros.
 */
void oracle_decode_attention(int dtype, const void* q, const void* k_pool, const void* v_pool,
                             const int32_t* block_tables, int32_t max_blocks_per_seq,
                             const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                             int32_t kv_heads, int32_t head_dim, int32_t block_size, double scale,
                             double* out) {
  const int32_t group = num_q_heads / kv_heads;
  const int64_t n_pairs = (int64_t)num_seqs * num_q_heads;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t pair = 0; pair < n_pairs; ++pair) {
    const int32_t s = (int32_t)(pair / num_q_heads);
    const int32_t h = (int32_t)(pair % num_q_heads);
    const int32_t kvh = h / group;
    const int32_t L = context_lens[s];
    double* o = out + pair * head_dim;
    for (int32_t d = 0; d < head_dim; ++d) o[d] = 0.0;
    if (L <= 0) continue;

    double* K = (double*)malloc(sizeof(double) * (size_t)L * head_dim);
    double* V = (double*)malloc(sizeof(double) * (size_t)L * head_dim);
    double* x = (double*)malloc(sizeof(double) * (size_t)L);
    double* qd = (double*)malloc(sizeof(double) * (size_t)head_dim);

    /* step 1: gather through the block table */
    for (int32_t t = 0; t < L; ++t) {
      int64_t blk = block_tables[(int64_t)s * max_blocks_per_seq + t / block_size];
      int64_t off = t % block_size;
      int64_t row = ((blk * kv_heads + kvh) * block_size + off) * head_dim;
      for (int32_t d = 0; d < head_dim; ++d) {
        K[(int64_t)t * head_dim + d] = load_elem(k_pool, row + d, dtype);
        V[(int64_t)t * head_dim + d] = load_elem(v_pool, row + d, dtype);
      }
    }
    for (int32_t d = 0; d < head_dim; ++d) qd[d] = load_elem(q, pair * head_dim + d, dtype);

    /* step 2: scaled scores */
    for (int32_t t = 0; t < L; ++t) {
      double acc = 0.0;
      for (int32_t d = 0; d < head_dim; ++d) acc += qd[d] * K[(int64_t)t * head_dim + d];
      x[t] = scale * acc;
    }
    /* step 3: softmax weights, max subtracted */
    double m = x[0];
    for (int32_t t = 1; t < L; ++t)
      if (x[t] > m) m = x[t];
    double Z = 0.0;
    for (int32_t t = 0; t < L; ++t) {
      x[t] = exp(x[t] - m);
      Z += x[t];
    }
    /* step 4: weighted sum of values */
    for (int32_t d = 0; d < head_dim; ++d) {
      double acc = 0.0;
      for (int32_t t = 0; t < L; ++t) acc += x[t] * V[(int64_t)t * head_dim + d];
      o[d] = acc / Z;
    }
    free(K);
    free(V);
    free(x);
    free(qd);
  }
}

/*
 * Write each new token's K and V rows (all heads) into the slot that
 * slot_mapping names: slot = physical_block * block_size + in-block offset.
 * A negative slot marks a padding token and is skipped.  Byte copy, so the
 * result is bit-exact whatever the dtype.
 * k_new, v_new: [num_tokens][heads][head_dim] of elem_bytes-sized elements.
 */
void oracle_reshape_and_cache(const void* k_new, const void* v_new, const int32_t* slot_mapping,
                              int32_t num_tokens, void* k_pool, void* v_pool, int32_t heads,
                              int32_t head_dim, int32_t block_size, int32_t elem_bytes) {
  const size_t row_bytes = (size_t)head_dim * elem_bytes;
  for (int32_t t = 0; t < num_tokens; ++t) {
    int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    int64_t blk = slot / block_size;
    int64_t off = slot % block_size;
    for (int32_t h = 0; h < heads; ++h) {
      size_t dst = (size_t)(((blk * heads + h) * block_size + off)) * row_bytes;
      size_t src = (size_t)((int64_t)t * heads + h) * row_bytes;
      memcpy((char*)k_pool + dst, (const char*)k_new + src, row_bytes);
      memcpy((char*)v_pool + dst, (const char*)v_new + src, row_bytes);
    }
  }
}

/*
 * Block-granular copy-on-write, device half: for each (src, dst) pair copy
 * the whole physical block (every head, every slot) of K and of V.
 * pairs: [num_pairs][2].  Destinations are fresh private blocks, so no pair
 * reads a block that another pair writes.
 */
void oracle_copy_blocks(void* k_pool, void* v_pool, const int32_t* pairs, int32_t num_pairs,
                        int32_t heads, int32_t head_dim, int32_t block_size, int32_t elem_bytes) {
  const size_t block_bytes = (size_t)heads * block_size * head_dim * elem_bytes;
  for (int32_t i = 0; i < num_pairs; ++i) {
    int64_t src = pairs[2 * i], dst = pairs[2 * i + 1];
    memcpy((char*)k_pool + dst * block_bytes, (const char*)k_pool + src * block_bytes, block_bytes);
    memcpy((char*)v_pool + dst * block_bytes, (const char*)v_pool + src * block_bytes, block_bytes);
  }
}

/* Physical slot of logical position pos in a sequence with the given block
 * table row: block_table[pos / block_size] * block_size + pos % block_size. */
int64_t oracle_slot_of(const int32_t* block_table_row, int64_t pos, int32_t block_size) {
  return (int64_t)block_table_row[pos / block_size] * block_size + pos % block_size;
}
