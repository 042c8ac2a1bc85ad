/*
 * pa_oracle.c -- plain, slow, fp64 CPU oracle for paged attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark load this library.  It shares no code,
 * header, table or helper with the CUDA library; the two meet only through the
 * seeded synthetic inputs.
 *
 * What it follows (page = "LLM推論エンジンvLLMの内部構造を徹底解説", techfeed.io
 * summary of "Inside vLLM: Anatomy of a High-Throughput LLM Inference System"):
 *   - section "PagedAttentionの仕組み": the KV cache is managed in fixed-size
 *     blocks, 16 tokens by default; a 17-token prefill receives ceil(17/16) = 2
 *     blocks; allocate_slots counts the blocks needed, then takes the first n
 *     blocks of free_block_queue and records them in req_to_blocks; in the
 *     forward pass every scheduled sequence is concatenated into one flat
 *     "super-sequence" and position indices plus an attention mask make each
 *     sequence attend only to its own tokens.
 *   - section "高度な機能群" (Chunked Prefill, Prefix Caching): a prefill chunk
 *     attends to the context already cached before it; requests that share a
 *     prompt prefix reuse the same KV blocks.
 *   - section "エンジンの中核": a decode step runs the newest token only, against
 *     the KV cache.
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes): cache layout [num_blocks][num_kv_heads][block_size][head_dim]
 * row-major, K and V in separate buffers; slot = block_id * block_size +
 * offset, negative slot = skip; the causal mask is aligned bottom-right (query
 * j of a sequence with q_len new tokens and seq_len total tokens sits at
 * position seq_len - q_len + j and sees keys 0..that position); grouped-query
 * heads map q-head h to kv-head h / (num_q_heads / num_kv_heads); softmax
 * attention is the exact two-pass definition, accumulated in fp64 over keys in
 * logical order.
 *
 * Parity pins (tests run without a GPU): the worked example 17 -> 2 blocks,
 * brute-force block/slot checks, torch's fp64 scaled-dot-product attention on
 * contiguous K/V (a library routine), permutation invariance of physical block
 * ids, closed-form special cases (one key, constant V, zero query), GQA equal to
 * MHA with repeated KV heads, chunked prefill equal to one-shot prefill, a
 * shared prefix equal to private copies, an exhaustive check of the bf16
 * rounding against exact rational arithmetic, and the step planner against
 * allocate_slots walked by hand over chained steps.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* dtype codes of the element buffers handed to the oracle */
#define ORACLE_F32 0
#define ORACLE_BF16 1

/* ------------------------------------------------------------------------- */
/* element access                                                            */
/* ------------------------------------------------------------------------- */

/* bf16 is the upper half of an IEEE binary32 pattern; widening is exact. */
static double bf16_bits_to_double(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static double load_elem(const void* base, int64_t idx, int dtype) {
  if (dtype == ORACLE_F32) return (double)((const float*)base)[idx];
  return bf16_bits_to_double(((const uint16_t*)base)[idx]);
}

/* ------------------------------------------------------------------------- */
/* block bookkeeping (section "PagedAttentionの仕組み")                      */
/* ------------------------------------------------------------------------- */

/* Number of blocks of block_size tokens that num_tokens tokens occupy:
 * ceil(num_tokens / block_size).  The page's worked example: 17 tokens with
 * 16-token blocks take 2 blocks. */
int64_t oracle_blocks_needed(int64_t num_tokens, int64_t block_size) {
  if (num_tokens <= 0 || block_size <= 0) return 0;
  int64_t whole = num_tokens / block_size;
  return (num_tokens % block_size == 0) ? whole : whole + 1;
}

/* allocate_slots, steps 1 and 3: count the blocks each request needs, then
 * take that many from the FRONT of free_block_queue, in request order, and
 * record them as the request's block list (its row of the block table).
 *
 * shared_prefix_tokens > 0 (a multiple of block_size) models prefix caching:
 * the prefix's blocks are taken from the queue first, once, and every request's
 * list starts with them; each request then takes only the blocks beyond the
 * prefix.  Step 2 (preemption when the pool runs dry) is scheduler policy and
 * is not modelled: running dry returns -1.
 *
 * Unused table entries are set to pad_value.  *blocks_taken receives how many
 * queue entries were consumed.  Returns 0, or -1 on exhaustion / bad sizes. */
int oracle_allocate_block_tables(const int32_t* free_queue, int64_t queue_len,
                                 int num_seqs, const int32_t* seq_lens,
                                 int shared_prefix_tokens, int block_size,
                                 int max_blocks_per_seq, int32_t pad_value,
                                 int32_t* block_tables, int64_t* blocks_taken) {
  int64_t head = 0;
  int64_t n_prefix = 0;
  if (block_size <= 0 || shared_prefix_tokens < 0) return -1;
  if (shared_prefix_tokens % block_size != 0) return -1;
  n_prefix = oracle_blocks_needed(shared_prefix_tokens, block_size);
  if (n_prefix > queue_len || n_prefix > max_blocks_per_seq) return -1;
  head = n_prefix; /* the prefix request is served first */

  for (int s = 0; s < num_seqs; ++s) {
    int32_t* row = block_tables + (int64_t)s * max_blocks_per_seq;
    for (int c = 0; c < max_blocks_per_seq; ++c) row[c] = pad_value;
    if (seq_lens[s] < shared_prefix_tokens) return -1;
    int64_t need = oracle_blocks_needed(seq_lens[s], block_size);
    if (need > max_blocks_per_seq) return -1;
    for (int64_t c = 0; c < n_prefix; ++c) row[c] = free_queue[c];
    for (int64_t c = n_prefix; c < need; ++c) {
      if (head >= queue_len) return -1;
      row[c] = free_queue[head++];
    }
  }
  if (blocks_taken) *blocks_taken = head;
  return 0;
}

/* Super-sequence offsets: all scheduled sequences are laid end to end, so
 * sequence s's query rows start where the previous sequences' rows end:
 * query_start_loc[0] = 0, query_start_loc[s+1] = query_start_loc[s] + q_len[s]. */
void oracle_query_start_loc(const int32_t* query_lens, int num_seqs, int32_t* query_start_loc) {
  query_start_loc[0] = 0;
  for (int s = 0; s < num_seqs; ++s) query_start_loc[s + 1] = query_start_loc[s] + query_lens[s];
}

/* Cache slot of every listed token: sequence s contributes the positions
 * first_pos[s] .. first_pos[s] + count[s] - 1, in order, and the output is the
 * concatenation over s.  A token at position p of sequence s lives in logical
 * block p / block_size at offset p % block_size, so its slot is
 * block_tables[s][p / block_size] * block_size + p % block_size. */
int oracle_slot_mapping(const int32_t* block_tables, int max_blocks_per_seq,
                        int num_seqs, const int32_t* first_pos,
                        const int32_t* count, int block_size, int64_t* slots) {
  int64_t out = 0;
  for (int s = 0; s < num_seqs; ++s) {
    for (int32_t k = 0; k < count[s]; ++k) {
      int64_t p = (int64_t)first_pos[s] + k;
      int64_t logical_block = p / block_size;
      int64_t offset = p % block_size;
      if (logical_block >= max_blocks_per_seq) return -1;
      int64_t phys = block_tables[(int64_t)s * max_blocks_per_seq + logical_block];
      slots[out++] = phys * block_size + offset;
    }
  }
  return 0;
}

/* One scheduler step of block planning for a running batch (page
 * "【ITニュース解説】Inside vLLM: Anatomy of a High-Throughput LLM Inference
 * System", its paragraph on Paging Attention: blocks are handed out as new
 * tokens are produced, only as many as needed).  Sequence s
 * holds the blocks of its first num_computed[s] tokens (the first
 * blocks_needed(num_computed[s]) entries of its row) and schedules
 * query_lens[s] new tokens.  allocate_slots, sequences in order: each takes
 * the blocks it still lacks for num_computed[s] + query_lens[s] tokens from
 * the front of the queue (which starts at *head) and appends them to its row.
 * Then seq_lens[s] = num_computed[s] + query_lens[s], the super-sequence
 * offsets of query_lens, and the slot of every new position num_computed[s] ..
 * seq_lens[s] - 1, in order.
 *
 * The whole step is checked before anything is written: a negative count, a
 * head outside the queue, a row that would grow past max_blocks_per_seq, a
 * queue that runs dry or more new tokens than max_tokens returns -1 and
 * writes nothing.  On success *head has moved past the blocks taken. */
int oracle_plan_step(const int32_t* free_queue, int64_t queue_len, int64_t* head,
                     const int32_t* num_computed, const int32_t* query_lens, int num_seqs,
                     int32_t* block_tables, int max_blocks_per_seq, int block_size,
                     int32_t* seq_lens, int32_t* query_start_loc, int64_t* slots,
                     int64_t max_tokens) {
  int64_t wanted = 0, tokens = 0;
  if (*head < 0 || *head > queue_len) return -1;
  for (int s = 0; s < num_seqs; ++s) {
    if (num_computed[s] < 0 || query_lens[s] < 0) return -1;
    int64_t len = (int64_t)num_computed[s] + query_lens[s];
    if (len > INT32_MAX) return -1;
    int64_t have = oracle_blocks_needed(num_computed[s], block_size);
    int64_t need = oracle_blocks_needed(len, block_size);
    if (need > max_blocks_per_seq) return -1;
    wanted += need - have;
    tokens += query_lens[s];
  }
  if (wanted > queue_len - *head || tokens > max_tokens) return -1;

  int64_t next = *head;
  for (int s = 0; s < num_seqs; ++s) {
    int32_t* row = block_tables + (int64_t)s * max_blocks_per_seq;
    int64_t len = (int64_t)num_computed[s] + query_lens[s];
    int64_t have = oracle_blocks_needed(num_computed[s], block_size);
    int64_t need = oracle_blocks_needed(len, block_size);
    for (int64_t c = have; c < need; ++c) row[c] = free_queue[next++];
    seq_lens[s] = (int32_t)len;
  }
  oracle_query_start_loc(query_lens, num_seqs, query_start_loc);
  if (oracle_slot_mapping(block_tables, max_blocks_per_seq, num_seqs, num_computed, query_lens,
                          block_size, slots) != 0)
    return -1; /* unreachable after the row check */
  *head = next;
  return 0;
}

/* ------------------------------------------------------------------------- */
/* cache write                                                               */
/* ------------------------------------------------------------------------- */

/* Copy the K and V rows of each new token into its cache slot.  Row i of k/v is
 * [num_kv_heads][head_dim]; the cache is [num_blocks][num_kv_heads][block_size]
 * [head_dim].  A negative slot means "no slot" and the row is skipped.  The
 * copy is exact (elements are moved, not converted). */
void oracle_reshape_and_cache(const void* k, const void* v, void* k_cache,
                              void* v_cache, const int64_t* slot_mapping,
                              int64_t num_tokens, int num_kv_heads,
                              int head_dim, int block_size, int elem_bytes) {
  const char* kin = (const char*)k;
  const char* vin = (const char*)v;
  char* kc = (char*)k_cache;
  char* vc = (char*)v_cache;
  for (int64_t i = 0; i < num_tokens; ++i) {
    int64_t slot = slot_mapping[i];
    if (slot < 0) continue;
    int64_t blk = slot / block_size;
    int64_t off = slot % block_size;
    for (int h = 0; h < num_kv_heads; ++h) {
      for (int d = 0; d < head_dim; ++d) {
        int64_t src = ((i * num_kv_heads + h) * head_dim + d) * elem_bytes;
        int64_t dst = (((blk * num_kv_heads + h) * block_size + off) * head_dim + d) *
                      elem_bytes;
        memcpy(kc + dst, kin + src, (size_t)elem_bytes);
        memcpy(vc + dst, vin + src, (size_t)elem_bytes);
      }
    }
  }
}

/* ------------------------------------------------------------------------- */
/* attention                                                                 */
/* ------------------------------------------------------------------------- */

/* index of the element (block b, kv-head h, offset o, dim d) in a cache */
static int64_t kv_at(int64_t b, int h, int o, int d, int num_kv_heads,
                     int block_size, int head_dim) {
  return (((b * num_kv_heads + h) * block_size + o) * (int64_t)head_dim) + d;
}

/* One output row: query token `tok` (index into the flattened super-sequence)
 * and query head `head`.  The sequence that owns tok is found from
 * query_start_loc; the token's position is seq_len - q_len + j; it attends to
 * keys 0..position of its own sequence only, read through the block table.
 * o = sum_t softmax_t(scale * q.k_t) v_t with the softmax taken in two passes
 * (max, then normalised exponentials) in fp64.  Returns -1 on a malformed
 * sequence description. */
static int attention_row(const void* q, const void* k_cache, const void* v_cache,
                         const int32_t* block_tables, int max_blocks_per_seq,
                         const int32_t* seq_lens, const int32_t* query_start_loc,
                         int num_seqs, int num_q_heads, int num_kv_heads,
                         int head_dim, int block_size, double scale, int dtype,
                         int64_t tok, int head, double* out_row) {
  int s = -1;
  for (int c = 0; c < num_seqs; ++c) {
    if (tok >= query_start_loc[c] && tok < query_start_loc[c + 1]) {
      s = c;
      break;
    }
  }
  if (s < 0) return -1;
  int64_t q_len = query_start_loc[s + 1] - query_start_loc[s];
  int64_t seq_len = seq_lens[s];
  if (q_len > seq_len) return -1;
  int64_t j = tok - query_start_loc[s];
  int64_t pos = seq_len - q_len + j; /* last key this query may see */
  int group = num_q_heads / num_kv_heads;
  int kvh = head / group;
  const int32_t* table = block_tables + (int64_t)s * max_blocks_per_seq;
  int64_t nkeys = pos + 1;

  double* x = (double*)malloc((size_t)nkeys * sizeof(double));
  if (!x) return -1;
  for (int64_t t = 0; t < nkeys; ++t) {
    int64_t b = table[t / block_size];
    int o = (int)(t % block_size);
    double dot = 0.0;
    for (int d = 0; d < head_dim; ++d) {
      double qd = load_elem(q, (tok * num_q_heads + head) * (int64_t)head_dim + d, dtype);
      double kd = load_elem(k_cache, kv_at(b, kvh, o, d, num_kv_heads, block_size, head_dim),
                            dtype);
      dot += qd * kd;
    }
    x[t] = scale * dot;
  }
  double m = -INFINITY;
  for (int64_t t = 0; t < nkeys; ++t)
    if (x[t] > m) m = x[t];
  double l = 0.0;
  for (int64_t t = 0; t < nkeys; ++t) {
    x[t] = exp(x[t] - m);
    l += x[t];
  }
  for (int d = 0; d < head_dim; ++d) out_row[d] = 0.0;
  for (int64_t t = 0; t < nkeys; ++t) {
    int64_t b = table[t / block_size];
    int o = (int)(t % block_size);
    for (int d = 0; d < head_dim; ++d)
      out_row[d] += x[t] * load_elem(v_cache,
                                     kv_at(b, kvh, o, d, num_kv_heads, block_size, head_dim),
                                     dtype);
  }
  for (int d = 0; d < head_dim; ++d) out_row[d] /= l;
  free(x);
  return 0;
}

/* Selected output rows: row r is (row_token[r], row_head[r]) and its head_dim
 * results go to out[r * head_dim ...].  Used for sampled checks at full size. */
int oracle_paged_attention_rows(const void* q, const void* k_cache, const void* v_cache,
                                const int32_t* block_tables, int max_blocks_per_seq,
                                const int32_t* seq_lens, const int32_t* query_start_loc,
                                int num_seqs, int num_q_heads, int num_kv_heads,
                                int head_dim, int block_size, double scale, int dtype,
                                int64_t num_rows, const int64_t* row_token,
                                const int32_t* row_head, double* out, int num_threads) {
  if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return -1;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(num_threads) reduction(| : bad)
  for (int64_t r = 0; r < num_rows; ++r) {
    bad |= attention_row(q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                         query_start_loc, num_seqs, num_q_heads, num_kv_heads, head_dim,
                         block_size, scale, dtype, row_token[r], row_head[r],
                         out + r * (int64_t)head_dim) != 0;
  }
  return bad ? -1 : 0;
}

/* Every output row of the step: out is [num_tokens][num_q_heads][head_dim]. */
int oracle_paged_attention(const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, int max_blocks_per_seq,
                           const int32_t* seq_lens, const int32_t* query_start_loc,
                           int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                           int block_size, double scale, int dtype, double* out,
                           int num_threads) {
  if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return -1;
  int64_t num_tokens = query_start_loc[num_seqs];
  int64_t rows = num_tokens * num_q_heads;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(num_threads) reduction(| : bad)
  for (int64_t r = 0; r < rows; ++r) {
    bad |= attention_row(q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                         query_start_loc, num_seqs, num_q_heads, num_kv_heads, head_dim,
                         block_size, scale, dtype, r / num_q_heads, (int)(r % num_q_heads),
                         out + r * (int64_t)head_dim) != 0;
  }
  return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------- */
/* output rounding                                                           */
/* ------------------------------------------------------------------------- */

/* The bf16 value nearest to x, ties to the even significand (round to nearest
 * even), straight from fp64 (no detour through fp32, which could round twice).
 * bf16 keeps 8 significant bits and binary32's exponent range. */
uint16_t oracle_bf16_bits(double x) {
  uint16_t sign = signbit(x) ? 0x8000u : 0u;
  double a = fabs(x);
  if (isnan(x)) return 0x7FC0u;
  if (a == 0.0) return sign;
  int e;
  frexp(a, &e); /* a = f * 2^e, f in [0.5, 1) -> leading bit has weight 2^(e-1) */
  int lead = e - 1;
  if (lead < -126) lead = -126; /* subnormal range: fixed quantum 2^-133 */
  /* quantum (weight of the last kept bit) is 2^(lead - 7) */
  double scaled = ldexp(a, 7 - lead);
  double ip = floor(scaled);
  double frac = scaled - ip; /* exact: scaled < 2^9 */
  if (frac > 0.5 || (frac == 0.5 && fmod(ip, 2.0) != 0.0)) ip += 1.0;
  double r = ldexp(ip, lead - 7);
  if (r >= 0x1.0p128) return (uint16_t)(sign | 0x7F80u); /* overflow -> inf */
  float rf = (float)r; /* exact: r is representable in bf16, hence in binary32 */
  uint32_t u;
  memcpy(&u, &rf, sizeof u);
  return (uint16_t)(sign | (uint16_t)((u >> 16) & 0x7FFFu));
}

void oracle_round_to_bf16(const double* x, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_bits(x[i]);
}
