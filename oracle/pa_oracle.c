/*
 * pa_oracle.c -- plain fp64 CPU oracle for the paged-KV-cache decode hot path.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the checker that the GPU kernels are
 * compared against. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load it. It shares no code, header, table or helper
 * with the CUDA library, and the CUDA library never calls it.
 *
 * What it follows (page titles and sections of the PagedAttention pages):
 *   - "Optimizing LLM Inference: From PagedAttention to AI Infra",
 *     "Understanding KV Cache ..." : decode stores each token's K and V once,
 *     at every layer, and later steps read them back instead of recomputing.
 *   - same page, "PagedAttention: Decoupling Logical Context ..." (Figure 2):
 *     the KV cache is cut into fixed blocks; a per-sequence block table maps
 *     logical block j to a physical block; the kernel reaches the context
 *     through that table, and the context is still one contiguous sequence
 *     from the model's point of view -- so the result is ordinary attention.
 *   - same page, "On-Demand Allocation": block size 16.
 *   - same page, "Copy-on-Write", and "PagedAttention" (ai-system-design-guide),
 *     "KV Cache Sharing (Copy-on-Write)": a shared block is copied whole when
 *     a sequence diverges; the shared original stays unchanged.
 *   - "The Memory Wall ...", "Show Me The Code": the kernel walks the block
 *     table in logical order and finds block p at pool + p * block_size rows.
 *
 * Layout (the plainest block-major reading; the pages fix none):
 *   k_cache, v_cache : [num_blocks][H_kv][block_size][D], 16-bit elements
 *   q, out           : [num_seqs][H_q][D]
 *   k, v (new rows)  : [num_tokens][H_kv][D]
 *   block_tables     : int32 [num_seqs][stride]
 *   slot_mapping     : int64 [num_tokens]; slot = block * block_size + offset,
 *                      negative = padding token, skipped.
 *   GQA: query head h reads KV head h / (H_q / H_kv).
 *
 * Arithmetic: every fp16 / bf16 input is decoded exactly to double by bit
 * manipulation written here; the attention is the textbook two-pass softmax
 * in double: x_t = scale * <q, K_t>, w = exp(x - max x) / sum exp(x - max x),
 * out = sum_t w_t V_t. No blocking, no online softmax, no split.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_F16 0
#define ORACLE_BF16 1

/* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
static double f16_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int frac = h & 0x3ff;
  double v;
  if (e == 0) {
    v = ldexp((double)frac, -24); /* subnormal: frac * 2^-14 * 2^-10 */
  } else if (e == 31) {
    v = frac ? NAN : INFINITY;
  } else {
    v = ldexp((double)(frac + 1024), e - 25); /* (1 + frac/1024) * 2^(e-15) */
  }
  return sign ? -v : v;
}

/* bfloat16: the top 16 bits of an IEEE binary32. */
static double bf16_to_double(uint16_t b) {
  int sign = (b >> 15) & 1;
  int e = (b >> 7) & 0xff;
  int frac = b & 0x7f;
  double v;
  if (e == 0) {
    v = ldexp((double)frac, -133); /* subnormal: frac * 2^-126 * 2^-7 */
  } else if (e == 255) {
    v = frac ? NAN : INFINITY;
  } else {
    v = ldexp((double)(frac + 128), e - 134); /* (1 + frac/128) * 2^(e-127) */
  }
  return sign ? -v : v;
}

static double decode16(uint16_t bits, int dtype) {
  return dtype == ORACLE_BF16 ? bf16_to_double(bits) : f16_to_double(bits);
}

/* Exposed so that the tests can check the decoders over all 65536 patterns. */
void oracle_decode16(const uint16_t* bits, int64_t n, int dtype, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = decode16(bits[i], dtype);
}

/*
 * Store the new tokens' K and V rows in their cache slots (the KV write of
 * every decode step). Returns the number of tokens whose slot lay outside
 * [0, num_blocks * block_size) and were therefore not written (negative
 * slots are padding and are not counted).
 */
int64_t oracle_write_kv(const uint16_t* k, const uint16_t* v, uint16_t* k_cache,
                        uint16_t* v_cache, const int64_t* slot_mapping,
                        int32_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                        int32_t block_size, int64_t num_blocks) {
  int64_t bad = 0;
  for (int32_t t = 0; t < num_tokens; ++t) {
    int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    if (slot >= num_blocks * (int64_t)block_size) {
      ++bad;
      continue;
    }
    int64_t block = slot / block_size;
    int64_t offset = slot % block_size;
    for (int32_t h = 0; h < num_kv_heads; ++h) {
      int64_t dst = ((block * num_kv_heads + h) * block_size + offset) * head_dim;
      int64_t src = ((int64_t)t * num_kv_heads + h) * head_dim;
      memcpy(k_cache + dst, k + src, sizeof(uint16_t) * (size_t)head_dim);
      memcpy(v_cache + dst, v + src, sizeof(uint16_t) * (size_t)head_dim);
    }
  }
  return bad;
}

/*
 * Copy-on-write block copies: for every (src, dst) pair and every layer, the
 * whole physical block (all KV heads, all slots) of K and of V is copied.
 */
void oracle_copy_blocks(uint16_t** k_caches, uint16_t** v_caches, int32_t num_layers,
                        const int64_t* block_mapping, int32_t num_pairs,
                        int32_t num_kv_heads, int32_t head_dim, int32_t block_size) {
  size_t block_elems = (size_t)num_kv_heads * block_size * head_dim;
  for (int32_t l = 0; l < num_layers; ++l) {
    for (int32_t p = 0; p < num_pairs; ++p) {
      int64_t src = block_mapping[2 * p];
      int64_t dst = block_mapping[2 * p + 1];
      memmove(k_caches[l] + dst * block_elems, k_caches[l] + src * block_elems,
              block_elems * sizeof(uint16_t));
      memmove(v_caches[l] + dst * block_elems, v_caches[l] + src * block_elems,
              block_elems * sizeof(uint16_t));
    }
  }
}

/*
 * Swap blocks between two pools (preemption moves a request's blocks from GPU
 * memory to CPU RAM and back: "PagedAttention", "Managing Virtual Memory
 * (Block Manager)"): for every (src, dst) pair and every layer, block src of
 * the source pool is copied whole to block dst of the destination pool.
 */
void oracle_swap_blocks(uint16_t** src_k, uint16_t** src_v, uint16_t** dst_k, uint16_t** dst_v,
                        int32_t num_layers, const int64_t* block_mapping, int32_t num_pairs,
                        int32_t num_kv_heads, int32_t head_dim, int32_t block_size) {
  size_t block_elems = (size_t)num_kv_heads * block_size * head_dim;
  for (int32_t l = 0; l < num_layers; ++l) {
    for (int32_t p = 0; p < num_pairs; ++p) {
      int64_t src = block_mapping[2 * p];
      int64_t dst = block_mapping[2 * p + 1];
      memcpy(dst_k[l] + dst * block_elems, src_k[l] + src * block_elems,
             block_elems * sizeof(uint16_t));
      memcpy(dst_v[l] + dst * block_elems, src_v[l] + src * block_elems,
             block_elems * sizeof(uint16_t));
    }
  }
}

typedef struct {
  const uint16_t* q;
  const uint16_t* k_cache;
  const uint16_t* v_cache;
  const int32_t* block_tables;
  int32_t block_table_stride;
  const int32_t* context_lens;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t block_size;
  int64_t num_blocks;
  double scale;
  int dtype;
  const int64_t* rows; /* (seq * H_q + head) for each output row, or NULL = all */
  int64_t num_rows;
  double* out; /* [num_rows][D] */
  int64_t next; /* work counter, guarded by lock */
  pthread_mutex_t lock;
  int error; /* set when a table entry is out of range */
} decode_job;

/*
 * One output row: attention of query head h of sequence s over the s-th
 * context, gathered in logical order through the block table.
 * Returns 0, or -1 if a block-table entry is outside [0, num_blocks).
 */
static int decode_row(const decode_job* a, int64_t row, double* o) {
  const int32_t D = a->head_dim;
  const int32_t g = a->num_q_heads / a->num_kv_heads;
  const int64_t s = row / a->num_q_heads;
  const int32_t h = (int32_t)(row % a->num_q_heads);
  const int32_t kvh = h / g;
  const int32_t L = a->context_lens[s];
  for (int32_t d = 0; d < D; ++d) o[d] = 0.0;
  if (L <= 0) return 0; /* empty context: zero output */

  double* qd = (double*)malloc(sizeof(double) * D);
  double* K = (double*)malloc(sizeof(double) * (size_t)L * D);
  double* V = (double*)malloc(sizeof(double) * (size_t)L * D);
  double* x = (double*)malloc(sizeof(double) * (size_t)L);
  int rc = 0;

  for (int32_t d = 0; d < D; ++d) qd[d] = decode16(a->q[(s * a->num_q_heads + h) * D + d], a->dtype);

  /* Gather: logical token t lives in logical block t / block_size, slot
   * t % block_size of the physical block the table names. */
  for (int32_t t = 0; t < L && rc == 0; ++t) {
    int32_t j = t / a->block_size;
    int32_t i = t % a->block_size;
    int64_t p = a->block_tables[s * a->block_table_stride + j];
    if (p < 0 || p >= a->num_blocks) {
      rc = -1;
      break;
    }
    int64_t base = ((p * a->num_kv_heads + kvh) * a->block_size + i) * D;
    for (int32_t d = 0; d < D; ++d) {
      K[(size_t)t * D + d] = decode16(a->k_cache[base + d], a->dtype);
      V[(size_t)t * D + d] = decode16(a->v_cache[base + d], a->dtype);
    }
  }

  if (rc == 0) {
    /* logits */
    double mx = -INFINITY;
    for (int32_t t = 0; t < L; ++t) {
      double acc = 0.0;
      for (int32_t d = 0; d < D; ++d) acc += qd[d] * K[(size_t)t * D + d];
      x[t] = a->scale * acc;
      if (x[t] > mx) mx = x[t];
    }
    /* two-pass softmax */
    double sum = 0.0;
    for (int32_t t = 0; t < L; ++t) {
      x[t] = exp(x[t] - mx);
      sum += x[t];
    }
    for (int32_t t = 0; t < L; ++t) x[t] /= sum;
    /* weighted sum of values */
    for (int32_t t = 0; t < L; ++t)
      for (int32_t d = 0; d < D; ++d) o[d] += x[t] * V[(size_t)t * D + d];
  }

  free(qd);
  free(K);
  free(V);
  free(x);
  return rc;
}

static void* decode_worker(void* arg) {
  decode_job* a = (decode_job*)arg;
  for (;;) {
    pthread_mutex_lock(&a->lock);
    int64_t r = a->next++;
    pthread_mutex_unlock(&a->lock);
    if (r >= a->num_rows) break;
    int64_t row = a->rows ? a->rows[r] : r;
    if (decode_row(a, row, a->out + r * a->head_dim) != 0) {
      pthread_mutex_lock(&a->lock);
      a->error = 1;
      pthread_mutex_unlock(&a->lock);
    }
  }
  return NULL;
}

int oracle_num_cores(void) {
  long n = sysconf(_SC_NPROCESSORS_ONLN);
  return n > 0 ? (int)n : 1;
}

/*
 * Paged decode attention for the requested output rows (or all
 * num_seqs * H_q rows when rows == NULL). out is [num_rows][D] doubles.
 * The rows are independent, so they are spread over n_threads threads
 * (0 = every online core). Returns 0, or -1 on an out-of-range table entry.
 */
int oracle_decode(double* out, const uint16_t* q, const uint16_t* k_cache,
                  const uint16_t* v_cache, const int32_t* block_tables,
                  int32_t block_table_stride, const int32_t* context_lens,
                  int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                  int32_t head_dim, int32_t block_size, int64_t num_blocks,
                  double scale, int dtype, const int64_t* rows, int64_t num_rows,
                  int n_threads) {
  decode_job a;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.block_tables = block_tables;
  a.block_table_stride = block_table_stride;
  a.context_lens = context_lens;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = num_kv_heads;
  a.head_dim = head_dim;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.scale = scale;
  a.dtype = dtype;
  a.rows = rows;
  a.num_rows = rows ? num_rows : (int64_t)num_seqs * num_q_heads;
  a.out = out;
  a.next = 0;
  a.error = 0;
  pthread_mutex_init(&a.lock, NULL);

  if (n_threads <= 0) n_threads = oracle_num_cores();
  if (n_threads > a.num_rows) n_threads = a.num_rows > 0 ? (int)a.num_rows : 1;
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)n_threads);
  for (int i = 0; i < n_threads; ++i) pthread_create(&th[i], NULL, decode_worker, &a);
  for (int i = 0; i < n_threads; ++i) pthread_join(th[i], NULL);
  free(th);
  pthread_mutex_destroy(&a.lock);
  return a.error ? -1 : 0;
}
