/*
 * Paged decode attention: the CPU oracle (fp64, plain C, OpenMP over rows).
 *
 * TEST INFRASTRUCTURE.  This is the slow, obviously correct reference that the
 * CUDA path is checked against.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load it; the library never does, and it shares
 * no code, header or table with the CUDA sources.
 *
 * What it computes is the definition, written out with no blocking, fusion or
 * reordering:
 *
 *   append   For every new token i whose slot s is >= 0 and every kv head h,
 *            copy the row new[i, h, :] to cache[s / bs, h, s % bs, :].
 *            The copy is byte for byte (no conversion).
 *            Source: nano-vllm (ovshake) README, "Key Concepts Explained: KV
 *            Cache" (a decode step computes K and V for the new token only and
 *            keeps the earlier ones) and "Key Concepts Explained:
 *            PagedAttention" (tokens live in fixed-size blocks of one pool).
 *
 *   decode   For every sequence b and query head h, with G = Hq / Hkv, kv head
 *            g = h / G (query heads form contiguous groups over one kv head),
 *            context length L and window start s0 = (W > 0 && L > W) ? L-W : 0:
 *              K_t = row (t % bs) of block block_tables[b][t / bs], kv head g
 *              x_t = scale * sum_d q[b,h,d] * K_t[d]           t in [s0, L)
 *              x_t = c * tanh(x_t / c)    when the softcap c is finite and > 0
 *              m   = max_t x_t,  w_t = exp(x_t - m),  Z = sum_t w_t
 *              out[b,h,:] = sum_t w_t * V_t[:] / Z
 *            L == 0 gives a zero row.
 *
 *   multi    Several new tokens per sequence (speculative-decoding verify, a
 *            chunk of a chunked prefill): T query tokens per sequence whose
 *            keys and values are already in the cache at positions
 *            L-T .. L-1.  Query token j sits at position p_j = L - T + j and
 *            attends causally: it is the decode above with the context
 *            [0, p_j + 1), i.e. positions t in [s0_j, p_j + 1) with
 *            s0_j = (W > 0 && p_j + 1 > W) ? p_j + 1 - W : 0.  A query with
 *            p_j < 0 (L < T) gets a zero row.
 *            Sources: nano-vllm (ovshake) README, "Features" ("Chunked
 *            Prefill", "Speculative Decoding") and the speculative-decoding
 *            command line (--num-speculative-tokens); causal attention over
 *            the cache as in "Key Concepts Explained: KV Cache".  The pages do
 *            not write the mask out; this file takes the causal mask of a
 *            decoder-only model.
 *
 *            Sources: nano-vllm (ovshake) README, "X-Ray Mode" (Step 1: 32 query
 *            heads share 8 KV heads; Step 2: scores = Q K^T / sqrt(head_dim))
 *            and "Key Concepts Explained: PagedAttention" (the per-sequence
 *            block list); flex-nano-vllm README (paged attention with a page
 *            table, for Gemma 2).  The softmax, the Gemma-2 tanh softcap and the
 *            sliding window are not written out on the pages; this file takes
 *            the standard max-subtracted softmax, the softcap applied to the
 *            scaled score, and a window that keeps the last W positions
 *            (the current one included).
 *
 * Inputs are read in their stored type (fp32 or bf16) and widened exactly to
 * double; all arithmetic is double.  Callers round the result themselves.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

enum {
  ORACLE_OK = 0,
  ORACLE_BAD_ARGS = 1,
  ORACLE_BAD_SLOT = 2,
  ORACLE_BAD_BLOCK = 3,
  ORACLE_BAD_LENGTH = 4,
  ORACLE_NO_MEMORY = 5
};

static size_t elem_size(int dtype) { return dtype == ORACLE_F32 ? 4 : 2; }

/* Element idx of an array stored as fp32 or bf16, widened to double. */
static double load(const void* base, int64_t idx, int dtype) {
  if (dtype == ORACLE_F32) return (double)((const float*)base)[idx];
  uint32_t bits = (uint32_t)((const uint16_t*)base)[idx] << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int oracle_write_kv(const void* k_new, const void* v_new, const int64_t* slot_mapping, int num_tokens,
                    void* k_cache, void* v_cache, int num_blocks, int block_size, int num_kv_heads,
                    int head_dim, int dtype) {
  if (num_tokens < 0 || num_blocks <= 0 || block_size <= 0 || num_kv_heads <= 0 || head_dim <= 0)
    return ORACLE_BAD_ARGS;
  const size_t row = (size_t)head_dim * elem_size(dtype);
  const int64_t num_slots = (int64_t)num_blocks * block_size;
  for (int i = 0; i < num_tokens; ++i) {
    int64_t s = slot_mapping[i];
    if (s < 0) continue; /* padding token */
    if (s >= num_slots) return ORACLE_BAD_SLOT;
  }
  for (int i = 0; i < num_tokens; ++i) {
    int64_t s = slot_mapping[i];
    if (s < 0) continue;
    int64_t blk = s / block_size, off = s % block_size;
    for (int h = 0; h < num_kv_heads; ++h) {
      size_t dst = (size_t)((blk * num_kv_heads + h) * block_size + off) * row;
      size_t src = (size_t)((int64_t)i * num_kv_heads + h) * row;
      memcpy((char*)k_cache + dst, (const char*)k_new + src, row);
      memcpy((char*)v_cache + dst, (const char*)v_new + src, row);
    }
  }
  return ORACLE_OK;
}

/* One output row: head h of query row `qrow` of q (a sequence-b query)
 * attending the positions [s0, end) of sequence b, where end = L - back:
 * back = 0 for decode, T - 1 - j for query token j of T (see the header).
 * Returns an ORACLE_* code. */
static int attend_row(const void* q, int q_dtype, int64_t qrow, const void* k_cache, const void* v_cache,
                      int kv_dtype, const int32_t* block_tables, const int32_t* context_lens, int hq, int hkv,
                      int d, int bs, int max_blocks, int num_blocks, double scale, double softcap, int window,
                      int b, int h, int back, double* out_row, double* x /* scratch, >= max_blocks*bs */) {
  const int G = hq / hkv;
  const int g = h / G;
  const int L = context_lens[b];
  for (int j = 0; j < d; ++j) out_row[j] = 0.0;
  if (L < 0 || (int64_t)L > (int64_t)max_blocks * bs) return ORACLE_BAD_LENGTH;
  const int end = L - back;
  if (end <= 0) return ORACLE_OK;
  const int s0 = (window > 0 && end > window) ? end - window : 0;
  const int use_cap = softcap > 0.0 && isfinite(softcap);
  const int64_t qbase = (qrow * hq + h) * d;

  /* Pass 1: scores. */
  double m = -INFINITY;
  for (int t = s0; t < end; ++t) {
    int32_t phys = block_tables[(int64_t)b * max_blocks + t / bs];
    if (phys < 0 || phys >= num_blocks) return ORACLE_BAD_BLOCK;
    int64_t kbase = (((int64_t)phys * hkv + g) * bs + t % bs) * d;
    double dot = 0.0;
    for (int j = 0; j < d; ++j) dot += load(q, qbase + j, q_dtype) * load(k_cache, kbase + j, kv_dtype);
    double s = scale * dot;
    if (use_cap) s = softcap * tanh(s / softcap);
    x[t - s0] = s;
    if (s > m) m = s;
  }
  /* Pass 2: weights and the weighted sum of values. */
  double Z = 0.0;
  for (int t = s0; t < end; ++t) {
    double w = exp(x[t - s0] - m);
    Z += w;
    int32_t phys = block_tables[(int64_t)b * max_blocks + t / bs];
    int64_t vbase = (((int64_t)phys * hkv + g) * bs + t % bs) * d;
    for (int j = 0; j < d; ++j) out_row[j] += w * load(v_cache, vbase + j, kv_dtype);
  }
  for (int j = 0; j < d; ++j) out_row[j] /= Z;
  return ORACLE_OK;
}

/*
 * rows == NULL: every (b, h), out is [batch, hq, d].
 * rows != NULL: n_rows pairs (b, h) stored as rows[2*r], rows[2*r+1]; out is [n_rows, d].
 */
int oracle_decode(const void* q, int q_dtype, const void* k_cache, const void* v_cache, int kv_dtype,
                  const int32_t* block_tables, const int32_t* context_lens, int batch, int hq, int hkv,
                  int d, int bs, int max_blocks, int num_blocks, double scale, double softcap, int window,
                  const int32_t* rows, int n_rows, double* out) {
  if (batch < 0 || hq <= 0 || hkv <= 0 || hq % hkv != 0 || d <= 0 || bs <= 0 || max_blocks <= 0)
    return ORACLE_BAD_ARGS;
  const int n = rows ? n_rows : batch * hq;
  const int64_t cap = (int64_t)max_blocks * bs;
  int status = ORACLE_OK;
#pragma omp parallel
  {
    double* x = (double*)malloc(sizeof(double) * (size_t)(cap > 0 ? cap : 1));
    if (!x) {
#pragma omp critical
      status = ORACLE_NO_MEMORY;
    } else {
#pragma omp for schedule(dynamic, 1)
      for (int r = 0; r < n; ++r) {
        int b = rows ? rows[2 * r] : r / hq;
        int h = rows ? rows[2 * r + 1] : r % hq;
        int st = ORACLE_BAD_ARGS;
        if (b >= 0 && b < batch && h >= 0 && h < hq)
          st = attend_row(q, q_dtype, b, k_cache, v_cache, kv_dtype, block_tables, context_lens, hq, hkv, d, bs,
                          max_blocks, num_blocks, scale, softcap, window, b, h, 0, out + (int64_t)r * d, x);
        if (st != ORACLE_OK) {
#pragma omp critical
          status = st;
        }
      }
      free(x);
    }
  }
  return status;
}


/*
 * Multi-query rows: q is [batch, q_len, hq, d]; query token j of sequence b
 * attends [s0_j, L - q_len + j + 1) (see the header).
 * rows == NULL: every (b, j, h), out is [batch, q_len, hq, d].
 * rows != NULL: n_rows triples (b, j, h) stored as rows[3*r .. 3*r+2]; out is [n_rows, d].
 */
int oracle_decode_multi(const void* q, int q_dtype, const void* k_cache, const void* v_cache, int kv_dtype,
                        const int32_t* block_tables, const int32_t* context_lens, int batch, int q_len, int hq,
                        int hkv, int d, int bs, int max_blocks, int num_blocks, double scale, double softcap,
                        int window, const int32_t* rows, int n_rows, double* out) {
  if (batch < 0 || q_len <= 0 || hq <= 0 || hkv <= 0 || hq % hkv != 0 || d <= 0 || bs <= 0 || max_blocks <= 0)
    return ORACLE_BAD_ARGS;
  const int n = rows ? n_rows : batch * q_len * hq;
  const int64_t cap = (int64_t)max_blocks * bs;
  int status = ORACLE_OK;
#pragma omp parallel
  {
    double* x = (double*)malloc(sizeof(double) * (size_t)(cap > 0 ? cap : 1));
    if (!x) {
#pragma omp critical
      status = ORACLE_NO_MEMORY;
    } else {
#pragma omp for schedule(dynamic, 1)
      for (int r = 0; r < n; ++r) {
        int b = rows ? rows[3 * r] : r / (q_len * hq);
        int j = rows ? rows[3 * r + 1] : (r / hq) % q_len;
        int h = rows ? rows[3 * r + 2] : r % hq;
        int st = ORACLE_BAD_ARGS;
        if (b >= 0 && b < batch && j >= 0 && j < q_len && h >= 0 && h < hq)
          st = attend_row(q, q_dtype, (int64_t)b * q_len + j, k_cache, v_cache, kv_dtype, block_tables,
                          context_lens, hq, hkv, d, bs, max_blocks, num_blocks, scale, softcap, window, b, h,
                          q_len - 1 - j, out + (int64_t)r * d, x);
        if (st != ORACLE_OK) {
#pragma omp critical
          status = st;
        }
      }
      free(x);
    }
  }
  return status;
}
