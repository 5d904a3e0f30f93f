/*
 * CPU oracle for paged decode attention and its cache companions.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * statement of what the paged KV-cache path computes, in fp64.  Only the test
 * suite, the smoke check and the benchmark's CPU-baseline leg load it.  It shares
 * no code, header or table with the CUDA library.
 *
 * What it follows (the vLLM paged-attention pages):
 *  - "IO-5 vLLM Paged Attention" note, section 4 (attention computation): the
 *    output is softmax(q K^T / sqrt(d_k)) V, where K (and V) are the sequence's
 *    pages concatenated in page-table order, K = concat(K_page1, K_page5, ...).
 *    The same note's misconception list says paging does not change the attention
 *    arithmetic, so the oracle gathers through the table into a contiguous array
 *    and then evaluates the textbook formula.
 *  - same note, section 3 (page-table structure): each sequence maps to a list
 *    of page indices; logical token t is in page table[t / bs] at offset t % bs.
 *  - "vLLM PagedAttention / dynamic memory" blog, first section: every generated
 *    token's K and V are stored into the cache (the cache write below), and pages
 *    may be shared between requests (block copy below makes a private copy).
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *  - cache layout [num_blocks][num_kv_heads][block_size][head_dim];
 *  - slot = block * block_size + offset, negative slot = no write;
 *  - q head h reads kv head h / (num_q_heads / num_kv_heads);
 *  - context length 0 gives an all-zero output;
 *  - sliding window W > 0 (the block manager's sliding_window setting in the
 *    dynamic-memory blog, BlockSpaceManager example): the query attends to the last
 *    W tokens of its context, positions max(0, L - W) .. L - 1, and table entries
 *    of pages wholly before that range are never read (their blocks may have been
 *    returned to the pool).
 *
 * Values arrive as 16-bit patterns (bf16 or fp16) and are widened exactly to double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_FP16 = 0, ORC_BF16 = 1 };

/* bf16: the upper 16 bits of an IEEE binary32. */
static double orc_bf16(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* fp16: IEEE binary16, 1 sign, 5 exponent (bias 15), 10 fraction bits. */
static double orc_fp16(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24); /* subnormal: f * 2^-14 * 2^-10 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(f + 1024), e - 25); /* (1 + f/1024) * 2^(e-15) */
    return sign ? -v : v;
}

static double orc_widen(uint16_t h, int dtype) {
    return dtype == ORC_BF16 ? orc_bf16(h) : orc_fp16(h);
}

/* Cache write: cache[slot / bs][h][slot % bs][:] = key[t][h][:] for slot >= 0.
 * Returns the number of slots that were out of range (and skipped). */
int orc_kv_write(const uint16_t *key, const uint16_t *value, const int64_t *slot_mapping,
                 int num_tokens, int num_kv_heads, int head_dim, int64_t key_token_stride,
                 int64_t value_token_stride, uint16_t *k_cache, uint16_t *v_cache,
                 int num_blocks, int block_size) {
    int bad = 0;
    for (int t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= (int64_t)num_blocks * block_size) { ++bad; continue; }
        int64_t blk = slot / block_size, off = slot % block_size;
        for (int h = 0; h < num_kv_heads; ++h) {
            size_t dst = (((size_t)blk * num_kv_heads + h) * block_size + off) * head_dim;
            const uint16_t *ks = key + (size_t)t * key_token_stride + (size_t)h * head_dim;
            const uint16_t *vs = value + (size_t)t * value_token_stride + (size_t)h * head_dim;
            for (int i = 0; i < head_dim; ++i) {
                k_cache[dst + i] = ks[i];
                v_cache[dst + i] = vs[i];
            }
        }
    }
    return bad;
}

/* Block copy: for each (src, dst) pair in order, whole block dst := block src in both
 * caches.  Returns the number of pairs with an id outside [0, num_blocks) (skipped). */
int orc_copy_blocks(uint16_t *k_cache, uint16_t *v_cache, const int64_t *pairs, int num_pairs,
                    int num_kv_heads, int block_size, int head_dim, int num_blocks) {
    int bad = 0;
    size_t blk = (size_t)num_kv_heads * block_size * head_dim;
    for (int p = 0; p < num_pairs; ++p) {
        int64_t src = pairs[2 * p], dst = pairs[2 * p + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) { ++bad; continue; }
        for (size_t i = 0; i < blk; ++i) {
            k_cache[(size_t)dst * blk + i] = k_cache[(size_t)src * blk + i];
            v_cache[(size_t)dst * blk + i] = v_cache[(size_t)src * blk + i];
        }
    }
    return bad;
}

/* Copy-on-write of the filled rows of a block: for each (src, dst, rows) triple in order,
 * rows r < rows of every kv head h of block dst := the same rows of block src, in both
 * caches; the other rows of dst keep their values.  Returns the number of triples with a
 * block id outside [0, num_blocks) or rows outside [0, block_size] (skipped). */
int orc_copy_rows(uint16_t *k_cache, uint16_t *v_cache, const int64_t *triples, int n,
                  int num_kv_heads, int block_size, int head_dim, int num_blocks) {
    int bad = 0;
    for (int c = 0; c < n; ++c) {
        int64_t src = triples[3 * c], dst = triples[3 * c + 1], rows = triples[3 * c + 2];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks || rows < 0 ||
            rows > block_size) {
            ++bad;
            continue;
        }
        for (int h = 0; h < num_kv_heads; ++h)
            for (int64_t r = 0; r < rows; ++r) {
                size_t from = (((size_t)src * num_kv_heads + h) * block_size + r) * head_dim;
                size_t to = (((size_t)dst * num_kv_heads + h) * block_size + r) * head_dim;
                for (int i = 0; i < head_dim; ++i) {
                    k_cache[to + i] = k_cache[from + i];
                    v_cache[to + i] = v_cache[from + i];
                }
            }
    }
    return bad;
}

/* Attention for one (sequence, q head), written as the definition:
 *   K_s = concat of the sequence's pages in table order (first L rows),
 *   z_t = scale * <q, K_s[t]>,  out = sum_t softmax(z)_t V_s[t],
 * with t over [t_lo, L): t_lo = 0, or L - window under a sliding window shorter
 * than the context.
 * Returns 0, or -1 if a table entry needed for a token in range is outside
 * [0, num_blocks). */
static int orc_one(double *out, const uint16_t *q, const uint16_t *k_cache,
                   const uint16_t *v_cache, const int32_t *table, int L, int h, int num_q_heads,
                   int num_kv_heads, int head_dim, int block_size, int num_blocks, double scale,
                   int dtype, int window) {
    int d = head_dim;
    int g = h / (num_q_heads / num_kv_heads);
    for (int i = 0; i < d; ++i) out[i] = 0.0;
    if (L <= 0) return 0;
    int t_lo = (window > 0 && L > window) ? L - window : 0;
    double *Kc = (double *)malloc(sizeof(double) * (size_t)L * d);
    double *Vc = (double *)malloc(sizeof(double) * (size_t)L * d);
    double *z = (double *)malloc(sizeof(double) * (size_t)L);
    double *qd = (double *)malloc(sizeof(double) * (size_t)d);
    int rc = 0;
    /* gather: logical token t lives in page table[t / bs] at row t % bs */
    for (int t = t_lo; t < L && rc == 0; ++t) {
        int blk = table[t / block_size];
        if (blk < 0 || blk >= num_blocks) { rc = -1; break; }
        size_t row = (((size_t)blk * num_kv_heads + g) * block_size + (t % block_size)) * d;
        for (int i = 0; i < d; ++i) {
            Kc[(size_t)t * d + i] = orc_widen(k_cache[row + i], dtype);
            Vc[(size_t)t * d + i] = orc_widen(v_cache[row + i], dtype);
        }
    }
    if (rc == 0) {
        for (int i = 0; i < d; ++i) qd[i] = orc_widen(q[i], dtype);
        double m = -INFINITY;
        for (int t = t_lo; t < L; ++t) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i) acc += qd[i] * Kc[(size_t)t * d + i];
            z[t] = scale * acc;
            if (z[t] > m) m = z[t];
        }
        double denom = 0.0;
        for (int t = t_lo; t < L; ++t) {
            z[t] = exp(z[t] - m); /* softmax numerator, max-shifted */
            denom += z[t];
        }
        for (int t = t_lo; t < L; ++t)
            for (int i = 0; i < d; ++i) out[i] += z[t] * Vc[(size_t)t * d + i];
        for (int i = 0; i < d; ++i) out[i] /= denom;
    }
    free(Kc);
    free(Vc);
    free(z);
    free(qd);
    return rc;
}

/* Decode attention for every (sequence, q head), or only for the n_sel pairs listed
 * in sel[2*i] = sequence, sel[2*i+1] = q head (out is then [n_sel][head_dim]).
 * out (fp64) is [num_seqs][num_q_heads][head_dim] when sel is NULL.  window > 0
 * restricts every query to the last `window` tokens of its context (0 = whole context).
 * Returns the number of (s, h) whose table referenced an out-of-range block. */
int orc_decode_window(double *out, const uint16_t *q, const uint16_t *k_cache,
                      const uint16_t *v_cache, const int32_t *block_tables,
                      const int32_t *context_lens, int num_seqs, int num_q_heads,
                      int num_kv_heads, int head_dim, int block_size, int num_blocks,
                      int max_blocks_per_seq, double scale, int dtype, int window,
                      const int32_t *sel, int n_sel, int nthreads) {
    int n = sel ? n_sel : num_seqs * num_q_heads;
    int bad = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(+ : bad)
#endif
    for (int i = 0; i < n; ++i) {
        int s = sel ? sel[2 * i] : i / num_q_heads;
        int h = sel ? sel[2 * i + 1] : i % num_q_heads;
        const int32_t *table = block_tables + (size_t)s * max_blocks_per_seq;
        int L = context_lens[s];
        if (L > max_blocks_per_seq * block_size) { ++bad; continue; }
        const uint16_t *qs = q + ((size_t)s * num_q_heads + h) * head_dim;
        if (orc_one(out + (size_t)i * head_dim, qs, k_cache, v_cache, table, L, h, num_q_heads,
                    num_kv_heads, head_dim, block_size, num_blocks, scale, dtype, window) != 0)
            ++bad;
    }
    (void)nthreads;
    return bad;
}

/* The whole context (no sliding window). */
int orc_decode(double *out, const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
               const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
               int num_q_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
               int max_blocks_per_seq, double scale, int dtype, const int32_t *sel, int n_sel,
               int nthreads) {
    return orc_decode_window(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs,
                             num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                             max_blocks_per_seq, scale, dtype, 0, sel, n_sel, nthreads);
}

/* Multi-query (prefill / chunked prefill) attention over the paged cache: section 4
 * of the "IO-5 vLLM Paged Attention" note with a matrix Q (one row per new token of a
 * request, as continuous batching -- section 6 -- brings new requests' prompts into
 * the batch).  Reading where the pages are silent: causal, as in an autoregressive
 * model -- the chunk's n tokens sit at positions L - n .. L - 1 of a context of L
 * tokens already in the cache, and the token at position p attends to positions
 * 0 .. p (the last `window` of them under a sliding window).  That is exactly the
 * decode attention of a context of length p + 1, which is how it is evaluated here.
 *
 * q, out: [num_tokens][num_q_heads][head_dim] (out fp64); the tokens of sequence s are
 * rows query_start_loc[s] .. query_start_loc[s+1]-1.  With sel != NULL only the n_sel
 * (token, head) pairs sel[2i], sel[2i+1] are computed, into out[i][head_dim].  Returns
 * the number of outputs that could not be computed (chunk longer than its context,
 * or an out-of-range table entry). */
int orc_prefill(double *out, const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                const int32_t *block_tables, const int32_t *context_lens,
                const int32_t *query_start_loc, int num_seqs, int num_tokens, int num_q_heads,
                int num_kv_heads, int head_dim, int block_size, int num_blocks,
                int max_blocks_per_seq, double scale, int dtype, int window, const int32_t *sel,
                int n_sel, int nthreads) {
    int n_items = sel ? n_sel : num_tokens * num_q_heads;
    int bad = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 4) num_threads(nthreads) reduction(+ : bad)
#endif
    for (int i = 0; i < n_items; ++i) {
        int tok = sel ? sel[2 * i] : i / num_q_heads;
        int h = sel ? sel[2 * i + 1] : i % num_q_heads;
        double *o = out + (size_t)i * head_dim;
        for (int e = 0; e < head_dim; ++e) o[e] = 0.0;
        int s = 0;
        while (s < num_seqs && !(query_start_loc[s] <= tok && tok < query_start_loc[s + 1])) ++s;
        if (s == num_seqs) { ++bad; continue; }
        int n = query_start_loc[s + 1] - query_start_loc[s];
        int L = context_lens[s];
        if (n > L || L > max_blocks_per_seq * block_size) { ++bad; continue; }
        int pos = L - n + (tok - query_start_loc[s]);
        const int32_t *table = block_tables + (size_t)s * max_blocks_per_seq;
        if (orc_one(o, q + ((size_t)tok * num_q_heads + h) * head_dim, k_cache, v_cache, table,
                    pos + 1, h,
                    num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale, dtype,
                    window) != 0)
            ++bad;
    }
    (void)nthreads;
    return bad;
}

/* Threads the OpenMP runtime would use (1 without OpenMP). */
int orc_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
