/*
 * Paged KV-cache oracle: plain, slow, obviously correct CPU code in fp64.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  It shares no
 * code, header, table or helper with the CUDA library; neither includes or
 * links the other.
 *
 * Sources (web pages on paged attention; cited by title and section):
 *   [Explained]  "Paged Attention Explained: How LLMs Manage GPU Memory for
 *                Faster AI Inference"
 *   [Wiki]       "PagedAttention: paging the KV cache like an OS pages memory"
 *   [Index]      "PagedAttention and KV Cache Compression: Optimizing LLM
 *                Inference"
 *
 * What is computed, function by function:
 *   oracle_calculate_blocks  block count = ceil(tokens / block_size), with the
 *                            two argument errors of the example program in
 *                            [Explained] "Practical Example: Understanding
 *                            Block Allocation".
 *   oracle_kv_write          the cache update: each new token's K and V row is
 *                            stored at its slot = physical_block * block_size +
 *                            offset ([Explained] "Step 1"/"Step 2",
 *                            [Index] "5. Real-World Consequences": a token
 *                            fills the current block, a new block only when
 *                            full).  slot < 0 means "no write".
 *   oracle_copy_blocks       block-granularity copy-on-write copies ([Wiki]
 *                            "How it works", second paragraph).
 *   oracle_paged_prefill     multi-query (prefill / chunked append) attention:
 *                            every query row is the decode definition over the
 *                            tokens up to its own position (causal).
 *   oracle_paged_decode      single-query attention over the paged cache.
 *                            The attention itself is ordinary softmax
 *                            attention; only the storage layout differs
 *                            ([Wiki] "How it works").  The oracle therefore
 *                            (1) resolves the block table into a contiguous
 *                            copy of the sequence's keys and values
 *                            ([Explained] "Step 3: Maintain a Block Table",
 *                            "Step 4: Retrieve Cached Data During Attention")
 *                            and (2) evaluates the textbook definition
 *                            out = sum_t w_t V_t / sum_t w_t,
 *                            w_t = exp(scale * q.K_t - max), in double.
 *   Grouped KV heads follow the cache-size formula of [Explained] "Why Does
 *   the KV Cache Consume So Much Memory?", where the number of KV heads is a
 *   factor of its own; query head h reads KV head h / (Hq / Hkv).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - decode has one query (the newest token); it attends to every cached
 *     token 0 .. seq_len-1 of its sequence, so no further causal mask applies;
 *   - seq_len == 0 yields an all-zero output row;
 *   - slots past seq_len in the last block and unused table entries are never
 *     read (the last block is partially filled, [Explained] "Partial Block
 *     Waste");
 *   - element types are bf16 or fp32; bf16 values are widened exactly.
 *
 * Pins: every function is checked in tests/test_oracle.py against values the
 * pages print, closed forms, invariants and brute force; none is unpinned.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_BF16 = 0, ORACLE_F32 = 1 };

/* Exact widening of one stored element to double.  A bf16 value is the upper
 * half of an IEEE binary32, so shifting its 16 bits up gives the same number. */
static double load_elem(const void *base, int64_t index, int dtype)
{
    float f;
    if (dtype == ORACLE_BF16) {
        uint16_t h = ((const uint16_t *)base)[index];
        uint32_t u = ((uint32_t)h) << 16;
        memcpy(&f, &u, sizeof f);
    } else {
        f = ((const float *)base)[index];
    }
    return (double)f;
}

static int64_t elem_size(int dtype) { return dtype == ORACLE_BF16 ? 2 : 4; }

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Block count for a request: rounded-up division of the cached token count by
 * the tokens per block.  Returns 0 on success, -1 for a negative token count
 * and -2 for a non-positive block size (the two errors of the example). */
int oracle_calculate_blocks(int64_t token_count, int64_t block_size, int64_t *blocks)
{
    if (token_count < 0) return -1;
    if (block_size <= 0) return -2;
    int64_t n = token_count / block_size;
    if (n * block_size < token_count) n += 1;
    *blocks = n;
    return 0;
}

/* Cache update.  k, v: [N, Hkv, D]; k_cache, v_cache: [num_blocks, bs, Hkv, D].
 * For token n with slot s >= 0: block = s / bs, offset = s % bs, and every
 * (h, d) element is copied byte for byte into
 * cache[block][offset][h][d].  Returns the number of slots that were out of
 * range (those are skipped). */
int64_t oracle_kv_write(const void *k, const void *v, void *k_cache, void *v_cache,
                        const int64_t *slot_mapping, int64_t N, int64_t Hkv, int64_t D,
                        int64_t bs, int64_t num_blocks, int dtype)
{
    const int64_t es = elem_size(dtype);
    int64_t bad = 0;
    for (int64_t n = 0; n < N; ++n) {
        const int64_t s = slot_mapping[n];
        if (s < 0) continue;
        const int64_t block = s / bs;
        const int64_t offset = s % bs;
        if (block >= num_blocks) { ++bad; continue; }
        for (int64_t h = 0; h < Hkv; ++h) {
            for (int64_t d = 0; d < D; ++d) {
                const int64_t src = (n * Hkv + h) * D + d;
                const int64_t dst = ((block * bs + offset) * Hkv + h) * D + d;
                memcpy((char *)k_cache + dst * es, (const char *)k + src * es, (size_t)es);
                memcpy((char *)v_cache + dst * es, (const char *)v + src * es, (size_t)es);
            }
        }
    }
    return bad;
}

/* Copy-on-write block copies.  mapping: [P, 2] (src, dst) physical block ids.
 * For each pair in order, the whole dst block (block_bytes bytes, i.e.
 * bs * Hkv * D * element size) of both caches becomes a copy of the src
 * block.  Returns the number of pairs skipped for an id outside
 * [0, num_blocks). */
int64_t oracle_copy_blocks(void *k_cache, void *v_cache, const int64_t *mapping, int64_t P,
                           int64_t block_bytes, int64_t num_blocks)
{
    int64_t bad = 0;
    for (int64_t i = 0; i < P; ++i) {
        const int64_t src = mapping[2 * i], dst = mapping[2 * i + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) { ++bad; continue; }
        for (int64_t byte = 0; byte < block_bytes; ++byte) {
            ((char *)k_cache)[dst * block_bytes + byte] = ((const char *)k_cache)[src * block_bytes + byte];
            ((char *)v_cache)[dst * block_bytes + byte] = ((const char *)v_cache)[src * block_bytes + byte];
        }
    }
    return bad;
}

/* One output row: the query at element offset q_off of q against the first L
 * cached tokens of sequence b, KV head kvh. */
static int attend_row(double *out_row, const void *q, int64_t q_off, const void *k_cache,
                      const void *v_cache, int dtype, const int32_t *block_tables,
                      int64_t max_blocks, int64_t b, int64_t L, int64_t kvh, int64_t Hkv,
                      int64_t D, int64_t bs, int64_t num_blocks, double scale)
{
    int64_t t, d;

    for (d = 0; d < D; ++d) out_row[d] = 0.0;
    if (L <= 0) return 0;
    if (L > max_blocks * bs) return -2;

    /* (1) Resolve the block table: logical token t lives in logical block
     *     t / bs at offset t % bs; the table gives that block's physical id. */
    double *Kc = (double *)malloc(sizeof(double) * (size_t)(L * D));
    double *Vc = (double *)malloc(sizeof(double) * (size_t)(L * D));
    double *s = (double *)malloc(sizeof(double) * (size_t)L);
    if (!Kc || !Vc || !s) { free(Kc); free(Vc); free(s); return -3; }
    for (t = 0; t < L; ++t) {
        const int64_t logical = t / bs;
        const int64_t offset = t % bs;
        const int64_t phys = block_tables[b * max_blocks + logical];
        if (phys < 0 || phys >= num_blocks) { free(Kc); free(Vc); free(s); return -2; }
        for (d = 0; d < D; ++d) {
            const int64_t idx = ((phys * bs + offset) * Hkv + kvh) * D + d;
            Kc[t * D + d] = load_elem(k_cache, idx, dtype);
            Vc[t * D + d] = load_elem(v_cache, idx, dtype);
        }
    }

    /* (2) Scores s_t = scale * sum_d q[b,h,d] * K[t,d]. */
    double smax = -INFINITY;
    for (t = 0; t < L; ++t) {
        double acc = 0.0;
        for (d = 0; d < D; ++d) acc += load_elem(q, q_off + d, dtype) * Kc[t * D + d];
        s[t] = scale * acc;
        if (s[t] > smax) smax = s[t];
    }

    /* (3) Softmax weights (shifted by the maximum only to stay in range) and
     *     the weighted sum of values. */
    double wsum = 0.0;
    for (t = 0; t < L; ++t) {
        const double w = exp(s[t] - smax);
        wsum += w;
        for (d = 0; d < D; ++d) out_row[d] += w * Vc[t * D + d];
    }
    for (d = 0; d < D; ++d) out_row[d] /= wsum;

    free(Kc); free(Vc); free(s);
    return 0;
}

/* Decode row: query head h of sequence b attends to all seq_lens[b] tokens. */
static int decode_row(double *out_row, const void *q, const void *k_cache, const void *v_cache,
                      int dtype, const int32_t *block_tables, int64_t max_blocks,
                      const int32_t *seq_lens, int64_t b, int64_t h, int64_t Hq, int64_t Hkv,
                      int64_t D, int64_t bs, int64_t num_blocks, double scale)
{
    const int64_t G = Hq / Hkv;
    const int64_t kvh = h / G;
    return attend_row(out_row, q, (b * Hq + h) * D, k_cache, v_cache, dtype, block_tables,
                      max_blocks, b, seq_lens[b], kvh, Hkv, D, bs, num_blocks, scale);
}

/* Decode attention.  q: [B, Hq, D]; caches: [num_blocks, bs, Hkv, D];
 * block_tables: [B, max_blocks] int32; seq_lens: [B] int32; out: [B, Hq, D]
 * doubles.  If rows_b/rows_h are non-NULL only the listed (b, h) rows are
 * computed, into out_rows[nrows, D]; otherwise all B*Hq rows go to out.
 * Returns 0, -1 for bad dimensions, -2 for a block id or length outside the
 * table/pool, -3 for an allocation failure. */
int oracle_paged_decode(double *out, const void *q, const void *k_cache, const void *v_cache,
                        int dtype, const int32_t *block_tables, int64_t max_blocks,
                        const int32_t *seq_lens, int64_t B, int64_t Hq, int64_t Hkv, int64_t D,
                        int64_t bs, int64_t num_blocks, double scale, const int64_t *rows_b,
                        const int64_t *rows_h, int64_t nrows)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || bs <= 0 || Hq % Hkv != 0) return -1;
    const int64_t total = rows_b ? nrows : B * Hq;
    int status = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < total; ++r) {
        const int64_t b = rows_b ? rows_b[r] : r / Hq;
        const int64_t h = rows_b ? rows_h[r] : r % Hq;
        const int rc = decode_row(out + r * D, q, k_cache, v_cache, dtype, block_tables,
                                  max_blocks, seq_lens, b, h, Hq, Hkv, D, bs, num_blocks, scale);
        if (rc != 0) {
#pragma omp critical
            status = rc;
        }
    }
    return status;
}

/* Multi-query (prefill / chunked append) attention.  Sequence b holds
 * L = seq_lens[b] tokens, the last Q = cu_q[b+1] - cu_q[b] of which are this
 * call's queries, packed as rows cu_q[b] .. cu_q[b+1]-1 of q [T, Hq, D].  Query
 * i of sequence b sits at position L - Q + i and attends causally, to tokens
 * 0 .. L - Q + i: each row is the decode definition with that many tokens.
 * out: [T, Hq, D] doubles.  Returns the first nonzero status of a row, -1 for
 * bad dimensions or Q > L. */
int oracle_paged_prefill(double *out, const void *q, const void *k_cache, const void *v_cache,
                         int dtype, const int32_t *block_tables, int64_t max_blocks,
                         const int32_t *seq_lens, const int32_t *cu_q, int64_t B, int64_t Hq,
                         int64_t Hkv, int64_t D, int64_t bs, int64_t num_blocks, double scale)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || bs <= 0 || Hq % Hkv != 0) return -1;
    const int64_t T = cu_q[B];
    for (int64_t b = 0; b < B; ++b)
        if (cu_q[b + 1] < cu_q[b] || cu_q[b + 1] - cu_q[b] > seq_lens[b]) return -1;
    int status = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < T * Hq; ++r) {
        const int64_t row = r / Hq, h = r % Hq;
        int64_t b = 0;
        while (cu_q[b + 1] <= row) ++b;
        const int64_t Q = cu_q[b + 1] - cu_q[b];
        const int64_t i = row - cu_q[b];
        const int64_t visible = seq_lens[b] - Q + i + 1; /* causal: up to its own position */
        const int64_t kv_head = h / (Hq / Hkv);
        const int rc = attend_row(out + r * D, q, r * D, k_cache, v_cache, dtype, block_tables,
                                  max_blocks, b, visible, kv_head, Hkv, D, bs, num_blocks, scale);
        if (rc != 0) {
#pragma omp critical
            status = rc;
        }
    }
    return status;
}
