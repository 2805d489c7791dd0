/*
 * CPU oracle for the Bloom-filtered int8 IVF top-k search.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may call this code:
 * only the tests, the smoke check and the benchmark's CPU-baseline leg load it.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * It is the plain definition, written out step by step, with no blocking,
 * fusion or reordering:
 *
 *   For each query b, independently:
 *   1. cs[c] = sum_j q[b][j] * cent[c][j] in int32, for every list c.
 *      (Probe: the most promising clusters are chosen first -- SilverTorch:
 *      Index as Model, section on how each component worked before.)
 *   2. Order the pairs (cs[c], c) by score descending, then list id ascending;
 *      the first P list ids are the probed lists.
 *   3. For every item i of every probed list (rows off[c] .. off[c+1]-1), the
 *      item is eligible when (sig[i][w] & m[b][w]) == m[b][w] for all words w
 *      (every item carries a compact signature written at publication time,
 *      and one bit operation tests it against the request at serving time --
 *      same page, Bloom index filter paragraph). Only eligible items are
 *      scored: the filter runs inside the chosen clusters and only the items
 *      that pass it are scored. A query may carry several alternative masks
 *      (an OR of values, e.g. any of several languages): the item is eligible
 *      when it passes at least one of them (oracle_search_or).
 *   4. Score = sum_j q[b][j] * x[i][j] in int32 (int8 storage, fused Int8 ANN
 *      paragraph). Order the candidates by score descending, then item id
 *      ascending, and output the first min(k, count); the remaining slots get
 *      id -1 and score INT32_MIN (large top-k: 2048 results from 64 probes,
 *      same paragraph).
 *
 * Readings where the pages are silent: inner product for both the probe and
 * the score; lower list id wins a probe tie; lower item id wins a score tie;
 * the item id is its row index unless the caller gives an id per row (an index
 * that has taken insertions keeps each list's rows together here, and the ids
 * say which items they are); the Bloom test alone decides eligibility (no
 * exact attribute re-check); short results are padded as above.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC oracle.c -o liboracle.so
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int32_t score;
    int64_t id;
} oracle_pair;

/* score descending, then id ascending */
static int pair_order(const void* pa, const void* pb)
{
    const oracle_pair* a = (const oracle_pair*)pa;
    const oracle_pair* b = (const oracle_pair*)pb;
    if (a->score != b->score) return a->score > b->score ? -1 : 1;
    if (a->id != b->id) return a->id < b->id ? -1 : 1;
    return 0;
}

/* sum_j a[j] * b[j], each factor widened to int32 */
int32_t oracle_dot(const int8_t* a, const int8_t* b, int32_t d)
{
    int32_t s = 0;
    for (int32_t j = 0; j < d; ++j) s += (int32_t)a[j] * (int32_t)b[j];
    return s;
}

/* 1 when every bit of the mask is set in the signature, word by word */
int32_t oracle_bloom_pass(const uint64_t* sig, const uint64_t* mask, int32_t W)
{
    for (int32_t w = 0; w < W; ++w)
        if ((sig[w] & mask[w]) != mask[w]) return 0;
    return 1;
}

/* Steps 1-2 for one query: the P best lists, best first. */
int32_t oracle_probe(const int8_t* q, const int8_t* cent, int32_t nlist, int32_t d,
                     int32_t P, int32_t* out_lists)
{
    oracle_pair* cs = (oracle_pair*)malloc(sizeof(oracle_pair) * (size_t)nlist);
    if (!cs) return -1;
    for (int32_t c = 0; c < nlist; ++c) {
        cs[c].score = oracle_dot(q, cent + (int64_t)c * d, d);
        cs[c].id = c;
    }
    qsort(cs, (size_t)nlist, sizeof(oracle_pair), pair_order);
    for (int32_t p = 0; p < P; ++p) out_lists[p] = (int32_t)cs[p].id;
    free(cs);
    return 0;
}

/* 1 when the signature passes at least one of the A masks m[0..A) (W words
 * each): an OR of alternative masks, each tested as above. */
static int32_t bloom_pass_any(const uint64_t* sig, const uint64_t* m, int32_t A, int32_t W)
{
    for (int32_t a = 0; a < A; ++a)
        if (oracle_bloom_pass(sig, m + (int64_t)a * W, W)) return 1;
    return 0;
}

/* Steps 3-4 for one query over a given set of lists, its A alternative masks
 * in m[0..A) (A = 1: the plain search). Row i is item row_ids[i] (item i when
 * row_ids is NULL). */
static int32_t search_lists(const int8_t* items, const uint64_t* sigs, const int64_t* off,
                            const int64_t* row_ids, int32_t d, int32_t W, const int8_t* q, const uint64_t* m,
                            int32_t A, const int32_t* lists, int32_t P, int32_t k,
                            int64_t* out_ids, int32_t* out_scores, int64_t* out_count)
{
    int64_t cap = 0;
    for (int32_t p = 0; p < P; ++p) cap += off[lists[p] + 1] - off[lists[p]];
    oracle_pair* cand = (oracle_pair*)malloc(sizeof(oracle_pair) * (size_t)(cap > 0 ? cap : 1));
    if (!cand) return -1;
    int64_t n = 0;
    for (int32_t p = 0; p < P; ++p) {
        int32_t c = lists[p];
        for (int64_t i = off[c]; i < off[c + 1]; ++i) {
            if (!bloom_pass_any(sigs + i * W, m, A, W)) continue;
            cand[n].score = oracle_dot(q, items + i * d, d);
            cand[n].id = row_ids ? row_ids[i] : i;
            ++n;
        }
    }
    qsort(cand, (size_t)n, sizeof(oracle_pair), pair_order);
    for (int32_t r = 0; r < k; ++r) {
        if (r < n) {
            out_ids[r] = cand[r].id;
            out_scores[r] = cand[r].score;
        } else {
            out_ids[r] = -1;
            out_scores[r] = INT32_MIN;
        }
    }
    if (out_count) *out_count = n;
    free(cand);
    return 0;
}

/*
 * The whole search for queries [b0, b1), each with A alternative masks (an
 * item is eligible when it passes any of them; A = 1 is the plain search).
 * Arrays are row-major: items int8 [n][d], sigs uint64 [n][W], off int64
 * [nlist+1], row_ids int64 [n] or NULL (item id of each row; NULL: the row
 * index), cent int8 [nlist][d], queries int8 [B][d], masks uint64 [B][A][W];
 * outputs int64/int32 [B][k]; out_probe int32 [B][P] and out_eligible int64
 * [B] may be NULL. nthreads > 1 runs queries in parallel (the result does not
 * depend on it). Returns 0, or -1 when an allocation failed.
 */
int32_t oracle_search_or(const int8_t* items, const uint64_t* sigs, const int64_t* off,
                         const int64_t* row_ids, const int8_t* cent, int64_t n, int32_t d, int32_t nlist,
                         int32_t W, const int8_t* queries, const uint64_t* masks, int32_t A, int32_t b0,
                         int32_t b1, int32_t P, int32_t k, int64_t* out_ids, int32_t* out_scores,
                         int32_t* out_probe, int64_t* out_eligible, int32_t nthreads)
{
    (void)n;
    int32_t err = 0;
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(| : err)
    for (int32_t b = b0; b < b1; ++b) {
        int32_t* lists = (int32_t*)malloc(sizeof(int32_t) * (size_t)P);
        if (!lists) { err |= 1; continue; }
        const int8_t* q = queries + (int64_t)b * d;
        const uint64_t* m = masks + (int64_t)b * A * W;
        if (oracle_probe(q, cent, nlist, d, P, lists) != 0) { err |= 1; free(lists); continue; }
        if (out_probe) memcpy(out_probe + (int64_t)(b - b0) * P, lists, sizeof(int32_t) * (size_t)P);
        int64_t cnt = 0;
        if (search_lists(items, sigs, off, row_ids, d, W, q, m, A, lists, P, k,
                         out_ids + (int64_t)(b - b0) * k, out_scores + (int64_t)(b - b0) * k,
                         &cnt) != 0)
            err |= 1;
        if (out_eligible) out_eligible[b - b0] = cnt;
        free(lists);
    }
    return err ? -1 : 0;
}

/* oracle_search_or with one mask per query (the plain search) */
int32_t oracle_search_ids(const int8_t* items, const uint64_t* sigs, const int64_t* off,
                          const int64_t* row_ids, const int8_t* cent, int64_t n, int32_t d, int32_t nlist,
                          int32_t W, const int8_t* queries, const uint64_t* masks, int32_t b0, int32_t b1,
                          int32_t P, int32_t k, int64_t* out_ids, int32_t* out_scores,
                          int32_t* out_probe, int64_t* out_eligible, int32_t nthreads)
{
    return oracle_search_or(items, sigs, off, row_ids, cent, n, d, nlist, W, queries, masks, 1, b0, b1, P, k,
                            out_ids, out_scores, out_probe, out_eligible, nthreads);
}

/* oracle_search_ids with every item id equal to its row index */
int32_t oracle_search(const int8_t* items, const uint64_t* sigs, const int64_t* off,
                      const int8_t* cent, int64_t n, int32_t d, int32_t nlist, int32_t W,
                      const int8_t* queries, const uint64_t* masks, int32_t b0, int32_t b1,
                      int32_t P, int32_t k, int64_t* out_ids, int32_t* out_scores,
                      int32_t* out_probe, int64_t* out_eligible, int32_t nthreads)
{
    return oracle_search_ids(items, sigs, off, NULL, cent, n, d, nlist, W, queries, masks, b0, b1, P, k,
                             out_ids, out_scores, out_probe, out_eligible, nthreads);
}

int32_t oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
