/*
 * st.h -- C ABI of the Bloom-filtered int8 IVF top-k search library (libst.so)
 * for NVIDIA B200 (sm_100a).
 *
 * What it computes. For each query b (an int8 vector q_b and a Bloom mask m_b):
 *   1. probe: score every IVF list c by the int32 inner product <q_b, cent_c>
 *      and keep the nprobe best lists (the best-scoring clusters are chosen
 *      first -- SilverTorch: Index as Model, section on how each component
 *      worked before);
 *   2. filter: inside the probed lists only, an item i is eligible when
 *      (sig_i[w] & m_b[w]) == m_b[w] for every signature word w (same page,
 *      section on redesigning each stage as a pure PyTorch module, Bloom index
 *      filter paragraph);
 *   3. score: eligible items only, by the int32 inner product <q_b, x_i> of
 *      int8 vectors (same section, fused Int8 ANN paragraph);
 *   4. top-k: the k best eligible items, ordered by score descending, then by
 *      item id ascending (large top-k: 2048 results from 64 probes with
 *      recall kept, same paragraph; SilverTorch: Index as Model, Spanish
 *      translation, table of compute cost efficiency, row on maximum top-k).
 *   Probe ties go to the lower list id. The item id is the row index in the
 *   arrays given to st_index_create. When fewer than k items are eligible, the
 *   remaining slots hold id -1 and score INT32_MIN. The Bloom test alone
 *   decides eligibility (a false-positive match is a legitimate result).
 *   The result is unique, so every call returns exactly the same bytes.
 *
 * Conventions. Arrays are dense and row-major. "Device" pointers are CUDA
 * device (or managed) memory on the index's device; "host" pointers may be
 * pageable or pinned. All calls return an st_status and never throw. Invalid
 * arguments are rejected on the host before any work is enqueued. There is no
 * CPU fallback: every step runs in the library's own CUDA kernels.
 */
#ifndef ST_H_
#define ST_H_

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct st_index st_index; /* opaque */

typedef enum {
    ST_OK = 0,
    ST_ERR_INVALID_ARG = 1,  /* null / non-device pointer, bad size, malformed offsets */
    ST_ERR_UNSUPPORTED = 2,  /* a size outside the supported limits below */
    ST_ERR_OOM = 3,          /* a device allocation failed */
    ST_ERR_CUDA = 4,         /* a CUDA runtime or launch error */
    ST_ERR_DEVICE = 5,       /* a kernel recorded an internal error (see st_index_check) */
    ST_ERR_SCRATCH_LIMIT = 6 /* st_probe_noalloc: the request needs more than its
                                fixed scratch (ST_PROBE_NOALLOC_SCRATCH_BYTES) */
} st_status;

/* Supported limits (ST_ERR_UNSUPPORTED outside them). */
#define ST_MAX_D 512         /* d must be a multiple of 16 in [16, 512] */
#define ST_MAX_K 262144      /* 1 <= k <= 262144 */
#define ST_SMALL_K 4096      /* k above this takes a global-memory final top-k and
                                needs device memory for the key of every row of the
                                probed lists (ST_ERR_OOM when it does not fit) */
#define ST_MAX_NPROBE 4096   /* 1 <= nprobe <= min(nlist, 4096) */
#define ST_MAX_B 32768       /* 1 <= B <= 32768 queries per call */
#define ST_MAX_OR 7          /* alternative masks per query (st_search_extras.n_or) */
/* n < 2^31 items; sig_words is 1 (64-bit signatures) or 2 (128-bit). */

/*
 * Build an index. Copies every input into library-owned device memory, so the
 * caller may free or reuse its arrays as soon as the call returns (the call
 * waits for its copies on `stream`). Inputs may be device or host memory.
 *
 *   items        int8   [n][d]          item embeddings, rows grouped by list:
 *                                       list c owns rows off[c] .. off[c+1]-1
 *   sigs         uint64 [n][sig_words]  Bloom signatures; word 0 holds bits
 *                                       0-63, word 1 bits 64-127
 *   list_offsets int64  [nlist+1]       CSR offsets: off[0] = 0, off[nlist] = n,
 *                                       nondecreasing (empty lists allowed)
 *   centroids    int8   [nlist][d]      IVF list centroids
 *   out          receives the index; *out is NULL on failure
 *
 * Errors: INVALID_ARG (null pointer, n < 1, nlist < 1, malformed offsets),
 * UNSUPPORTED (d or sig_words outside the limits, n >= 2^31), OOM, CUDA.
 * The index lives on the device that is current during this call.
 */
st_status st_index_create(const int8_t* items, const uint64_t* sigs,
                          const int64_t* list_offsets, const int8_t* centroids,
                          int64_t n, int32_t d, int32_t nlist, int32_t sig_words,
                          cudaStream_t stream, st_index** out);

/*
 * Search B queries. Asynchronous on `stream`: it enqueues the kernels and
 * returns without waiting for them; results are valid once `stream` reaches
 * this point. Never synchronizes the host.
 *
 *   queries    device int8   [B][d]
 *   qmasks     device uint64 [B][sig_words]
 *   out_ids    device int64  [B][k]   caller-owned
 *   out_scores device int32  [B][k]   caller-owned
 *
 * Scratch memory comes from a stream-ordered pool owned by the index and is
 * returned to it when the search completes, so concurrent calls on different
 * streams may share one index. The index itself is never modified.
 *
 * Errors: INVALID_ARG (null or non-device pointer, B < 1, k < 1, nprobe < 1 or
 * nprobe > nlist), UNSUPPORTED (B, k or nprobe above the limits), OOM, CUDA.
 * A kernel-side internal error is reported by st_index_check.
 */
st_status st_search(const st_index* idx, const int8_t* queries, const uint64_t* qmasks,
                    int32_t B, int32_t nprobe, int32_t k,
                    int64_t* out_ids, int32_t* out_scores, cudaStream_t stream);

/* Optional extra inputs and outputs of st_search_ex; any member may be NULL. */
typedef struct {
    int64_t* eligible; /* device int64 [B]: items of each query's probed lists
                          that pass its mask (the number of (query, item) scores
                          computed; items later dropped by exclusion or deletion
                          are included) */
    int32_t* probe;    /* device int32 [B][nprobe]: the probed lists, best first */
    /* Timing hooks: each non-NULL event is recorded on `stream` at a stage
       boundary -- [0] before the probe kernel, [1] after it, [2] after the plan
       kernels, [3] after the list scan, [4] after the final top-k. */
    cudaEvent_t stage_events[5];
    /* device uint64 [B][sig_words]: negative rules. An item whose signature
       holds every bit of query b's exclude mask is not a result of query b
       (an all-zero exclude mask excludes nothing). A negative targeting rule
       of the pages' advertiser-defined targeting, tested like the mask itself
       (so a Bloom false positive excludes too). */
    const uint64_t* exclude_masks;
    /* device int64 [B]: candidate keys the list scan wrote for each query's
       final top-k (at most its eligible count; fewer when the scan dropped
       keys that could no longer enter the top-k). */
    int64_t* candidates;
    /* device uint64 [B][n_or][sig_words]: alternative masks, an OR of values
       (for example any of several languages). An item is eligible for query b
       when its signature passes qmasks[b] or any of query b's n_or
       alternatives, each tested like the mask itself; the list scan tests
       them all in the same pass, and eligible counts count an item once.
       n_or = 0 (or_masks may then be NULL): the plain mask. INVALID_ARG when
       n_or is outside [0, ST_MAX_OR] or or_masks is not a device pointer. */
    const uint64_t* or_masks;
    int32_t n_or;
} st_search_extras;

/* st_search with optional extra outputs (extras may be NULL). */
st_status st_search_ex(const st_index* idx, const int8_t* queries, const uint64_t* qmasks,
                       int32_t B, int32_t nprobe, int32_t k,
                       int64_t* out_ids, int32_t* out_scores,
                       const st_search_extras* extras, cudaStream_t stream);

/*
 * st_search for host-resident queries and results: copies queries and masks to
 * the device, searches, copies ids and scores back, and waits for `stream`
 * before returning, so the outputs are ready on return. Pinned host memory
 * makes the copies asynchronous DMA; pageable memory also works.
 * Same arguments and errors as st_search, with every array in host memory.
 */
st_status st_search_host(const st_index* idx, const int8_t* queries, const uint64_t* qmasks,
                         int32_t B, int32_t nprobe, int32_t k,
                         int64_t* out_ids, int32_t* out_scores, cudaStream_t stream);

/*
 * st_search_host without the wait, for a serving loop that keeps several
 * batches in flight (one stream each): enqueues the copy of queries and masks
 * to the device, the search and the copy of ids and scores back, and returns.
 * Every host array must be page-locked (cudaHostAlloc / cudaHostRegister) --
 * pageable memory is refused with INVALID_ARG, since its copies would block.
 * The outputs are complete once `stream` has finished this work (an event or
 * a stream synchronize); until then the caller must neither read the outputs
 * nor change the inputs. Same arguments and errors as st_search otherwise.
 */
st_status st_search_host_async(const st_index* idx, const int8_t* queries, const uint64_t* qmasks,
                               int32_t B, int32_t nprobe, int32_t k,
                               int64_t* out_ids, int32_t* out_scores, cudaStream_t stream);

/*
 * Wait for `stream`, then report and clear the index's device-side error word.
 * Returns ST_OK, ST_ERR_DEVICE when a kernel recorded an internal error since
 * the last check (no result produced meanwhile should be trusted), or
 * ST_ERR_CUDA when the stream itself failed.
 */
st_status st_index_check(const st_index* idx, cudaStream_t stream);

/* Tuning options (all have working defaults). */
typedef enum {
    /* Device memory (bytes) that one search may use for candidate keys
       (default 2 GiB). Searches whose candidates exceed it stay exact: the
       affected queries take a slower exact path. */
    ST_OPT_CANDIDATE_BYTES = 1,
    /* Force the per-query candidate capacity (keys) instead of deriving it;
       0 restores the default. Values below k + 1024 are raised to that. */
    ST_OPT_CANDIDATE_CAPACITY = 2,
    /* Added to every item id the index returns (default 0): an index built
       from rows [r0, r1) of a larger collection, with this option set to r0,
       returns ids of that collection -- one document shard of it (see
       st_merge_topk). Rejected with UNSUPPORTED unless offset plus the rows
       the index has room for stays below 2^31. */
    ST_OPT_ID_OFFSET = 3,
    /* Make room now for insertions (st_index_insert): at least
       ceil(value / ST_INSERT_CHUNK) more append chunks, i.e. value rows added
       to one list, without a reallocation later. Growing copies the index
       once and needs the old and the new arrays at the same time. 0 is a
       no-op; the room is never given back. OOM when it cannot be had,
       UNSUPPORTED when the ids would reach 2^31 (with the id offset). */
    ST_OPT_INSERT_RESERVE = 4,
    /* Lists probed by at least this many queries of a batch are scanned as
       dense tiles on the tensor cores (int8 x int8 -> int32, up to 32 queries
       per tile) instead of per-pair dp4a; results are identical. With a value
       above 1, a list probed by fewer queries goes there too when the batch
       has at least 2048 (query, list) probes and its queries expect together
       at least 0.75 eligible pairs per row (each query's share of a fixed
       sample of 512 of the index's rows, taken at creation, that passes its
       masks). Default 8; 1 sends every probed list there; 0 turns the
       tensor-core scan off. Only d = 64 and d = 128 have the tensor-core
       scan. At most ST_MAX_B. */
    ST_OPT_DENSE_MIN_QUERIES = 5
} st_option;

/* Set an option; INVALID_ARG for an unknown option or a negative value.
   Not safe to call while a search on the same index is being enqueued, and
   ST_OPT_INSERT_RESERVE waits for the device like st_index_insert does. */
st_status st_index_set_option(st_index* idx, st_option opt, int64_t value);

/*
 * Allocation-free coarse probe: step 1 above alone (each query's nprobe best
 * lists, best first, ties to the lower list id -- exactly the lists st_search
 * probes and reports in st_search_extras.probe), without allocating any
 * memory. The method has no such call: it is a library addition for callers
 * that must not allocate device memory at query time, e.g. a request router
 * that has handed the rest of the GPU's memory to a fixed-size cache or to
 * another process, or that cannot accept the synchronisation and latency
 * spikes that cudaMalloc/cudaFree and a memory pool's growth can cause, and
 * only needs to know which lists (or the shards holding them) a query reaches.
 *
 *   queries    device int8  [B][d]
 *   out_probe  device int32 [B][nprobe]   caller-owned
 *
 * Its scratch is one fixed array of ST_PROBE_NOALLOC_SCRATCH_BYTES in the
 * library's device memory (one per device, created when the library is
 * loaded), needing B*4 (rounded up to 256) + B*S*nprobe*8 bytes, S being the
 * number of centroid slices per query the probe picks (S = 1 for B >= 296 on
 * a 148-SM GPU, at most 32), plus B*nlist*8 bytes when nlist exceeds 16384*S.
 * Requests that need more are rejected on the host with ST_ERR_SCRATCH_LIMIT
 * before anything is enqueued; smaller B or nprobe fit. The part that must
 * start at zero (the per-query completion counters) is cleared on `stream`
 * by every call (cudaMemsetAsync, which allocates nothing).
 *
 * All calls on a device share the one array, so calls whose work may overlap
 * on the GPU -- on different streams, or from different host threads without
 * ordering -- race on it and give wrong results. Issue them on one stream, or
 * order them with events.
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, which may load the library's GPU code) and raises
 * the kernel's shared-memory limit; make that first call, for example with a
 * small warm-up request, before any stream capture begins.
 *
 * Asynchronous on `stream` like st_search; kernel-side errors are reported by
 * st_index_check. Errors: INVALID_ARG (null index, null or non-device pointer,
 * misaligned queries (16 bytes) or out_probe (4 bytes), B < 1, nprobe < 1 or
 * nprobe > nlist), UNSUPPORTED (nprobe above ST_MAX_NPROBE, B*nprobe >= 2^31),
 * SCRATCH_LIMIT, CUDA.
 */
#define ST_PROBE_NOALLOC_SCRATCH_BYTES (16u << 20) /* 16 MiB */
st_status st_probe_noalloc(const st_index* idx, const int8_t* queries, int32_t B, int32_t nprobe,
                           int32_t* out_probe, cudaStream_t stream);

/*
 * Exact merge of document-shard results. Splitting the items into disjoint
 * shards (each searched as its own index with the same centroids, nprobe and
 * the shard's ST_OPT_ID_OFFSET) and keeping the k best of the union of the
 * shards' top-k lists gives exactly the unsharded top-k: every item of the
 * global top-k is in the top-k of its own shard. The pages name document
 * sharding as the way to scale out once one GPU is used up (SilverTorch:
 * Index as Model, section on engineering for scale and freshness, vertical and
 * horizontal scaling paragraph); this call is its merge step, after the
 * caller has gathered the shards' results (for example with an NCCL
 * all-gather) into one device buffer.
 *
 *   ids        device int64 [G][B][k]   shard g's ids for query b (id -1 = padding)
 *   scores     device int32 [G][B][k]
 *   out_ids    device int64 [B][k]      merged, ordered like st_search, padded
 *   out_scores device int32 [B][k]
 *
 * Ids must be distinct across shards (disjoint shards) and below 2^31.
 * Asynchronous on `stream`; allocates nothing. Errors: INVALID_ARG (null or
 * non-device pointer, G < 1, B < 1, k < 1), UNSUPPORTED (k above ST_SMALL_K, or
 * G * k above ST_MERGE_MAX_KEYS), CUDA. A kernel-side error (an id out of
 * range) sets the calling device's merge error word, read by st_merge_check.
 */
#define ST_MERGE_MAX_KEYS 16384
st_status st_merge_topk(const int64_t* ids, const int32_t* scores, int32_t G, int32_t B, int32_t k,
                        int64_t* out_ids, int32_t* out_scores, cudaStream_t stream);

/*
 * Exact top-k of the union of G result lists that may share items (the same
 * item, with the same score, in several lists): like st_merge_topk, except
 * that an item is kept once. Each list must be ordered as st_search orders
 * its results (score descending, then id ascending, padding last) -- every
 * st_search result is. This is the merge step of an OR of several masks per
 * query (pass if any mask passes; a targeting rule allowing several values
 * of a field): search once per mask, then take the union. Same arguments,
 * limits and errors as st_merge_topk.
 */
st_status st_merge_topk_union(const int64_t* ids, const int32_t* scores, int32_t G, int32_t B, int32_t k,
                              int64_t* out_ids, int32_t* out_scores, cudaStream_t stream);

/* Wait for `stream`, then report and clear the merge error word of the
   current device: ST_OK, ST_ERR_DEVICE (an input id was out of range), or
   ST_ERR_CUDA. */
st_status st_merge_check(cudaStream_t stream);

/*
 * Streaming in-place update: replace the embedding rows and/or the Bloom
 * signatures of m existing items, without a rebuild. The pages keep the
 * index fresh between full snapshots by streaming new signals into the
 * in-memory model (SilverTorch: Index as Model, section on engineering for
 * scale and freshness, index freshness paragraph); this call is that step for
 * items whose row stays in its list (new items: st_index_insert; removal:
 * st_index_delete).
 *
 *   ids    device int64 [m]             item ids of the index (without any
 *                                       ST_OPT_ID_OFFSET): rows given to
 *                                       st_index_create or ids returned by
 *                                       st_index_insert; distinct within a call
 *   items  device int8  [m][d] or NULL  new rows (NULL: rows unchanged)
 *   sigs   device uint64 [m][sig_words] or NULL  new signatures (NULL: unchanged)
 *
 * The signature bit-planes the search reads are rewritten with the
 * signatures. Asynchronous on `stream`: searches enqueued later on the same
 * stream see the new values; searches on other streams must be ordered after
 * it by the caller (they read the same memory), and two updates must not
 * overlap. An id that the index never handed out (outside [0, n) and not
 * returned by st_index_insert) is skipped and recorded in the index's error
 * word (st_index_check). Errors: INVALID_ARG (null index, m < 0, null or
 * non-device ids when m > 0, non-device items / sigs, both NULL), CUDA.
 */
st_status st_index_update(st_index* idx, const int64_t* ids, const int8_t* items, const uint64_t* sigs,
                          int64_t m, cudaStream_t stream);

/*
 * Delete m items in place (tombstones): a deleted item is never returned
 * again, by any later search on `stream` (other streams: order them after it).
 * ids are item ids of the index, as for st_index_update; deleting twice is
 * harmless; st_index_update does not revive an item. Deleted rows still take
 * part in the scan (their scores are dropped before the final top-k) and in
 * st_search_extras.eligible. The first deletion allocates a bitmap with one
 * bit per row the index has room for. An id the index never handed out is
 * skipped and recorded in the index's error word. Errors: INVALID_ARG (null index, m < 0, null or
 * non-device ids when m > 0), OOM, CUDA.
 */
st_status st_index_delete(st_index* idx, const int64_t* ids, int64_t m, cudaStream_t stream);

/*
 * Insert m new items into existing IVF lists without a rebuild (the insertion
 * half of index freshness: SilverTorch: Index as Model, section on engineering
 * for scale and freshness, index freshness paragraph).
 *
 *   lists   HOST int32 [m]                 the list each new item joins, in [0, nlist)
 *   items   device int8 [m][d]             the new rows (16-byte aligned)
 *   sigs    device uint64 [m][sig_words]   their Bloom signatures
 *   out_ids HOST int64 [m]                 receives the id given to each item
 *
 * Layout: each list owns, after its creation rows, zero or more append chunks
 * of ST_INSERT_CHUNK rows placed after all creation rows; a list's new items
 * fill its last append chunk in argument order, then a fresh one. An item's
 * id is its row, so ids are >= n (the creation rows), unique, never reused and
 * stable, but not consecutive: the unfilled rows of each list's last append
 * chunk are ids no call returned yet. ST_OPT_ID_OFFSET is added to them in
 * search results, like to every id; on a document shard built from rows
 * [r0, r1) of a collection, inserted ids land at r1 - r0 + offset and above,
 * which may be ids of the next shard, so a sharded deployment needs its own
 * id map for inserted items (or one shard that takes all insertions last in
 * the id space). The item's Bloom bit-planes are written as
 * by st_index_update, and later searches on `stream` see it (other streams:
 * order them after this call). When the append chunks run out, the index
 * grows (the item, signature and plane arrays are copied once into arrays
 * with at least twice the append room; see ST_OPT_INSERT_RESERVE).
 *
 * The call waits for `stream` (and, when it grows the index or its chunk
 * table, for the device) before it returns, so the host arrays may be reused
 * at once. Errors, with the index unchanged: INVALID_ARG (null index, m < 0,
 * null host arrays or non-device items / sigs when m > 0, a list id outside
 * [0, nlist)), UNSUPPORTED (ids would reach 2^31 with the id offset), OOM;
 * CUDA if a copy or kernel fails (the index should then be destroyed).
 */
#define ST_INSERT_CHUNK 512
st_status st_index_insert(st_index* idx, const int32_t* lists, const int8_t* items, const uint64_t* sigs,
                          int64_t m, int64_t* out_ids, cudaStream_t stream);

/* Free the index (NULL-safe). Waits for the device to finish work that may
   still use it. */
void st_index_destroy(st_index* idx);

/* Static text for a status code. */
const char* st_status_string(st_status s);

#ifdef __cplusplus
}
#endif
#endif /* ST_H_ */
