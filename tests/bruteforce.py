"""An independent numpy restatement of the search, for pinning the C oracle.

It takes each step from its plain definition with library primitives only:
int64 matrix products for the inner products, numpy bitwise ops for the Bloom
test and np.lexsort for the (score descending, id ascending) order. It shares
nothing with oracle/oracle.c beyond the definition.
"""
import numpy as np

INT32_MIN = np.iinfo(np.int32).min


def scores(q: np.ndarray, x: np.ndarray) -> np.ndarray:
    """int32 inner products of rows of q with rows of x, via an int64 matmul."""
    s = q.astype(np.int64) @ x.astype(np.int64).T
    assert np.all(np.abs(s) < 2**31)
    return s.astype(np.int32)


def order_desc(score: np.ndarray, ids: np.ndarray) -> np.ndarray:
    """Indices ordering by score descending, then id ascending."""
    return np.lexsort((ids, -score.astype(np.int64)))


def bloom_pass(sigs: np.ndarray, mask: np.ndarray) -> np.ndarray:
    """Boolean per row: all mask bits present in the signature (all words)."""
    sigs = sigs.view(np.uint64).reshape(sigs.shape[0], -1)
    mask = mask.view(np.uint64).reshape(1, -1)
    return np.all((sigs & mask) == mask, axis=1)


def probe(q, cent, P):
    cs = scores(q[None, :], cent)[0]
    o = order_desc(cs, np.arange(cent.shape[0]))
    return o[:P].astype(np.int32)


def search(items, sigs, offsets, centroids, queries, masks, nprobe, k, row_ids=None):
    """row_ids (optional): the item id of each row; by default the row index."""
    B = queries.shape[0]
    ids = np.full((B, k), -1, dtype=np.int64)
    out = np.full((B, k), INT32_MIN, dtype=np.int32)
    probes = np.zeros((B, nprobe), dtype=np.int32)
    elig = np.zeros(B, dtype=np.int64)
    for b in range(B):
        lists = probe(queries[b], centroids, nprobe)
        probes[b] = lists
        rows = np.concatenate([np.arange(offsets[c], offsets[c + 1]) for c in lists]) \
            if len(lists) else np.zeros(0, np.int64)
        rows = rows[bloom_pass(sigs[rows], masks[b])]
        elig[b] = rows.size
        if rows.size == 0:
            continue
        s = scores(queries[b][None, :], items[rows])[0]
        item = rows if row_ids is None else np.asarray(row_ids, dtype=np.int64)[rows]
        o = order_desc(s, item)[:k]
        ids[b, :o.size] = item[o]
        out[b, :o.size] = s[o]
    return ids, out, probes, elig


def search_or(items, sigs, offsets, centroids, queries, mask_sets, nprobe, k, row_ids=None):
    """search() with mask_sets [B, A, W]: an item is eligible when it passes any
    of its query's A masks."""
    B = queries.shape[0]
    ids = np.full((B, k), -1, dtype=np.int64)
    out = np.full((B, k), INT32_MIN, dtype=np.int32)
    probes = np.zeros((B, nprobe), dtype=np.int32)
    elig = np.zeros(B, dtype=np.int64)
    for b in range(B):
        lists = probe(queries[b], centroids, nprobe)
        probes[b] = lists
        rows = np.concatenate([np.arange(offsets[c], offsets[c + 1]) for c in lists]) \
            if len(lists) else np.zeros(0, np.int64)
        ok = np.zeros(rows.size, dtype=bool)
        for m in mask_sets[b]:
            ok |= bloom_pass(sigs[rows], m)
        rows = rows[ok]
        elig[b] = rows.size
        if rows.size == 0:
            continue
        s = scores(queries[b][None, :], items[rows])[0]
        item = rows if row_ids is None else np.asarray(row_ids, dtype=np.int64)[rows]
        o = order_desc(s, item)[:k]
        ids[b, :o.size] = item[o]
        out[b, :o.size] = s[o]
    return ids, out, probes, elig
