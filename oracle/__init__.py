"""ctypes front end of the CPU oracle (oracle.c).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the CUDA library or its binding.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import OUT, build

_lib = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load (building first if needed) the oracle, or a given build of it."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        build()
        _lib = _bind(ctypes.CDLL(OUT))
    return _lib


def _bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    P = ctypes.c_void_p
    i32, i64 = ctypes.c_int32, ctypes.c_int64
    lib.oracle_dot.argtypes = [P, P, i32]
    lib.oracle_dot.restype = i32
    lib.oracle_bloom_pass.argtypes = [P, P, i32]
    lib.oracle_bloom_pass.restype = i32
    lib.oracle_probe.argtypes = [P, P, i32, i32, i32, P]
    lib.oracle_probe.restype = i32
    lib.oracle_search.argtypes = [P, P, P, P, i64, i32, i32, i32, P, P, i32, i32, i32, i32,
                                  P, P, P, P, i32]
    lib.oracle_search.restype = i32
    lib.oracle_search_ids.argtypes = [P, P, P, P, P, i64, i32, i32, i32, P, P, i32, i32, i32, i32,
                                      P, P, P, P, i32]
    lib.oracle_search_ids.restype = i32
    lib.oracle_search_or.argtypes = [P, P, P, P, P, i64, i32, i32, i32, P, P, i32, i32, i32, i32, i32,
                                     P, P, P, P, i32]
    lib.oracle_search_or.restype = i32
    lib.oracle_max_threads.argtypes = []
    lib.oracle_max_threads.restype = i32
    return lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def dot(a: np.ndarray, b: np.ndarray, lib=None) -> int:
    lib = lib or load()
    a = np.ascontiguousarray(a, dtype=np.int8)
    b = np.ascontiguousarray(b, dtype=np.int8)
    return int(lib.oracle_dot(_ptr(a), _ptr(b), a.size))


def bloom_pass(sig: np.ndarray, mask: np.ndarray, lib=None) -> bool:
    lib = lib or load()
    sig = np.ascontiguousarray(sig, dtype=np.uint64)
    mask = np.ascontiguousarray(mask, dtype=np.uint64)
    return bool(lib.oracle_bloom_pass(_ptr(sig), _ptr(mask), sig.size))


def probe(q: np.ndarray, cent: np.ndarray, P: int, lib=None) -> np.ndarray:
    lib = lib or load()
    q = np.ascontiguousarray(q, dtype=np.int8)
    cent = np.ascontiguousarray(cent, dtype=np.int8)
    out = np.empty(P, dtype=np.int32)
    assert lib.oracle_probe(_ptr(q), _ptr(cent), cent.shape[0], cent.shape[1], P, _ptr(out)) == 0
    return out


def search(items, sigs, offsets, centroids, queries, masks, nprobe, k, b0=0, b1=None,
           nthreads=1, lib=None, row_ids=None):
    """Search queries [b0, b1). Returns (ids int64 [nb,k], scores int32 [nb,k],
    probe int32 [nb,P], eligible int64 [nb]). row_ids (int64 [n], optional)
    gives the item id of each row; by default it is the row index."""
    lib = lib or load()
    items = np.ascontiguousarray(items, dtype=np.int8)
    sigs = np.ascontiguousarray(sigs).view(np.uint64)
    if sigs.ndim == 1:
        sigs = sigs.reshape(-1, 1)
    offsets = np.ascontiguousarray(offsets, dtype=np.int64)
    centroids = np.ascontiguousarray(centroids, dtype=np.int8)
    queries = np.ascontiguousarray(queries, dtype=np.int8)
    masks = np.ascontiguousarray(masks).view(np.uint64)
    if masks.ndim == 1:
        masks = masks.reshape(-1, 1)
    n, d = items.shape
    W = sigs.shape[1]
    nlist = centroids.shape[0]
    B = queries.shape[0]
    b1 = B if b1 is None else b1
    nb = b1 - b0
    ids = np.empty((nb, k), dtype=np.int64)
    scores = np.empty((nb, k), dtype=np.int32)
    probe_out = np.empty((nb, nprobe), dtype=np.int32)
    elig = np.empty(nb, dtype=np.int64)
    if row_ids is None:
        rc = lib.oracle_search(_ptr(items), _ptr(sigs), _ptr(offsets), _ptr(centroids), n, d, nlist,
                               W, _ptr(queries), _ptr(masks), b0, b1, nprobe, k, _ptr(ids),
                               _ptr(scores), _ptr(probe_out), _ptr(elig), nthreads)
    else:
        row_ids = np.ascontiguousarray(row_ids, dtype=np.int64)
        assert row_ids.shape == (n,)
        rc = lib.oracle_search_ids(_ptr(items), _ptr(sigs), _ptr(offsets), _ptr(row_ids), _ptr(centroids), n,
                                   d, nlist, W, _ptr(queries), _ptr(masks), b0, b1, nprobe, k, _ptr(ids),
                                   _ptr(scores), _ptr(probe_out), _ptr(elig), nthreads)
    assert rc == 0, "oracle allocation failed"
    return ids, scores, probe_out, elig


def search_or(items, sigs, offsets, centroids, queries, mask_sets, nprobe, k, b0=0, b1=None,
              nthreads=1, lib=None, row_ids=None):
    """Search with A alternative masks per query, mask_sets uint64 [B, A, W]:
    an item is eligible when it passes any of its query's masks. Same outputs
    as search()."""
    lib = lib or load()
    items = np.ascontiguousarray(items, dtype=np.int8)
    sigs = np.ascontiguousarray(sigs).view(np.uint64)
    if sigs.ndim == 1:
        sigs = sigs.reshape(-1, 1)
    offsets = np.ascontiguousarray(offsets, dtype=np.int64)
    centroids = np.ascontiguousarray(centroids, dtype=np.int8)
    queries = np.ascontiguousarray(queries, dtype=np.int8)
    mask_sets = np.ascontiguousarray(mask_sets).view(np.uint64)
    n, d = items.shape
    W = sigs.shape[1]
    B = queries.shape[0]
    assert mask_sets.ndim == 3 and mask_sets.shape[0] == B and mask_sets.shape[2] == W
    A = mask_sets.shape[1]
    nlist = centroids.shape[0]
    b1 = B if b1 is None else b1
    nb = b1 - b0
    ids = np.empty((nb, k), dtype=np.int64)
    scores = np.empty((nb, k), dtype=np.int32)
    probe_out = np.empty((nb, nprobe), dtype=np.int32)
    elig = np.empty(nb, dtype=np.int64)
    rid = None if row_ids is None else np.ascontiguousarray(row_ids, dtype=np.int64)
    rc = lib.oracle_search_or(_ptr(items), _ptr(sigs), _ptr(offsets), None if rid is None else _ptr(rid),
                              _ptr(centroids), n, d, nlist, W, _ptr(queries), _ptr(mask_sets), A, b0, b1,
                              nprobe, k, _ptr(ids), _ptr(scores), _ptr(probe_out), _ptr(elig), nthreads)
    assert rc == 0, "oracle allocation failed"
    return ids, scores, probe_out, elig


def max_threads(lib=None) -> int:
    lib = lib or load()
    return int(lib.oracle_max_threads())
