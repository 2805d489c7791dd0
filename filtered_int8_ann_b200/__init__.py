"""Python binding of libst.so, the Bloom-filtered int8 IVF top-k search library.

Argument marshalling only: every step of a search runs in the library's CUDA
kernels. The functions keep the C names of include/st.h; torch tensors supply
device memory and torch streams supply the CUDA stream. Loading fails loudly
when libst.so has not been built (python -m filtered_int8_ann_b200.build):
there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libst.so")

(ST_OK, ST_ERR_INVALID_ARG, ST_ERR_UNSUPPORTED, ST_ERR_OOM, ST_ERR_CUDA, ST_ERR_DEVICE,
 ST_ERR_SCRATCH_LIMIT) = range(7)
ST_PROBE_NOALLOC_SCRATCH_BYTES = 16 << 20
(ST_OPT_CANDIDATE_BYTES, ST_OPT_CANDIDATE_CAPACITY, ST_OPT_ID_OFFSET, ST_OPT_INSERT_RESERVE,
 ST_OPT_DENSE_MIN_QUERIES) = 1, 2, 3, 4, 5
ST_INSERT_CHUNK = 512
ST_MERGE_MAX_KEYS = 16384
ST_MAX_D, ST_MAX_K, ST_MAX_NPROBE, ST_SMALL_K, ST_MAX_B = 512, 262144, 4096, 4096, 32768
ST_MAX_OR = 7

# Every symbol include/st.h declares.
EXPORTS = ("st_index_create", "st_search", "st_search_ex", "st_search_host", "st_search_host_async",
           "st_index_check",
           "st_index_set_option", "st_probe_noalloc", "st_merge_topk", "st_merge_check", "st_index_update",
           "st_index_delete", "st_merge_topk_union", "st_index_insert", "st_index_destroy", "st_status_string")


class StError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


class _Extras(ctypes.Structure):
    _fields_ = [("eligible", ctypes.c_void_p), ("probe", ctypes.c_void_p),
                ("stage_events", ctypes.c_void_p * 5), ("exclude_masks", ctypes.c_void_p),
                ("candidates", ctypes.c_void_p), ("or_masks", ctypes.c_void_p), ("n_or", ctypes.c_int32)]


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with `python -m filtered_int8_ann_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    L.st_index_create.argtypes = [P, P, P, P, i64, i32, i32, i32, P, ctypes.POINTER(P)]
    L.st_search.argtypes = [P, P, P, i32, i32, i32, P, P, P]
    L.st_search_ex.argtypes = [P, P, P, i32, i32, i32, P, P, ctypes.POINTER(_Extras), P]
    L.st_search_host.argtypes = [P, P, P, i32, i32, i32, P, P, P]
    L.st_search_host_async.argtypes = [P, P, P, i32, i32, i32, P, P, P]
    L.st_index_check.argtypes = [P, P]
    L.st_index_set_option.argtypes = [P, ctypes.c_int, i64]
    L.st_probe_noalloc.argtypes = [P, P, i32, i32, P, P]
    L.st_merge_topk.argtypes = [P, P, i32, i32, i32, P, P, P]
    L.st_merge_check.argtypes = [P]
    L.st_index_update.argtypes = [P, P, P, P, i64, P]
    L.st_index_delete.argtypes = [P, P, i64, P]
    L.st_merge_topk_union.argtypes = [P, P, i32, i32, i32, P, P, P]
    L.st_index_insert.argtypes = [P, P, P, P, i64, P, P]
    for f in ("st_index_create", "st_search", "st_search_ex", "st_search_host", "st_search_host_async",
              "st_index_check",
              "st_index_set_option", "st_probe_noalloc", "st_merge_topk", "st_merge_check", "st_index_update",
              "st_index_delete", "st_merge_topk_union", "st_index_insert"):
        getattr(L, f).restype = ctypes.c_int
    L.st_index_destroy.argtypes = [P]
    L.st_index_destroy.restype = None
    L.st_status_string.argtypes = [ctypes.c_int]
    L.st_status_string.restype = ctypes.c_char_p
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().st_status_string(status).decode()


def _check(status: int, what: str):
    if status != ST_OK:
        raise StError(status, what)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        return t.data_ptr()
    return int(t)


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _as_words(t: torch.Tensor) -> torch.Tensor:
    """Signatures / masks as int64 words [rows, W] (bit patterns of uint64)."""
    if t.dtype == torch.uint64:
        t = t.view(torch.int64)
    assert t.dtype == torch.int64, "signatures and masks are 64-bit words"
    return t if t.dim() == 2 else t.reshape(-1, 1)


def st_index_create(items: torch.Tensor, sigs: torch.Tensor, list_offsets: torch.Tensor,
                    centroids: torch.Tensor, stream=None) -> int:
    """Build an index from int8 items [n,d], signature words [n,W], int64 offsets
    [nlist+1] and int8 centroids [nlist,d]; returns the opaque handle."""
    sigs = _as_words(sigs).contiguous()
    items, list_offsets, centroids = items.contiguous(), list_offsets.contiguous(), centroids.contiguous()
    assert items.dtype == torch.int8 and centroids.dtype == torch.int8 and list_offsets.dtype == torch.int64
    n, d = items.shape
    h = ctypes.c_void_p()
    _check(lib().st_index_create(_ptr(items), _ptr(sigs), _ptr(list_offsets), _ptr(centroids), n, d,
                                 centroids.shape[0], sigs.shape[1], _stream(stream), ctypes.byref(h)),
           "st_index_create")
    return h.value


def st_search(index: int, queries: torch.Tensor, qmasks: torch.Tensor, nprobe: int, k: int,
              out_ids: Optional[torch.Tensor] = None, out_scores: Optional[torch.Tensor] = None,
              stream=None, eligible: Optional[torch.Tensor] = None,
              probe: Optional[torch.Tensor] = None, stage_events=None,
              exclude: Optional[torch.Tensor] = None, candidates: Optional[torch.Tensor] = None,
              or_masks: Optional[torch.Tensor] = None):
    """Asynchronous search of device-resident queries; returns (ids int64 [B,k],
    scores int32 [B,k]). `eligible` [B] int64 and `probe` [B,nprobe] int32 are
    optional extra outputs, as is `candidates` [B] int64 (keys the scan wrote
    for each query's final top-k); `stage_events` is a list of up to five recorded
    torch.cuda.Event objects marking the stage boundaries; `exclude` [B,W]
    holds per-query exclude masks; `or_masks` [B,A,W] alternative masks (an
    item passing qmasks[b] or any of or_masks[b] is eligible) (st_search_ex)."""
    qmasks = _as_words(qmasks)
    B = queries.shape[0]
    dev = queries.device
    if out_ids is None:
        out_ids = torch.empty((B, k), dtype=torch.int64, device=dev)
    if out_scores is None:
        out_scores = torch.empty((B, k), dtype=torch.int32, device=dev)
    if exclude is not None:
        exclude = _as_words(exclude)
    n_or = 0
    if or_masks is not None:
        if or_masks.dtype == torch.uint64:
            or_masks = or_masks.view(torch.int64)
        if or_masks.dtype != torch.int64:
            raise ValueError("or_masks are 64-bit words")
        if or_masks.dim() == 2:  # [B, A] of one-word masks
            or_masks = or_masks.unsqueeze(-1)
        or_masks = or_masks.contiguous()
        if or_masks.dim() != 3 or or_masks.shape[0] != B or or_masks.shape[2] != qmasks.shape[-1]:
            raise ValueError("or_masks must be [B, A, W] with the masks' W")
        n_or = int(or_masks.shape[1])
    if eligible is None and probe is None and not stage_events and exclude is None and candidates is None \
            and n_or == 0:
        st = lib().st_search(index, _ptr(queries), _ptr(qmasks), B, nprobe, k, _ptr(out_ids),
                             _ptr(out_scores), _stream(stream))
        _check(st, "st_search")
    else:
        ex = _Extras(_ptr(eligible), _ptr(probe))
        ex.exclude_masks = _ptr(exclude)
        ex.candidates = _ptr(candidates)
        ex.or_masks = _ptr(or_masks) if n_or else None
        ex.n_or = n_or
        for i, ev in enumerate(stage_events or ()):
            ex.stage_events[i] = ev.cuda_event if ev is not None else None
        st = lib().st_search_ex(index, _ptr(queries), _ptr(qmasks), B, nprobe, k, _ptr(out_ids),
                                _ptr(out_scores), ctypes.byref(ex), _stream(stream))
        _check(st, "st_search_ex")
    return out_ids, out_scores


def st_search_host(index: int, queries: torch.Tensor, qmasks: torch.Tensor, nprobe: int, k: int,
                   out_ids: Optional[torch.Tensor] = None, out_scores: Optional[torch.Tensor] = None,
                   stream=None):
    """Search host-resident (ideally pinned) queries; results land in host
    tensors and are ready when the call returns."""
    qmasks = _as_words(qmasks)
    assert queries.device.type == "cpu" and qmasks.device.type == "cpu"
    B = queries.shape[0]
    if out_ids is None:
        out_ids = torch.empty((B, k), dtype=torch.int64)
    if out_scores is None:
        out_scores = torch.empty((B, k), dtype=torch.int32)
    _check(lib().st_search_host(index, _ptr(queries), _ptr(qmasks), B, nprobe, k, _ptr(out_ids),
                                _ptr(out_scores), _stream(stream)), "st_search_host")
    return out_ids, out_scores


def st_search_host_async(index: int, queries: torch.Tensor, qmasks: torch.Tensor, nprobe: int, k: int,
                         out_ids: torch.Tensor, out_scores: torch.Tensor, stream=None):
    """Enqueue a search on page-locked host tensors and return at once; the
    outputs are complete when the stream has finished it."""
    qmasks = _as_words(qmasks)
    B = queries.shape[0]
    _check(lib().st_search_host_async(index, _ptr(queries), _ptr(qmasks), B, nprobe, k, _ptr(out_ids),
                                      _ptr(out_scores), _stream(stream)), "st_search_host_async")
    return out_ids, out_scores


def st_index_check(index: int, stream=None) -> int:
    """Synchronize and return the device-side status (ST_OK or ST_ERR_DEVICE)."""
    return lib().st_index_check(index, _stream(stream))


def st_index_set_option(index: int, option: int, value: int):
    _check(lib().st_index_set_option(index, option, value), "st_index_set_option")


def st_probe_noalloc(index: int, queries: torch.Tensor, nprobe: int, out_probe: torch.Tensor,
                     stream=None) -> torch.Tensor:
    """Probe-only call that allocates no device memory (its scratch is a fixed
    array inside the library); `out_probe` is the caller's int32 [B, nprobe]
    device tensor. Calls on one device share that array: keep them ordered."""
    B = queries.shape[0]
    _check(lib().st_probe_noalloc(index, _ptr(queries), B, nprobe, _ptr(out_probe), _stream(stream)),
           "st_probe_noalloc")
    return out_probe


def st_merge_topk(ids: torch.Tensor, scores: torch.Tensor, out_ids: Optional[torch.Tensor] = None,
                  out_scores: Optional[torch.Tensor] = None, stream=None):
    """Exact merge of G document shards' results: ids int64 [G, B, k] and
    scores int32 [G, B, k] (device, contiguous) -> (ids [B, k], scores [B, k])."""
    G, B, k = ids.shape
    if out_ids is None:
        out_ids = torch.empty((B, k), dtype=torch.int64, device=ids.device)
    if out_scores is None:
        out_scores = torch.empty((B, k), dtype=torch.int32, device=ids.device)
    _check(lib().st_merge_topk(_ptr(ids), _ptr(scores), G, B, k, _ptr(out_ids), _ptr(out_scores),
                               _stream(stream)), "st_merge_topk")
    return out_ids, out_scores


def st_merge_topk_union(ids: torch.Tensor, scores: torch.Tensor, out_ids: Optional[torch.Tensor] = None,
                        out_scores: Optional[torch.Tensor] = None, stream=None):
    """Exact top-k of the union of G result lists [G, B, k] that may share items."""
    G, B, k = ids.shape
    if out_ids is None:
        out_ids = torch.empty((B, k), dtype=torch.int64, device=ids.device)
    if out_scores is None:
        out_scores = torch.empty((B, k), dtype=torch.int32, device=ids.device)
    _check(lib().st_merge_topk_union(_ptr(ids), _ptr(scores), G, B, k, _ptr(out_ids), _ptr(out_scores),
                                     _stream(stream)), "st_merge_topk_union")
    return out_ids, out_scores


def st_merge_check(stream=None) -> int:
    """Synchronize and return the merge's device-side status (ST_OK or ST_ERR_DEVICE)."""
    return lib().st_merge_check(_stream(stream))


def st_index_destroy(index: Optional[int]):
    if index:
        lib().st_index_destroy(index)


class Index:
    """Owning wrapper: builds on construction, frees on close()/GC."""

    def __init__(self, items, sigs, list_offsets, centroids, stream=None):
        self.handle = st_index_create(items, sigs, list_offsets, centroids, stream)
        self.d = items.shape[1]
        self.nlist = centroids.shape[0]

    def search(self, queries, qmasks, nprobe, k, **kw):
        return st_search(self.handle, queries, qmasks, nprobe, k, **kw)

    def search_host(self, queries, qmasks, nprobe, k, **kw):
        return st_search_host(self.handle, queries, qmasks, nprobe, k, **kw)

    def search_host_async(self, queries, qmasks, nprobe, k, out_ids, out_scores, stream=None):
        return st_search_host_async(self.handle, queries, qmasks, nprobe, k, out_ids, out_scores, stream)

    def update(self, ids, items=None, sigs=None, stream=None):
        """Replace the rows and/or signatures of existing items in place (device tensors)."""
        if sigs is not None:
            sigs = _as_words(sigs)
        _check(lib().st_index_update(self.handle, _ptr(ids), _ptr(items), _ptr(sigs), int(ids.numel()),
                                     _stream(stream)), "st_index_update")

    def search_any(self, queries, mask_sets, nprobe, k, stream=None, **kw):
        """OR of several masks per query: an item is eligible if any of the masks
        passes. mask_sets [M, B, W] (M alternatives, M <= ST_MAX_OR + 1): one
        search whose scan tests every alternative (st_search_extras.or_masks)."""
        M = mask_sets.shape[0]
        alt = mask_sets[1:].permute(1, 0, 2).contiguous() if M > 1 else None
        return self.search(queries, mask_sets[0].contiguous(), nprobe, k, stream=stream, or_masks=alt, **kw)

    def search_any_merged(self, queries, mask_sets, nprobe, k, stream=None, **kw):
        """search_any as one search per alternative followed by the exact union
        merge of their results (st_merge_topk_union; k <= 4096, M * k <=
        ST_MERGE_MAX_KEYS): the same result, for checking the fused scan."""
        M, B = mask_sets.shape[0], queries.shape[0]
        ids = torch.empty((M, B, k), dtype=torch.int64, device=queries.device)
        sc = torch.empty((M, B, k), dtype=torch.int32, device=queries.device)
        for j in range(M):
            self.search(queries, mask_sets[j].contiguous(), nprobe, k, out_ids=ids[j], out_scores=sc[j],
                        stream=stream, **kw)
        return st_merge_topk_union(ids, sc, stream=stream)

    def insert(self, lists, items, sigs, stream=None):
        """Insert new items: lists (host, one list id per item), items int8 [m, d]
        and sigs [m, W] (device tensors). Returns the ids given to them (numpy
        int64 [m]); waits for the stream."""
        lists = np.ascontiguousarray(np.asarray(lists, dtype=np.int32).reshape(-1))
        m = lists.shape[0]
        out = np.empty(m, dtype=np.int64)
        if m:
            items = items.contiguous()
            sigs = _as_words(sigs).contiguous()
            if items.shape[0] != m or sigs.shape[0] != m:
                raise ValueError("lists, items and sigs must have the same number of rows")
        _check(lib().st_index_insert(self.handle, lists.ctypes.data_as(ctypes.c_void_p) if m else None,
                                     _ptr(items) if m else None, _ptr(sigs) if m else None, m,
                                     out.ctypes.data_as(ctypes.c_void_p) if m else None, _stream(stream)),
               "st_index_insert")
        return out

    def delete(self, ids, stream=None):
        """Delete items in place (device int64 item ids)."""
        _check(lib().st_index_delete(self.handle, _ptr(ids), int(ids.numel()), _stream(stream)), "st_index_delete")

    def probe_noalloc(self, queries, nprobe, out_probe, stream=None):
        return st_probe_noalloc(self.handle, queries, nprobe, out_probe, stream)

    def check(self, stream=None) -> int:
        return st_index_check(self.handle, stream)

    @classmethod
    def shard(cls, items, sigs, list_offsets, centroids, shards, g, stream=None):
        """Index of document shard g of `shards` (rows split by contiguous ranges,
        global ids returned)."""
        from .shard import shard_arrays
        it, sg, off, base = shard_arrays(items, sigs, list_offsets, shards, g)
        idx = cls(it.contiguous(), sg.contiguous(), off, centroids, stream)
        idx.set_option(ST_OPT_ID_OFFSET, base)
        return idx

    def set_option(self, option, value):
        st_index_set_option(self.handle, option, value)

    def close(self):
        if getattr(self, "handle", None):
            st_index_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
