"""Seeded synthetic inputs for the Bloom-filtered int8 IVF top-k search.

This module only draws inputs. It holds none of the search arithmetic (no probe,
no filter test, no top-k): the CUDA library and the CPU oracle both consume the
arrays it returns, and neither is imported here.

Recipe (stated once, used for every workload):

* Centroids: nlist fp32 vectors ~ N(0, 1). Int8 centroids = round-half-even(40 v),
  clipped to [-127, 127].
* Items: pick a centroid (uniform, or p(j) ~ (j+1)^-s for the Zipf-skewed
  workload), add N(0, 0.5^2) noise per dimension, quantise the same way.
  The flat bandwidth workload instead draws uniform int8 in [-127, 127].
* List of an item: argmax over the int8 centroids of the int32 inner product,
  ties to the lower list id. Items are then stable-sorted by list (ties keep
  generation order), so the row index is the item id and each list is a
  contiguous row range given by CSR offsets.
* Attributes: language (50 values, Zipf s=1.1), country (200 values, Zipf 1.1),
  6 policy flags each true with p=0.9. Zipf here is finite, p(v) ~ (v+1)^-s,
  v = 0 the most frequent.
* Bloom signature of S bits (64 or 128, stored as S/64 little-endian uint64
  words): every (field, value) pair present on the item -- language is field 0,
  country field 1, flag f field 2+f with value 1, only true flags inserted -- is
  hashed with h = splitmix64(seed ^ (field << 32) ^ value) and sets `bits` bits:
  bit t = (h >> (t * log2 S)) & (S - 1).
* Queries are drawn like items. A query mask is the OR of the signature bits of
  the (field, value) pairs it requires. Mask mode "head" requires the most
  frequent language / country (value 0) plus a uniformly random subset of the
  flags of the stated size; mode "item" copies language / country from a random
  item (flags as in "head").

Randomness comes from a torch.Generator seeded per workload on the requested
device, drawn in fixed 2^22-item chunks, so a (workload, seed, device) triple
always gives the same arrays.

The pages describe these structures only in words: item signatures checked with
simple bit operations (SilverTorch: Index as Model, section on redesigning each
stage as a pure PyTorch module -- Bloom index filter paragraph), int8 item
embeddings (same section, fused Int8 ANN paragraph) and probing the most
promising clusters (same page, section on how the components worked before).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

MASK64 = (1 << 64) - 1
CHUNK = 1 << 22          # items drawn per RNG chunk (part of the recipe)
N_LANG, N_COUNTRY, N_FLAGS = 50, 200, 6
FIELD_LANG, FIELD_COUNTRY, FIELD_FLAG0 = 0, 1, 2


# ----------------------------------------------------------------------------
# splitmix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
# generators", OOPSLA 2014): one step = add the golden-ratio increment, then the
# 64-bit finaliser (two xor-shift-multiply rounds and a final xor-shift).
# ----------------------------------------------------------------------------
_GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB


def splitmix64(x: int) -> int:
    z = (x + _GAMMA) & MASK64
    z = ((z ^ (z >> 30)) * _M1) & MASK64
    z = ((z ^ (z >> 27)) * _M2) & MASK64
    return z ^ (z >> 31)


def bloom_bits(seed: int, field: int, value: int, sig_bits: int, nbits: int) -> list[int]:
    """Bit positions set by one (field, value) pair."""
    assert sig_bits in (64, 128)
    chunk = 6 if sig_bits == 64 else 7
    h = splitmix64((seed ^ (field << 32) ^ value) & MASK64)
    return [(h >> (t * chunk)) & (sig_bits - 1) for t in range(nbits)]


def bloom_words(seed: int, field: int, value: int, sig_bits: int, nbits: int) -> list[int]:
    """The (field, value) pattern as sig_bits/64 unsigned 64-bit words."""
    words = [0] * (sig_bits // 64)
    for b in bloom_bits(seed, field, value, sig_bits, nbits):
        words[b >> 6] |= 1 << (b & 63)
    return words


def _to_i64(u: int) -> int:
    return u - (1 << 64) if u >= (1 << 63) else u


def _table(seed: int, field: int, nvalues: int, sig_bits: int, nbits: int) -> torch.Tensor:
    rows = [[_to_i64(w) for w in bloom_words(seed, field, v, sig_bits, nbits)] for v in range(nvalues)]
    return torch.tensor(rows, dtype=torch.int64)


# ----------------------------------------------------------------------------
# Workload descriptions (named by what they are, with their sizes)
# ----------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    n: int                      # items
    d: int                      # dimensions (int8)
    nlist: int                  # IVF lists (1 = flat)
    sig_bits: int               # 64 or 128
    hash_bits: int              # bits set per (field, value)
    B: int                      # queries
    nprobe: int
    k: int
    centroid_zipf: Optional[float] = None   # None = uniform centroid choice
    uniform_items: bool = False             # flat uniform int8 items (no mixture)
    mask_lang: bool = True
    mask_country: bool = True
    mask_flags: int = 3
    seed: int = 1000
    bloom_seed: int = 0x51F7E2C0FFEE1234

    @property
    def W(self) -> int:
        return self.sig_bits // 64

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # 100k items, d=64, 256 lists, 64-bit signatures with 2 bits per pair.
    "tiny_ivf": Workload("tiny_ivf", 100_000, 64, 256, 64, 2, 8, 16, 100,
                         mask_flags=3, seed=1000, bloom_seed=0x51F7E2C0FFEE0000),
    # 1M items, d=128, 1024 lists, 128-bit signatures with 3 bits per pair.
    "mid_ivf": Workload("mid_ivf", 1_000_000, 128, 1024, 128, 3, 32, 32, 512,
                        mask_flags=4, seed=1001, bloom_seed=0x51F7E2C0FFEE0001),
    # 10M uniform int8 items, d=128, flat, one query, language + 2 flags.
    "flat_10m": Workload("flat_10m", 10_000_000, 128, 1, 128, 3, 1, 1, 2048,
                         uniform_items=True, mask_country=False, mask_flags=2,
                         seed=1002, bloom_seed=0x51F7E2C0FFEE0002),
    # 80M items, d=64, 16384 Zipf(0.8)-skewed lists, B=64, nprobe=64, k=2048.
    "ivf_80m": Workload("ivf_80m", 80_000_000, 64, 16384, 128, 3, 64, 64, 2048,
                        centroid_zipf=0.8, mask_flags=4, seed=1003,
                        bloom_seed=0x51F7E2C0FFEE0003),
    # 10M items, d=128, 4096 lists, 2-flag masks (~80% selectivity), B up to 1024.
    "sweep_10m": Workload("sweep_10m", 10_000_000, 128, 4096, 128, 3, 1024, 64, 1024,
                          mask_lang=False, mask_country=False, mask_flags=2,
                          seed=1004, bloom_seed=0x51F7E2C0FFEE0004),
}
# Same items as tiny_ivf searched flat: one list holding every item, a zero
# centroid, nprobe = 1 (equal to IVF with nprobe = nlist).
SWEEP_BATCHES = (1, 8, 64, 256, 1024)


@dataclasses.dataclass
class Data:
    """Arrays of one workload. Tensors live on `device`; sigs and masks are
    int64 tensors whose bit patterns are the uint64 words."""
    wl: Workload
    items: torch.Tensor        # int8  [n, d]   rows grouped by list
    sigs: torch.Tensor         # int64 [n, W]
    offsets: torch.Tensor      # int64 [nlist + 1]
    centroids: torch.Tensor    # int8  [nlist, d]
    queries: torch.Tensor      # int8  [B, d]
    masks: torch.Tensor        # int64 [B, W]
    # exact attributes (for the no-false-negative invariant)
    lang: torch.Tensor         # int16 [n]
    country: torch.Tensor      # int16 [n]
    flags: torch.Tensor        # bool  [n, 6]
    q_lang: torch.Tensor       # int16 [B]  (-1 = not required)
    q_country: torch.Tensor    # int16 [B]
    q_flags: torch.Tensor      # bool  [B, 6] required flags

    def flat(self) -> "Data":
        """The same items searched flat (one list, zero centroid)."""
        wl = self.wl.with_(name=self.wl.name + "_flat", nlist=1, nprobe=1)
        off = torch.tensor([0, self.wl.n], dtype=torch.int64, device=self.items.device)
        cen = torch.zeros((1, self.wl.d), dtype=torch.int8, device=self.items.device)
        return dataclasses.replace(self, wl=wl, offsets=off, centroids=cen)

    def head(self, B: int) -> "Data":
        """The first B queries."""
        return dataclasses.replace(
            self, wl=self.wl.with_(B=B), queries=self.queries[:B].contiguous(),
            masks=self.masks[:B].contiguous(), q_lang=self.q_lang[:B],
            q_country=self.q_country[:B], q_flags=self.q_flags[:B])

    def to(self, device) -> "Data":
        kw = {f.name: getattr(self, f.name).to(device) for f in dataclasses.fields(self)
              if isinstance(getattr(self, f.name), torch.Tensor)}
        return dataclasses.replace(self, **kw)


def _zipf_cdf(nvalues: int, s: float, device) -> torch.Tensor:
    p = (torch.arange(1, nvalues + 1, dtype=torch.float64) ** (-s))
    c = torch.cumsum(p / p.sum(), 0)
    c[-1] = 1.0
    return c.to(device)


def _draw_categorical(cdf: torch.Tensor, n: int, g: torch.Generator, device) -> torch.Tensor:
    u = torch.rand(n, generator=g, device=device, dtype=torch.float64)
    return torch.searchsorted(cdf, u, right=True).clamp_(max=cdf.numel() - 1)


def _quantise(v: torch.Tensor) -> torch.Tensor:
    return torch.round(v * 40.0).clamp_(-127, 127).to(torch.int8)


def _assign_lists(items_q: torch.Tensor, cent_q: torch.Tensor) -> torch.Tensor:
    """argmax_c <x, cent_c> in int32, ties to the lower c.

    Done as an fp32 GEMM, which is exact here: every partial sum is an integer
    of magnitude <= d * 127 * 127 < 2^24 for d <= 128 (checked below), so any
    summation order gives the int32 value. TF32 is switched off.
    """
    d = items_q.shape[1]
    assert d * 127 * 127 < (1 << 24), "fp32 assignment is exact only for d <= 1040"
    old = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        cf = cent_q.float().t().contiguous()
        out = torch.empty(items_q.shape[0], dtype=torch.int64, device=items_q.device)
        step = 1 << 16
        for s in range(0, items_q.shape[0], step):
            sc = items_q[s:s + step].float() @ cf
            # torch.max returns the first index among equal maxima
            out[s:s + step] = torch.max(sc, dim=1).indices
        return out
    finally:
        torch.backends.cuda.matmul.allow_tf32 = old


def generate(wl: Workload, device="cpu", mask_mode: str = "head", seed: Optional[int] = None) -> Data:
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(wl.seed if seed is None else seed)
    n, d, nlist, W = wl.n, wl.d, wl.nlist, wl.W

    # --- centroids and items --------------------------------------------------
    if wl.uniform_items:
        assert nlist == 1
        cent_f = None
        cent_q = torch.zeros((1, d), dtype=torch.int8, device=device)
    else:
        cent_f = torch.randn((nlist, d), generator=g, device=device, dtype=torch.float32)
        cent_q = _quantise(cent_f)
    cdf_c = _zipf_cdf(nlist, wl.centroid_zipf, device) if wl.centroid_zipf else None

    def draw_vectors(m: int) -> torch.Tensor:
        out = torch.empty((m, d), dtype=torch.int8, device=device)
        for s in range(0, m, CHUNK):
            e = min(m, s + CHUNK)
            if wl.uniform_items:
                out[s:e] = torch.randint(-127, 128, (e - s, d), generator=g, device=device,
                                         dtype=torch.int16).to(torch.int8)
                continue
            if cdf_c is None:
                ch = torch.randint(0, nlist, (e - s,), generator=g, device=device)
            else:
                ch = _draw_categorical(cdf_c, e - s, g, device)
            noise = torch.randn((e - s, d), generator=g, device=device, dtype=torch.float32)
            out[s:e] = _quantise(cent_f[ch] + 0.5 * noise)
        return out

    items_q = draw_vectors(n)

    # --- attributes ----------------------------------------------------------
    cdf_l = _zipf_cdf(N_LANG, 1.1, device)
    cdf_k = _zipf_cdf(N_COUNTRY, 1.1, device)
    lang = torch.empty(n, dtype=torch.int16, device=device)
    country = torch.empty(n, dtype=torch.int16, device=device)
    flags = torch.empty((n, N_FLAGS), dtype=torch.bool, device=device)
    for s in range(0, n, CHUNK):
        e = min(n, s + CHUNK)
        lang[s:e] = _draw_categorical(cdf_l, e - s, g, device).to(torch.int16)
        country[s:e] = _draw_categorical(cdf_k, e - s, g, device).to(torch.int16)
        flags[s:e] = torch.rand((e - s, N_FLAGS), generator=g, device=device) < 0.9

    # --- list assignment and list-major order --------------------------------
    if nlist > 1:
        lists = _assign_lists(items_q, cent_q)
        order = torch.sort(lists, stable=True).indices
        items_q = items_q[order]
        lang, country, flags = lang[order], country[order], flags[order]
        counts = torch.bincount(lists, minlength=nlist)
        del order, lists
    else:
        counts = torch.tensor([n], dtype=torch.int64, device=device)
    offsets = torch.zeros(nlist + 1, dtype=torch.int64, device=device)
    offsets[1:] = torch.cumsum(counts, 0)

    # --- signatures ------------------------------------------------------------
    tl = _table(wl.bloom_seed, FIELD_LANG, N_LANG, wl.sig_bits, wl.hash_bits).to(device)
    tk = _table(wl.bloom_seed, FIELD_COUNTRY, N_COUNTRY, wl.sig_bits, wl.hash_bits).to(device)
    tf = torch.cat([_table(wl.bloom_seed, FIELD_FLAG0 + f, 2, wl.sig_bits, wl.hash_bits)[1:]
                    for f in range(N_FLAGS)]).to(device)            # [6, W], value 1
    sigs = torch.empty((n, W), dtype=torch.int64, device=device)
    for s in range(0, n, CHUNK):
        e = min(n, s + CHUNK)
        sg = tl[lang[s:e].long()] | tk[country[s:e].long()]
        for f in range(N_FLAGS):
            sg |= torch.where(flags[s:e, f:f + 1], tf[f:f + 1], torch.zeros_like(tf[f:f + 1]))
        sigs[s:e] = sg

    # --- queries and masks -----------------------------------------------------
    B = wl.B
    queries = draw_vectors(B)
    if mask_mode == "head":
        q_lang = torch.zeros(B, dtype=torch.int16, device=device)
        q_country = torch.zeros(B, dtype=torch.int16, device=device)
    elif mask_mode == "item":
        src = torch.randint(0, n, (B,), generator=g, device=device)
        q_lang, q_country = lang[src].clone(), country[src].clone()
    else:
        raise ValueError(mask_mode)
    if not wl.mask_lang:
        q_lang.fill_(-1)
    if not wl.mask_country:
        q_country.fill_(-1)
    perm = torch.argsort(torch.rand((B, N_FLAGS), generator=g, device=device), dim=1)
    q_flags = torch.zeros((B, N_FLAGS), dtype=torch.bool, device=device)
    if wl.mask_flags:
        q_flags.scatter_(1, perm[:, :wl.mask_flags], True)
    masks = torch.zeros((B, W), dtype=torch.int64, device=device)
    masks |= torch.where((q_lang >= 0)[:, None], tl[q_lang.clamp(min=0).long()], 0)
    masks |= torch.where((q_country >= 0)[:, None], tk[q_country.clamp(min=0).long()], 0)
    for f in range(N_FLAGS):
        masks |= torch.where(q_flags[:, f:f + 1], tf[f:f + 1], 0)

    return Data(wl, items_q.contiguous(), sigs, offsets, cent_q.contiguous(), queries, masks,
                lang, country, flags, q_lang, q_country, q_flags)


def small(n=2000, d=32, nlist=16, sig_bits=64, hash_bits=2, B=8, nprobe=4, k=50,
          seed=7, mask_flags=2, mask_lang=True, mask_country=False, centroid_zipf=None,
          uniform_items=False, mask_mode="head", device="cpu") -> Data:
    """A small workload of the same recipe, for tests."""
    wl = Workload("small", n, d, nlist, sig_bits, hash_bits, B, nprobe, k,
                  centroid_zipf=centroid_zipf, uniform_items=uniform_items,
                  mask_lang=mask_lang, mask_country=mask_country, mask_flags=mask_flags,
                  seed=seed, bloom_seed=0xB10057 + seed)
    return generate(wl, device=device, mask_mode=mask_mode)


def to_numpy(data: Data) -> dict:
    """Host numpy views with the C types (uint64 words for sigs and masks)."""
    f = lambda t: t.detach().cpu().contiguous().numpy()
    return dict(items=f(data.items), sigs=f(data.sigs).view(np.uint64),
                offsets=f(data.offsets), centroids=f(data.centroids),
                queries=f(data.queries), masks=f(data.masks).view(np.uint64))
