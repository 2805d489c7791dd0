#!/usr/bin/env python
"""Benchmark of the Bloom-filtered int8 IVF top-k search on B200.

One step = one st_search call (probe -> plan -> scan -> final top-k) over one
batch of queries, inputs resident in HBM. Default workload: 80M items, d=64,
16384 Zipf(0.8)-skewed lists, 128-bit signatures, B=64 queries, nprobe=64,
k=2048. The timed steps cycle through a pool of distinct query batches; the
index (6.4 GB) is far larger than L2.

Besides the timed headline it reports, on the same GPU in the same run:
  * the same search with the L2 flushed before every step (median of R);
  * the roofline of the dominant kernel and of the whole step against HBM
    bandwidth, the int8 tensor peak and the measured dp4a issue rate;
  * recall@k of the IVF search against the flat filtered search;
  * every other workload (tiny, mid, flat 10M, the 10M batch sweep at each B)
    with the same figures (`per_config`);
  * large k and streamed-update costs on the headline index.

Prints one JSON line (rank 0). `--impl reference` times the CPU oracle instead
(the reference arm; host cores only).
"""
import argparse
import ctypes
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import SWEEP_BATCHES, WORKLOADS, generate  # noqa: E402

METRIC = "queries/s & item-scores/s (80M int8 IVF, nprobe64, top-2048); % HBM roofline"
E2E_INFLIGHT = 4  # query batches in flight in the end-to-end loop (2: 572k, 3: 616k, 4: 644k, 6: 225k queries/s measured)
E2E_REPS = 3      # timed end-to-end loops (the median is reported)
CHUNK_ROWS = 512  # rows per signature bit-plane chunk in the index
FLUSH_BYTES = 512 << 20  # written between L2-flushed steps (L2 is 126 MB)


def kernels_per_search(k, B, d):
    """Kernels one search launches: probe score + select, units alloc + write,
    the warp scan, the tensor-core scan (when a list can have the dense-unit
    threshold of queries: B >= that threshold, d = 64 or 128), then the
    cluster final top-k (k <= 4096, B > 8), hist + scatter + finish (k <= 4096,
    B <= 8) or hist + scatter + ties + rank (larger k). The memset node is not
    counted."""
    dmq = 8 if DENSE_MIN_Q is None else DENSE_MIN_Q
    tc = 1 if (d in (64, 128) and dmq > 0 and B >= dmq) else 0
    if k > 4096:
        return 9 + tc
    return (8 if B <= 8 else 6) + tc


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="ivf_80m", choices=sorted(WORKLOADS))
    p.add_argument("--batch", type=int, default=None, help="queries per step (default: workload B)")
    p.add_argument("--pool", type=int, default=8, help="distinct query batches cycled by the steps")
    p.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU-baseline sample budget")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-extras", action="store_true",
                   help="skip recall, large k, freshness and the other workloads")
    p.add_argument("--config-steps", type=int, default=100, help="timed steps per other workload")
    p.add_argument("--flush-reps", type=int, default=30, help="L2-flushed steps timed per workload")
    p.add_argument("--n", type=int, default=None, help="override the item count (profiling cases)")
    p.add_argument("--nlist", type=int, default=None, help="override the list count (profiling cases)")
    p.add_argument("--dense-min-queries", type=int, default=None,
                   help="ST_OPT_DENSE_MIN_QUERIES for every index (default: the library's; 0 = no tensor-core scan)")
    p.add_argument("--inflight", type=int, default=None,
                   help="query batches in flight (one stream each) in the end-to-end and in-flight loops")
    p.add_argument("--mode", default="replica", choices=["replica", "shard"],
                   help="N>1: replicas search their own batches (default), or document shards search the "
                        "same batch, all-gather their top-k over NCCL and merge it exactly")
    return p.parse_args()


# ----------------------------------------------------------------------------
# Peaks (roofline denominators)
# ----------------------------------------------------------------------------
class Peaks:
    """HBM and bf16 tensor peaks measured on this machine's B200s (driver-written
    MEASURED_PEAKS.json; else the pool's earlier measurement as a fallback);
    the int8 tensor peak as 2x the measured bf16 dense peak (the nominal
    int8 : bf16 ratio of the part, 4.5 : 2.25 PFLOP/s); the dp4a issue rate
    measured here by the microbenchmark in filtered_int8_ann_b200/microbench."""

    def __init__(self):
        self.hbm_gbs, self.bf16_tflops, self.bf16_sustained, self.kind = 6650.0, 1590.0, 1400.0, "fallback"
        try:
            with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
                j = json.load(f)
            self.hbm_gbs = float(j["hbm_gbs"])
            self.bf16_tflops = float(j.get("bf16_tflops", self.bf16_tflops))
            self.bf16_sustained = float(j.get("bf16_tflops_sustained", self.bf16_sustained))
            self.kind = "measured"
        except Exception:
            pass
        self.int8_tensor_tops = 2.0 * self.bf16_tflops
        self.dp4a_tops = self._dp4a()

    @staticmethod
    def _dp4a():
        from filtered_int8_ann_b200 import build as libbuild
        path = libbuild.PEAKS_OUT
        if not os.path.exists(path):
            return None
        L = ctypes.CDLL(path)
        L.st_peak_dp4a_tops.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_double)]
        L.st_peak_dp4a_tops.restype = ctypes.c_int
        v = ctypes.c_double(0.0)
        return float(v.value) if L.st_peak_dp4a_tops(5, ctypes.byref(v)) == 0 else None

    def describe(self):
        return {"hbm_gbs": self.hbm_gbs, "hbm_kind": self.kind,
                "int8_tensor_tops": self.int8_tensor_tops,
                "int8_tensor_kind": f"2 x bf16 dense {self.bf16_tflops:.0f} TFLOP/s ({self.kind}, burst)",
                "dp4a_tops": self.dp4a_tops, "dp4a_kind": "measured (dp4a_peak.cu, 8 chains per thread)"}


def roofline(bytes_, ops, ms, pk, dense_frac=0.0):
    """Bound times of one launch (or step) and the fraction of the slower bound
    achieved. The int8 products of the dense units (a fraction `dense_frac` of
    the eligible pairs) ran on the tensor cores, the others on dp4a: the
    compute bound is the sum of the two parts' times at their peaks."""
    t = ms * 1e-3
    t_hbm = bytes_ / (pk.hbm_gbs * 1e9)
    t_tensor = ops / (pk.int8_tensor_tops * 1e12)
    t_dp4a = ops / (pk.dp4a_tops * 1e12) if pk.dp4a_tops else None
    t_tc_part = ops * dense_frac / (pk.int8_tensor_tops * 1e12)
    t_dp_part = (ops * (1.0 - dense_frac) / (pk.dp4a_tops * 1e12)) if pk.dp4a_tops else 0.0
    t_comp = t_tc_part + t_dp_part
    bound = "hbm" if t_hbm >= t_comp else ("alu" if t_dp_part >= t_tc_part else "tensor")
    return {"bound": bound, "frac": max(t_hbm, t_comp) / t if t > 0 else None,
            "hbm_frac": t_hbm / t if t > 0 else None, "achieved_gbs": bytes_ / t / 1e9 if t > 0 else None,
            "int8_tensor_frac": t_tensor / t if t > 0 else None,
            "dp4a_frac": (t_dp4a / t) if (t_dp4a is not None and t > 0) else None,
            "achieved_tops": ops / t / 1e12 if t > 0 else None,
            "dense_pair_frac": dense_frac, "compute_frac": t_comp / t if t > 0 else None}


def scan_traffic(workload):
    """DRAM bytes per scan launch from the committed ncu record, if it was
    measured on the scan source as it is now (else None)."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "scan_kernel_traffic.json")) as f:
            rec = json.load(f)
        h = hashlib.sha256()
        for fn in rec["sources"]:
            with open(os.path.join(ROOT, "filtered_int8_ann_b200", "csrc", fn), "rb") as fh:
                h.update(fh.read())
        if h.hexdigest() != rec["source_sha256"]:
            return None
        return float(rec["per_launch"][workload]["dram_bytes"])
    except Exception:
        return None


class Clocks:
    """nvidia-smi sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------
# Ranks
# ----------------------------------------------------------------------------
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def allreduce_max(x, world, device="cuda"):
    """Max over ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def allreduce_sum(x, world, device="cuda"):
    """Sum over ranks (whole-job work)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def rank_query_rows(rank, B, pool):
    """Rows of the generated query set that rank `rank` searches: its own
    `pool` batches of B queries, disjoint from every other rank's."""
    return rank * B * pool, (rank + 1) * B * pool


def make_data(args, world, rank, device="cuda", name=None, B=None, pool=None):
    wl = WORKLOADS[name or args.workload]
    if name is None and (args.n or args.nlist):
        n = args.n or wl.n
        nl = args.nlist or wl.nlist
        wl = wl.with_(name=f"{wl.name}[n={n},nlist={nl}]", n=n, nlist=nl)
    B = B or args.batch or wl.B
    pool = max(1, pool or args.pool)
    # every rank builds the same index; each draws its own query batches
    total_q = B * pool * world
    data = generate(wl.with_(B=total_q), device=device)
    r0, r1 = rank_query_rows(rank, B, pool)
    q = data.queries[r0:r1].reshape(pool, B, -1).contiguous()
    m = data.masks[r0:r1].reshape(pool, B, -1).contiguous()
    return wl.with_(B=B), data, q, m


# ----------------------------------------------------------------------------
# Byte and operation models
# ----------------------------------------------------------------------------
def _probed_rows(off, sizes, lists):
    """Row indices of the lists `lists` (1-D), concatenated."""
    starts, lens = off[lists], sizes[lists]
    return torch.repeat_interleave(starts - torch.cumsum(lens, 0) + lens, lens) + torch.arange(
        int(lens.sum()), device=off.device)


def byte_model(data, probe, qmasks, W, d, k, nlist, alt=None):
    """Algorithmic bytes of one search (probe [B, P] of the batch).

    Scan kernel, index layout of the library: every probed list is read once
    per batch; its signatures are bit-planes per 512-row chunk (64 bytes per
    plane) and a chunk needs the planes of the bits set in the union of the
    masks of the queries probing the list; a row (d bytes) is read only when it
    is eligible for at least one of those queries (`scan_planes`).
    The same with row-major signatures (8W bytes for every scanned row), the
    model the method's description implies (`scan_rowmajor`).
    Whole step: the scan plus the centroids (nlist d), the queries and masks
    (B (d + 8W)) and the outputs (B k 12) -- `step_planes`, `step_rowmajor`.
    Full scan: every row and signature of every distinct probed list.
    alt [B, A, W] (optional): alternative masks of each query (an item passing
    any of the query's masks is eligible): a list's planes are those of the
    union of all of them, a row is read when it passes any."""
    off = data.offsets
    sizes = off[1:] - off[:-1]
    lists = torch.unique(probe.flatten().long())
    scanned = int(sizes[lists].sum())
    pr = probe.long().cpu().numpy()
    mk = qmasks.cpu().numpy().view(np.uint64).reshape(qmasks.shape[0], -1)
    if alt is not None:
        mk = mk | np.bitwise_or.reduce(alt.cpu().numpy().view(np.uint64), axis=1)
    union = np.zeros((sizes.numel(), mk.shape[1]), dtype=np.uint64)
    for w in range(mk.shape[1]):
        np.bitwise_or.at(union[:, w], pr.reshape(-1), np.repeat(mk[:, w], pr.shape[1]))
    ls = lists.cpu().numpy()
    bits = np.zeros(ls.size, dtype=np.int64)
    for w in range(mk.shape[1]):
        bits += np.array([bin(int(x)).count("1") for x in union[ls, w]], dtype=np.int64)
    chunks = (sizes[lists].cpu().numpy() + CHUNK_ROWS - 1) // CHUNK_ROWS
    plane_bytes = int((chunks * bits * (CHUNK_ROWS // 8)).sum())
    # rows eligible for at least one query probing their list, queries in
    # groups of at most ~32M probed rows
    surv = torch.zeros(data.items.shape[0], dtype=torch.bool, device=off.device)
    per_q = sizes[probe.long()].sum(1)
    b0, B = 0, probe.shape[0]
    # eligible (query, item) pairs in lists the tensor-core scan takes (probed
    # by at least the dense-unit threshold of queries) and in all lists
    dmq = 8 if DENSE_MIN_Q is None else DENSE_MIN_Q
    qcount = torch.bincount(probe.flatten().long(), minlength=nlist)
    dense_list = (qcount >= dmq) if (dmq > 0 and d in (64, 128)) else torch.zeros_like(qcount, dtype=torch.bool)
    pairs = pairs_dense = 0
    while b0 < B:
        b1, acc = b0, 0
        while b1 < B and (b1 == b0 or acc + int(per_q[b1]) <= (32 << 20)):
            acc += int(per_q[b1])
            b1 += 1
        pl = probe[b0:b1].long()
        idx = _probed_rows(off, sizes, pl.reshape(-1))
        owner = torch.repeat_interleave(torch.arange(b0, b1, device=off.device), sizes[pl].sum(1))
        m = qmasks[owner]
        ok = torch.all((data.sigs[idx] & m) == m, dim=1)
        for j in range(alt.shape[1] if alt is not None else 0):
            ma = alt[owner, j]
            ok |= torch.all((data.sigs[idx] & ma) == ma, dim=1)
        surv[idx[ok]] = True
        lst = torch.repeat_interleave(pl.reshape(-1), sizes[pl.reshape(-1)])
        pairs += int(ok.sum())
        pairs_dense += int((ok & dense_list[lst]).sum())
        b0 = b1
    n_surv = int(surv.sum())
    extra = nlist * d + B * (d + 8 * W) + B * k * 12
    scan_planes = plane_bytes + d * n_surv
    scan_rowmajor = 8 * W * scanned + d * n_surv
    return {"scan_planes": scan_planes, "scan_rowmajor": scan_rowmajor,
            "step_planes": scan_planes + extra, "step_rowmajor": scan_rowmajor + extra,
            "full_scan": (8 * W + d) * scanned, "plane_bytes": plane_bytes,
            "scanned_items": scanned, "survivor_rows": n_surv, "distinct_lists": int(lists.numel()),
            "dense_pair_frac": pairs_dense / pairs if pairs else 0.0}


def bloom_fp(data, probe, q0):
    """Bloom false positives of one batch: over every (query, item of a list
    the query probes) pair, the items whose signature passes the query's mask
    and the ones among them whose exact attributes do not match the query's
    (language, country, required flags). Queries are rows q0 .. q0+B-1 of the
    generated data. Returns (pairs passing the Bloom test, false positives,
    exact matches that fail the Bloom test -- always 0: Bloom filters have no
    false negatives)."""
    off = data.offsets
    sizes = off[1:] - off[:-1]
    passed = fp = fn = 0
    for b in range(probe.shape[0]):
        idx = _probed_rows(off, sizes, probe[b].long())
        m = data.masks[q0 + b].view(1, -1)
        ok = torch.all((data.sigs[idx] & m) == m, dim=1)
        ql, qc, qf = int(data.q_lang[q0 + b]), int(data.q_country[q0 + b]), data.q_flags[q0 + b]
        exact = torch.all(data.flags[idx] | ~qf.view(1, -1), dim=1)
        if ql >= 0:
            exact &= data.lang[idx] == ql
        if qc >= 0:
            exact &= data.country[idx] == qc
        passed += int(ok.sum())
        fp += int((ok & ~exact).sum())
        fn += int((exact & ~ok).sum())
    return passed, fp, fn


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def cpu_baseline(data, q, m, wl, budget_s):
    """The CPU oracle timed on the host cores over a bounded sample of the same
    workload: batches of one query per host thread, cycling through the query
    pool, until about `budget_s` seconds of wall time have passed; then, for a
    third of that budget, one query at a time on one thread."""
    import oracle
    from workloads import to_numpy
    a = to_numpy(data)
    qs = q.reshape(-1, q.shape[-1]).cpu().numpy()
    ms = m.reshape(-1, m.shape[-1]).cpu().numpy().view(np.uint64)
    cores = oracle.max_threads()
    nq_total = qs.shape[0]
    done, start, t0 = 0, 0, time.perf_counter()
    while True:
        b1 = min(nq_total, start + cores)
        oracle.search(a["items"], a["sigs"], a["offsets"], a["centroids"], qs, ms, wl.nprobe, wl.k,
                      b0=start, b1=b1, nthreads=cores)
        done += b1 - start
        start = 0 if b1 >= nq_total else b1
        dt = time.perf_counter() - t0
        if dt >= budget_s:
            break
    done1, start, t0 = 0, 0, time.perf_counter()
    while True:
        oracle.search(a["items"], a["sigs"], a["offsets"], a["centroids"], qs, ms, wl.nprobe, wl.k,
                      b0=start, b1=start + 1, nthreads=1)
        done1 += 1
        start = (start + 1) % nq_total
        dt1 = time.perf_counter() - t0
        if dt1 >= budget_s / 3:
            break
    return {"value": done / dt, "unit": "queries/s", "cores": cores, "kind": "oracle",
            "sample": f"{done} queries of the timed workload in batches of {cores} (one per host thread, "
                      f"OpenMP over queries), {dt:.1f} s wall",
            "single_thread": {"value": done1 / dt1, "unit": "queries/s",
                              "sample": f"{done1} queries one at a time on one thread, {dt1:.1f} s wall"},
            "cpu_model": cpu_model()}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from workloads import to_numpy
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    wl, data, q, m = make_data(args, 1, 0)
    a = to_numpy(data)
    del data
    torch.cuda.empty_cache()
    qs = q.reshape(-1, q.shape[-1]).cpu().numpy()
    ms = m.reshape(-1, m.shape[-1]).cpu().numpy().view(np.uint64)
    cores = oracle.max_threads()
    nq_total = qs.shape[0]

    def step(i):
        b0 = (i * cores) % nq_total
        b1 = min(nq_total, b0 + cores)
        oracle.search(a["items"], a["sigs"], a["offsets"], a["centroids"], qs, ms, wl.nprobe, wl.k,
                      b0=b0, b1=b1, nthreads=cores)
        return b1 - b0

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    done = 0
    for i in range(args.steps):
        done += step(args.warmup + i)
    dt = time.perf_counter() - t0
    v = done / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "queries/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8/int32",
        "data": "synthetic",
        "config": {"workload": wl.name, "n": wl.n, "d": wl.d, "nlist": wl.nlist, "B": wl.B,
                   "nprobe": wl.nprobe, "k": wl.k, "sig_bits": wl.sig_bits,
                   "note": "CPU oracle, each step one query per host thread"},
        "cpu_baseline": {"value": v, "unit": "queries/s", "cores": cores, "kind": "oracle",
                         "sample": f"{done} queries over {args.steps} steps of {cores} queries"},
        "e2e": {"value": v, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


DENSE_MIN_Q = None  # set from --dense-min-queries


def open_index(st, items, sigs, offsets, centroids):
    idx = st.Index(items, sigs, offsets, centroids)
    if DENSE_MIN_Q is not None:
        idx.set_option(st.ST_OPT_DENSE_MIN_QUERIES, DENSE_MIN_Q)
    return idx


# ----------------------------------------------------------------------------
# Timing helpers
# ----------------------------------------------------------------------------
def sampled_steps(K, pool):
    """Steps whose search is repeated with stage events after the timed
    region: one in `stride`, the stride coprime with the batch pool so every
    batch is sampled equally. An event between two kernels ends the
    programmatic dependent launch across it, so the timed steps record none
    and run exactly as a caller's searches do."""
    stride = next(s_ for s_ in range(3, 1000) if math.gcd(s_, pool) == 1)
    return stride, list(range(0, K, stride))


def stage_times(evs, sampled):
    st_ms = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(4)] for i in sampled])
    return st_ms


def flushed_steps(search, reps, flush):
    """Median device time of one search with the L2 flushed before it: a
    buffer larger than L2 is written between the timed searches, outside the
    events."""
    ts = []
    pairs = []
    for r in range(reps):
        flush.fill_(r & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        search(r)
        e1.record()
        pairs.append((e0, e1))
    torch.cuda.synchronize()
    for e0, e1 in pairs:
        ts.append(e0.elapsed_time(e1))
    return float(statistics.median(ts))


def recall(ivf_ids, flat_ids):
    """Mean over queries of |IVF top-k ∩ flat top-k| / |flat top-k| (flat =
    exact filtered search over every item)."""
    r = []
    for a, b in zip(ivf_ids, flat_ids):
        fb = set(int(x) for x in b if x >= 0)
        if fb:
            r.append(len(fb & set(int(x) for x in a if x >= 0)) / len(fb))
    return float(np.mean(r)) if r else None


# ----------------------------------------------------------------------------
# One workload measured the same way as the headline (used for per_config)
# ----------------------------------------------------------------------------
def measure_config(st, name, B, steps, warmup, flush_reps, flush, pk, pool=4, data=None, idx=None,
                   recall_flat=False):
    wl = WORKLOADS[name].with_(B=B)
    own = data is None
    if own:
        data = generate(wl.with_(B=B * pool), device="cuda")
        idx = open_index(st, data.items, data.sigs, data.offsets, data.centroids)
    q = data.queries[:B * pool].reshape(pool, B, -1).contiguous()
    m = data.masks[:B * pool].reshape(pool, B, -1).contiguous()
    P, k, d, W = wl.nprobe, wl.k, wl.d, wl.W
    ids = torch.empty((B, k), dtype=torch.int64, device="cuda")
    sc = torch.empty((B, k), dtype=torch.int32, device="cuda")
    elig = torch.empty((pool, B), dtype=torch.int64, device="cuda")
    cands = torch.empty((pool, B), dtype=torch.int64, device="cuda")
    probe = torch.empty((pool, B, P), dtype=torch.int32, device="cuda")
    for b in range(pool):
        idx.search(q[b], m[b], P, k, out_ids=ids, out_scores=sc, eligible=elig[b], probe=probe[b],
                   candidates=cands[b])
    assert idx.check() == st.ST_OK
    models = [byte_model(data, probe[b], m[b], W, d, k, wl.nlist) for b in range(min(pool, 2))]
    mdl = {key: float(np.mean([x[key] for x in models])) for key in models[0]}
    for i in range(warmup):
        idx.search(q[i % pool], m[i % pool], P, k, out_ids=ids, out_scores=sc)
    stride, sampled = sampled_steps(steps, pool)
    evs = {i: [torch.cuda.Event(enable_timing=True) for _ in range(5)] for i in sampled}
    for row in evs.values():  # torch creates the CUDA event at its first record
        for e in row:
            e.record()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s0.record()
    for i in range(steps):
        idx.search(q[i % pool], m[i % pool], P, k, out_ids=ids, out_scores=sc)
    s1.record()
    torch.cuda.synchronize()
    assert idx.check() == st.ST_OK
    ms = s0.elapsed_time(s1) / steps
    for i in sampled:  # stage times, outside the timed region
        idx.search(q[i % pool], m[i % pool], P, k, out_ids=ids, out_scores=sc, stage_events=evs[i])
    torch.cuda.synchronize()
    stg = stage_times(evs, sampled).mean(0)
    fl_ms = flushed_steps(lambda r: idx.search(q[r % pool], m[r % pool], P, k, out_ids=ids, out_scores=sc),
                          flush_reps, flush)
    el = float(elig.sum(1).double().mean())
    ops_scan = 2.0 * d * el
    ops_step = ops_scan + 2.0 * d * B * wl.nlist
    out = {"workload": name, "B": B, "nprobe": P, "k": k, "n": wl.n, "d": d, "nlist": wl.nlist,
           "queries_per_s": B / (ms * 1e-3), "item_scores_per_s": el / (ms * 1e-3), "ms_per_step": ms,
           "l2_flushed": {"ms_per_step": fl_ms, "queries_per_s": B / (fl_ms * 1e-3)},
           "stage_ms": {"probe": stg[0], "plan": stg[1], "scan": stg[2], "select": stg[3]},
           "selectivity": el / max(1.0, float((data.offsets[1:] - data.offsets[:-1])[probe.long()]
                                              .sum(2).double().mean()) * B),
           "eligible_per_query": el / B,
           "candidates_per_query": float(cands.double().mean()),
           "candidate_bytes_per_step": float(cands.sum(1).double().mean()) * 8,
           "bytes": mdl, "int8_ops": {"scan": ops_scan, "step": ops_step},
           "scan_roofline": {"planes": roofline(mdl["scan_planes"], ops_scan, stg[2], pk, mdl["dense_pair_frac"]),
                             "rowmajor": roofline(mdl["scan_rowmajor"], ops_scan, stg[2], pk, mdl["dense_pair_frac"])},
           "step_roofline": {"planes": roofline(mdl["step_planes"], ops_step, ms, pk, mdl["dense_pair_frac"]),
                             "rowmajor": roofline(mdl["step_rowmajor"], ops_step, ms, pk, mdl["dense_pair_frac"])},
           "l2": f"steps cycle {pool} query batches; l2_flushed writes {FLUSH_BYTES >> 20} MB between steps"}
    if recall_flat and P < wl.nlist <= 4096:
        # flat filtered search = the same index probed with nprobe = nlist
        idx.set_option(st.ST_OPT_CANDIDATE_BYTES, 12 << 30)
        Bq = min(B, 64)
        fids, _ = idx.search(q[0][:Bq].contiguous(), m[0][:Bq].contiguous(), wl.nlist, k)
        vids, _ = idx.search(q[0][:Bq].contiguous(), m[0][:Bq].contiguous(), P, k)
        idx.set_option(st.ST_OPT_CANDIDATE_BYTES, 2 << 30)
        assert idx.check() == st.ST_OK
        out["recall_at_k"] = {"value": recall(vids.cpu().numpy(), fids.cpu().numpy()), "queries": Bq,
                              "flat": f"same index, nprobe = nlist = {wl.nlist}"}
    if own:
        idx.close()
        del data
        torch.cuda.empty_cache()
    return out


def freshness(st, idx, src_items, src_sigs, nlist, q, m, P, k, m_rows=100_000, batch=10_000):
    """Streamed-update costs on a live index: rows/s of insertion (random
    lists), in-place update and deletion of m_rows items, and the search time
    before and after."""
    ids = torch.empty((q.shape[1], k), dtype=torch.int64, device="cuda")
    sc = torch.empty((q.shape[1], k), dtype=torch.int32, device="cuda")

    def search_ms(reps=50):
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(reps):
            idx.search(q[i % q.shape[0]], m[i % m.shape[0]], P, k, out_ids=ids, out_scores=sc)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    before = search_ms()
    rng = np.random.default_rng(7)
    lists = rng.integers(0, nlist, m_rows).astype(np.int32)
    # room for the insertions first (one copy of the index, untimed)
    idx.set_option(st.ST_OPT_INSERT_RESERVE, int(min(nlist, m_rows)) * 512)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    new_ids = []
    for b0 in range(0, m_rows, batch):
        b1 = min(m_rows, b0 + batch)
        new_ids.append(idx.insert(lists[b0:b1], src_items[b0:b1], src_sigs[b0:b1]))
    t_ins = time.perf_counter() - t0
    new_ids = torch.from_numpy(np.concatenate(new_ids)).cuda()
    perm = torch.randperm(m_rows, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for b0 in range(0, m_rows, batch):
        sel = perm[b0:b0 + batch]
        idx.update(new_ids[sel], items=src_items[sel], sigs=src_sigs[sel])
    torch.cuda.synchronize()
    t_upd = time.perf_counter() - t0
    after_insert = search_ms()
    t0 = time.perf_counter()
    for b0 in range(0, m_rows, batch):
        idx.delete(new_ids[perm[b0:b0 + batch]])
    torch.cuda.synchronize()
    t_del = time.perf_counter() - t0
    after_delete = search_ms()
    assert idx.check() == st.ST_OK
    return {"rows": m_rows, "batch": batch,
            "insert_rows_per_s": m_rows / t_ins, "update_rows_per_s": m_rows / t_upd,
            "delete_rows_per_s": m_rows / t_del,
            "search_ms_before": before, "search_ms_after_insert": after_insert,
            "search_ms_after_delete": after_delete,
            "note": "host wall time per call sequence (insert waits for its stream); searches warm, cycling batches"}


# ----------------------------------------------------------------------------
def main():
    args = parse()
    global DENSE_MIN_Q, E2E_INFLIGHT
    DENSE_MIN_Q = args.dense_min_queries
    if args.inflight is not None:
        E2E_INFLIGHT = max(1, args.inflight)
    if args.impl == "reference":
        return run_reference(args)
    world, rank, local = dist_setup(args)
    import filtered_int8_ann_b200 as st

    shard = args.mode == "shard"
    extras = (not args.no_extras) and world == 1 and not shard and args.n is None and args.nlist is None
    pk = Peaks()
    # shards all search rank 0's batches; replicas search their own
    wl, data, q, m = make_data(args, 1 if shard else world, 0 if shard else rank)
    B, P, k, d, W = wl.B, wl.nprobe, wl.k, wl.d, wl.W
    pool = q.shape[0]
    dev = torch.device("cuda", local)
    if shard:
        from types import SimpleNamespace
        from filtered_int8_ann_b200.shard import shard_arrays
        it, sg, off, base = shard_arrays(data.items, data.sigs, data.offsets, world, rank)
        data = SimpleNamespace(items=it.contiguous(), sigs=sg.contiguous(), offsets=off, centroids=data.centroids,
                               queries=data.queries, masks=data.masks)
        idx = open_index(st, data.items, data.sigs, data.offsets, data.centroids)
        idx.set_option(st.ST_OPT_ID_OFFSET, base)
        g_ids = torch.empty((world, B, k), dtype=torch.int64, device=dev)
        g_sc = torch.empty((world, B, k), dtype=torch.int32, device=dev)
        m_ids = torch.empty((B, k), dtype=torch.int64, device=dev)
        m_sc = torch.empty((B, k), dtype=torch.int32, device=dev)
    else:
        idx = open_index(st, data.items, data.sigs, data.offsets, data.centroids)
    ids = torch.empty((B, k), dtype=torch.int64, device=dev)
    scores = torch.empty((B, k), dtype=torch.int32, device=dev)

    # per-batch eligible counts, candidates and byte model (untimed)
    elig = torch.empty((pool, B), dtype=torch.int64, device=dev)
    cands = torch.empty((pool, B), dtype=torch.int64, device=dev)
    probe = torch.empty((pool, B, P), dtype=torch.int32, device=dev)
    for b in range(pool):
        idx.search(q[b], m[b], P, k, out_ids=ids, out_scores=scores, eligible=elig[b], probe=probe[b],
                   candidates=cands[b])
    assert idx.check() == st.ST_OK
    models = [byte_model(data, probe[b], m[b], W, d, k, wl.nlist) for b in range(pool)]
    fp_stats = None
    if hasattr(data, "lang"):  # the generator's exact attributes (not kept for a shard's arrays)
        r0 = rank_query_rows(rank, B, pool)[0]
        fp_stats = np.array([bloom_fp(data, probe[b], r0 + b * B) for b in range(pool)]).sum(0)
    elig_per_batch = elig.sum(1).double().cpu().numpy()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(data, q, m, wl, args.cpu_seconds)
    # kept for the extras: the flat index (recall) and rows to insert
    flat_src = None
    if extras:
        nsrc = 100_000
        sel = torch.randint(0, data.items.shape[0], (nsrc,), device=dev, generator=torch.Generator(device=dev).manual_seed(5))
        flat_src = (data.items[sel].contiguous(), data.sigs[sel].contiguous())
        flat_idx = open_index(st, data.items, data.sigs,
                            torch.tensor([0, data.items.shape[0]], dtype=torch.int64, device=dev),
                            torch.zeros((1, d), dtype=torch.int8, device=dev))
    # OR of M masks per query (the extras): M - 1 alternatives per query, the
    # masks of the next queries of the batch (other languages and countries);
    # the scan's algorithmic bytes of one fused search and of M single searches
    or_alts, or_bytes = {}, {}
    if extras:
        for M in (2, 4):
            or_alts[M] = [torch.stack([torch.roll(m[b], -j, dims=0) for j in range(1, M)], dim=1).contiguous()
                          for b in range(pool)]
            sets0 = [m[0]] + [or_alts[M][0][:, j].contiguous() for j in range(M - 1)]
            or_bytes[M] = (byte_model(data, probe[0], m[0], W, d, k, wl.nlist, alt=or_alts[M][0])["scan_planes"],
                           sum(byte_model(data, probe[0], x, W, d, k, wl.nlist)["scan_planes"] for x in sets0))
    del data
    torch.cuda.empty_cache()

    def step(i, stage_events=None):
        if stage_events is None:
            idx.search(q[i % pool], m[i % pool], P, k, out_ids=ids, out_scores=scores)
        else:
            idx.search(q[i % pool], m[i % pool], P, k, out_ids=ids, out_scores=scores, stage_events=stage_events)
        if shard:
            # every shard's top-k to every rank, then the exact merge
            if world > 1:
                import torch.distributed as dist
                dist.all_gather_into_tensor(g_ids, ids)
                dist.all_gather_into_tensor(g_sc, scores)
            else:
                g_ids[0].copy_(ids)
                g_sc[0].copy_(scores)
            st.st_merge_topk(g_ids, g_sc, out_ids=m_ids, out_scores=m_sc)

    # warm-up
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    K = args.steps
    stride, sampled = sampled_steps(K, pool)
    evs = {i: [torch.cuda.Event(enable_timing=True) for _ in range(5)] for i in sampled}
    for row in evs.values():  # torch creates the CUDA event at its first record
        for e in row:
            e.record()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    start.record()
    for i in range(K):
        step(i)
    end.record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    assert idx.check() == st.ST_OK
    for i in sampled:  # stage times, outside the timed region
        step(i, evs[i])
    torch.cuda.synchronize()
    ms_local = start.elapsed_time(end)
    ms = allreduce_max(ms_local, world)

    stage_ms = stage_times(evs, sampled)
    stage_mean = stage_ms.mean(0)
    scan_b = np.array([models[i % pool]["scan_planes"] for i in sampled], dtype=np.float64)
    scan_gbs = float(scan_b.sum() / (stage_ms[:, 2].sum() * 1e-3) / 1e9)
    scan_ms = float(stage_ms[:, 2].mean())
    mean = {key: float(np.mean([x[key] for x in models])) for key in models[0]}
    elig_mean = float(elig_per_batch.mean())
    ops_scan = 2.0 * d * elig_mean
    ops_step = ops_scan + 2.0 * d * B * wl.nlist

    # shards share one batch per step (their eligible counts add up); replicas each run their own
    total_q = float(B * K) if shard else allreduce_sum(float(B * K), world)
    elig_total = allreduce_sum(float(sum(elig_per_batch[i % pool] for i in range(K))), world)
    value = total_q / (ms * 1e-3)

    # the same search with the L2 flushed before every step
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    fl_ms = allreduce_max(flushed_steps(lambda r: step(r), args.flush_reps, flush), world)

    # the same device-resident searches with E2E_INFLIGHT batches in flight on
    # as many streams (no copies): how much of the end-to-end figure comes from
    # running two searches at once rather than from the copies overlapping
    Kc = 0 if (args.no_e2e or shard) else min(K, 500)
    inflight = None
    if Kc:
        cstreams = [torch.cuda.Stream() for _ in range(E2E_INFLIGHT)]
        couts = [(torch.empty((B, k), dtype=torch.int64, device=dev), torch.empty((B, k), dtype=torch.int32, device=dev))
                 for _ in range(E2E_INFLIGHT)]

        def conc_step(i):
            j = i % E2E_INFLIGHT
            idx.search(q[i % pool], m[i % pool], P, k, out_ids=couts[j][0], out_scores=couts[j][1], stream=cstreams[j])

        for i in range(3 * E2E_INFLIGHT):
            conc_step(i)
        barrier(world)
        torch.cuda.synchronize()
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record()
        for st_ in cstreams:
            st_.wait_event(c0)
        for i in range(Kc):
            conc_step(i)
        for st_ in cstreams:
            torch.cuda.current_stream().wait_stream(st_)
        c1.record()
        torch.cuda.synchronize()
        assert idx.check() == st.ST_OK
        inflight = allreduce_sum(float(B * Kc), world) / (allreduce_max(c0.elapsed_time(c1), world) * 1e-3)

    # end to end through the host-buffer entry point (page-locked memory): a
    # serving loop with E2E_INFLIGHT batches in flight, one stream each, so one
    # batch's host<->device copies overlap another's kernels. A slot's host
    # buffers are reused only after its previous batch has completed.
    Ke = 0 if (args.no_e2e or shard) else min(K, 200)
    hq = [q[b].cpu().pin_memory() for b in range(pool)]
    hm = [m[b].cpu().pin_memory() for b in range(pool)]
    streams = [torch.cuda.Stream() for _ in range(E2E_INFLIGHT)]
    hids = [torch.empty((B, k), dtype=torch.int64).pin_memory() for _ in range(E2E_INFLIGHT)]
    hsc = [torch.empty((B, k), dtype=torch.int32).pin_memory() for _ in range(E2E_INFLIGHT)]
    done = [torch.cuda.Event() for _ in range(E2E_INFLIGHT)]

    def e2e_step(i):
        j = i % E2E_INFLIGHT
        done[j].synchronize()  # the slot's previous results are on the host
        idx.search_host_async(hq[i % pool], hm[i % pool], P, k, hids[j], hsc[j], stream=streams[j])
        done[j].record(streams[j])

    for i in range(2 * E2E_INFLIGHT if Ke else 0):
        e2e_step(i)
    # three timed loops, the median reported: this loop depends on the host
    # thread issuing calls and waiting on events, and a busy host (other jobs
    # on a shared machine) can slow one loop several-fold
    e2e_runs = []
    for _rep in range(E2E_REPS if Ke else 0):
        barrier(world)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for st_ in streams:
            st_.wait_event(e0)
        for i in range(Ke):
            e2e_step(i)
        for st_ in streams:
            torch.cuda.current_stream().wait_stream(st_)
        e1.record()
        torch.cuda.synchronize()
        ems = allreduce_max(e0.elapsed_time(e1), world)
        e2e_runs.append(allreduce_sum(float(B * Ke), world) / (ems * 1e-3))
    e2e = statistics.median(e2e_runs) if e2e_runs else None

    # ---- extras (1 GPU, replica mode, default workload sizes) --------------
    ext = {}
    if extras:
        # recall of the IVF search (nprobe P) against the exact flat filtered search
        flat_idx.set_option(st.ST_OPT_CANDIDATE_BYTES, 12 << 30)
        fids, _ = flat_idx.search(q[0], m[0], 1, k)
        assert flat_idx.check() == st.ST_OK
        flat_idx.close()
        idx.search(q[0], m[0], P, k, out_ids=ids, out_scores=scores)
        ext["recall_at_k"] = {"value": recall(ids.cpu().numpy(), fids.cpu().numpy()), "queries": B,
                              "flat": "index of one list holding every item, zero centroid, nprobe 1"}
        del fids
        # large k on the same index
        lk = {}
        for kk in (16384, 65536):
            try:
                li = torch.empty((B, kk), dtype=torch.int64, device=dev)
                ls = torch.empty((B, kk), dtype=torch.int32, device=dev)
                for i in range(3):
                    idx.search(q[i % pool], m[i % pool], P, kk, out_ids=li, out_scores=ls)
                torch.cuda.synchronize()
                x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                reps = 20
                x0.record()
                for i in range(reps):
                    idx.search(q[i % pool], m[i % pool], P, kk, out_ids=li, out_scores=ls)
                x1.record()
                torch.cuda.synchronize()
                assert idx.check() == st.ST_OK
                t = x0.elapsed_time(x1) / reps
                lk[str(kk)] = {"ms_per_step": t, "queries_per_s": B / (t * 1e-3)}
                del li, ls
            except st.StError as ex:
                lk[str(kk)] = {"error": str(ex)}
        ext["large_k"] = lk
        # OR of M masks per query (M - 1 alternatives: other queries' masks of
        # the batch, i.e. other languages and countries): one fused search
        # against M single-mask searches merged, with the scan's algorithmic
        # bytes of each
        orr = {}
        for M in (2, 4):
            alts = or_alts[M]
            sets = [torch.cat([m[b].unsqueeze(0), alts[b].permute(1, 0, 2)], dim=0).contiguous() for b in range(pool)]
            for i in range(3):
                idx.search(q[i % pool], m[i % pool], P, k, out_ids=ids, out_scores=scores, or_masks=alts[i % pool])
                idx.search_any_merged(q[i % pool], sets[i % pool], P, k)
            torch.cuda.synchronize()
            reps = 20
            x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            x0.record()
            for i in range(reps):
                idx.search(q[i % pool], m[i % pool], P, k, out_ids=ids, out_scores=scores, or_masks=alts[i % pool])
            x1.record()
            torch.cuda.synchronize()
            t_fused = x0.elapsed_time(x1) / reps
            x0.record()
            for i in range(reps):
                idx.search_any_merged(q[i % pool], sets[i % pool], P, k)
            x1.record()
            torch.cuda.synchronize()
            t_sep = x0.elapsed_time(x1) / reps
            assert idx.check() == st.ST_OK and st.st_merge_check() == st.ST_OK
            fused_b, sep_b = or_bytes[M]
            orr[str(M)] = {"fused_ms_per_step": t_fused, "separate_ms_per_step": t_sep,
                           "fused_scan_bytes": fused_b, "separate_scan_bytes": sep_b,
                           "separate": "M single-mask searches, then the exact union merge"}
        ext["or_masks"] = orr
        # streamed updates, last: they change the headline index
        ext["freshness"] = freshness(st, idx, flat_src[0], flat_src[1], wl.nlist, q, m, P, k)
        del flat_src
    idx.close()
    if extras:
        torch.cuda.empty_cache()
        # the other workloads
        pc = []
        for name in ("tiny_ivf", "mid_ivf", "flat_10m"):
            wlx = WORKLOADS[name]
            pc.append(measure_config(st, name, wlx.B, args.config_steps, 5, args.flush_reps, flush, pk))
        sw = WORKLOADS["sweep_10m"]
        pool_sw = 4
        data_sw = generate(sw.with_(B=max(SWEEP_BATCHES) * pool_sw), device=dev)
        idx_sw = open_index(st, data_sw.items, data_sw.sigs, data_sw.offsets, data_sw.centroids)
        for Bs in SWEEP_BATCHES:
            pc.append(measure_config(st, "sweep_10m", Bs, args.config_steps if Bs < 1024 else max(20, args.config_steps // 4),
                                     5, args.flush_reps, flush, pk, pool=pool_sw, data=data_sw, idx=idx_sw,
                                     recall_flat=(Bs == 64)))
        idx_sw.close()
        del data_sw
        ext["per_config"] = pc

    if rank == 0:
        traffic = scan_traffic(wl.name)
        scan_rf = roofline(mean["scan_planes"], ops_scan, scan_ms, pk, mean["dense_pair_frac"])
        line = {
            "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True,
            "scaling": "strong" if shard else "weak",
            "vs_baseline": None, "dtype": "int8/int32", "data": "synthetic",
            "config": {"workload": wl.name, "n": wl.n, "d": d, "nlist": wl.nlist, "B": B, "nprobe": P,
                       "k": k, "sig_bits": wl.sig_bits, "mask_mode": "head",
                       "l2": f"inputs larger than L2 (index {wl.n * (d + 8 * W) / 1e9:.1f} GB); steps cycle "
                             f"{pool} distinct query batches; l2_flushed: {FLUSH_BYTES >> 20} MB written "
                             f"before each of {args.flush_reps} steps",
                       "parallelism": (f"document shards x{world} (NCCL all-gather of the shards' top-k, exact merge)"
                                       if shard else f"replicas x{world} (independent query batches)")},
            "item_scores_per_s": elig_total / (ms * 1e-3),
            "l2_flushed": {"ms_per_step": fl_ms, "queries_per_s": B / (fl_ms * 1e-3) * (1 if shard else world)},
            "stage_ms": {"probe": stage_mean[0], "plan": stage_mean[1], "scan": stage_mean[2],
                         "select": stage_mean[3]},
            "roofline": {"bound": scan_rf["bound"], "kernel": "scan_kernel", "achieved": scan_gbs,
                         "peak": pk.hbm_gbs, "unit": "GB/s", "frac": scan_gbs / pk.hbm_gbs,
                         "traffic": traffic, "peak_kind": pk.kind,
                         "bytes_per_launch": mean["scan_planes"],
                         "int8_ops_per_launch": ops_scan,
                         "int8_tensor_frac": scan_rf["int8_tensor_frac"], "dp4a_frac": scan_rf["dp4a_frac"],
                         "signature_plane_bytes_per_launch": mean["plane_bytes"],
                         "rowmajor_model_bytes_per_launch": mean["scan_rowmajor"],
                         "rowmajor_model_frac": roofline(mean["scan_rowmajor"], ops_scan, scan_ms, pk,
                                                                         mean["dense_pair_frac"])["hbm_frac"],
                         "dense_pair_frac": mean["dense_pair_frac"],
                         "full_scan_bytes_per_launch": mean["full_scan"]},
            "step_roofline": {"planes": roofline(mean["step_planes"], ops_step, ms / K, pk, mean["dense_pair_frac"]),
                              "rowmajor": roofline(mean["step_rowmajor"], ops_step, ms / K, pk, mean["dense_pair_frac"]),
                              "step_bytes_planes": mean["step_planes"], "step_bytes_rowmajor": mean["step_rowmajor"],
                              "int8_ops_per_step": ops_step},
            "peaks": pk.describe(),
            "cpu_baseline": cpu,
            "e2e": {"value": e2e, "unit": "queries/s", "h2d_bytes_per_step": B * (d + 8 * W),
                    "d2h_bytes_per_step": B * k * 12,
                    "call": f"st_search_host_async, page-locked buffers, {E2E_INFLIGHT} batches in flight",
                    "runs": e2e_runs, "reported": f"median of {len(e2e_runs)} timed loops of {Ke} steps"},
            "device_inflight": None if inflight is None else {
                "value": inflight, "unit": "queries/s",
                "note": f"device-resident searches, {E2E_INFLIGHT} batches in flight on {E2E_INFLIGHT} streams"},
            "stage_sampling": f"stage events on {len(sampled)} searches repeated after the timed region "
                              f"(one step in {stride}); the timed steps record none",
            "gpu_launches": (kernels_per_search(k, B, d) + (1 if shard else 0)) * K,
            "clocks": clk,
            "workload_stats": {"scanned_items": mean["scanned_items"], "survivor_rows": mean["survivor_rows"],
                               "distinct_lists": mean["distinct_lists"],
                               "eligible_per_query": elig_mean / B,
                               "candidates_per_query": float(cands.double().mean()),
                               "candidate_bytes_per_step": float(cands.sum(1).double().mean()) * 8,
                               "bloom_false_positive_rate": (None if fp_stats is None or fp_stats[0] == 0
                                                             else float(fp_stats[1] / fp_stats[0])),
                               "bloom_false_negatives": None if fp_stats is None else int(fp_stats[2]),
                               **({"recall_at_k": ext["recall_at_k"]} if "recall_at_k" in ext else {})},
        }
        for key in ("large_k", "or_masks", "freshness", "per_config"):
            if key in ext:
                line[key] = ext[key]
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
