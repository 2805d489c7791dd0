#!/usr/bin/env python
"""Benchmark of the Bloom-filtered int8 IVF top-k search on B200.

One step = one st_search call (probe -> plan -> scan -> final top-k) over one
batch of queries, inputs resident in HBM. Default workload: 80M items, d=64,
16384 Zipf(0.8)-skewed lists, 128-bit signatures, B=64 queries, nprobe=64,
k=2048. The timed steps cycle through a pool of distinct query batches; the
index (6.4 GB) is far larger than L2.

Prints one JSON line (rank 0). `--impl reference` times the CPU oracle instead
(the reference arm; host cores only).
"""
import argparse
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

from workloads import WORKLOADS, generate  # noqa: E402

METRIC = "queries/s & item-scores/s (80M int8 IVF, nprobe64, top-2048); % HBM roofline"
KERNELS_PER_SEARCH = 8  # probe score + probe select, units alloc + write, scan, select hist + scatter + finish
E2E_INFLIGHT = 2  # query batches in flight in the end-to-end loop


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
    p.add_argument("--n", type=int, default=None, help="override the item count (profiling cases)")
    p.add_argument("--nlist", type=int, default=None, help="override the list count (profiling cases)")
    p.add_argument("--mode", default="replica", choices=["replica", "shard"],
                   help="N>1: replicas search their own batches (default), or document shards search the "
                        "same batch, all-gather their top-k over NCCL and merge it exactly")
    return p.parse_args()


def scan_traffic():
    """DRAM bytes per scan launch from the committed ncu summary, if it was
    measured on the scan source as it is now (else None)."""
    import hashlib
    try:
        text = open(os.path.join(ROOT, "profiles", "scan_kernel_traffic_ivf_80m.md")).read()
        fields = dict(l.split(": ", 1) for l in text.splitlines() if l.startswith(("source_sha256", "dram_bytes")))
        h = hashlib.sha256()
        for f in ("scan.cu", "st_internal.cuh"):
            with open(os.path.join(ROOT, "filtered_int8_ann_b200", "csrc", f), "rb") as fh:
                h.update(fh.read())
        if h.hexdigest() != fields["source_sha256"].strip():
            return None
        return float(fields["dram_bytes_per_launch_mean"])
    except Exception:
        return None


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


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


def make_data(args, world, rank, device="cuda"):
    wl = WORKLOADS[args.workload]
    if args.n or args.nlist:
        n = args.n or wl.n
        nl = args.nlist or wl.nlist
        wl = wl.with_(name=f"{wl.name}[n={n},nlist={nl}]", n=n, nlist=nl)
    B = args.batch or wl.B
    pool = max(1, args.pool)
    # every rank builds the same index; each draws its own query batches
    total_q = B * pool * world
    data = generate(wl.with_(B=total_q), device=device)
    r0, r1 = rank_query_rows(rank, B, pool)
    q = data.queries[r0:r1].reshape(pool, B, -1).contiguous()
    m = data.masks[r0:r1].reshape(pool, B, -1).contiguous()
    return wl.with_(B=B), data, q, m


CHUNK_ROWS = 512  # rows per signature bit-plane chunk in the index


def byte_model(data, probe, qmasks, W, d):
    """Algorithmic bytes of one search's list scan, for the index layout the
    library uses: every probed list is read once per batch; its signatures are
    stored as bit-planes per 512-row chunk (64 bytes per plane), and the scan
    needs, per chunk, the planes of the bits set in the union of the masks of
    the queries probing the list; a row (d bytes) is read only when it is
    eligible for at least one of those queries.
    Also returned: the same model with row-major signatures (8W bytes for every
    scanned row, the earlier layout) and the full-scan bytes (every row and
    signature of every distinct probed list)."""
    off = data.offsets
    sizes = (off[1:] - off[:-1])
    lists = torch.unique(probe.flatten())
    scanned = int(sizes[lists].sum())
    # union of the masks of the queries probing each list
    pr = probe.long().cpu().numpy()
    mk = qmasks.cpu().numpy().view(np.uint64).reshape(qmasks.shape[0], -1)
    nl = int(sizes.numel())
    union = np.zeros((nl, mk.shape[1]), dtype=np.uint64)
    for w in range(mk.shape[1]):
        np.bitwise_or.at(union[:, w], pr.reshape(-1), np.repeat(mk[:, w], pr.shape[1]))
    ls = lists.cpu().numpy()
    bits = np.zeros(ls.size, dtype=np.int64)
    for w in range(mk.shape[1]):
        u = union[ls, w]
        bits += np.array([bin(int(x)).count("1") for x in u], dtype=np.int64)
    chunks = (sizes[lists].cpu().numpy() + CHUNK_ROWS - 1) // CHUNK_ROWS
    plane_bytes = int((chunks * bits * (CHUNK_ROWS // 8)).sum())
    surv = torch.zeros(data.items.shape[0], dtype=torch.bool, device=off.device)
    for b in range(probe.shape[0]):
        lsb = probe[b].long()
        starts, lens = off[lsb], sizes[lsb]
        idx = torch.repeat_interleave(starts - torch.cumsum(lens, 0) + lens, lens) + torch.arange(
            int(lens.sum()), device=off.device)
        sg = data.sigs[idx]
        m = qmasks[b].view(1, -1)
        ok = torch.all((sg & m) == m, dim=1)
        surv[idx[ok]] = True
    n_surv = int(surv.sum())
    method = plane_bytes + d * n_surv
    rowmajor = 8 * W * scanned + d * n_surv
    full = (8 * W + d) * scanned
    return method, full, scanned, n_surv, int(lists.numel()), rowmajor, plane_bytes


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
        lsb = probe[b].long()
        starts, lens = off[lsb], sizes[lsb]
        idx = torch.repeat_interleave(starts - torch.cumsum(lens, 0) + lens, lens) + torch.arange(
            int(lens.sum()), device=off.device)
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


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    world, rank, local = dist_setup(args)
    import filtered_int8_ann_b200 as st

    shard = args.mode == "shard"
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
        idx = st.Index(data.items, data.sigs, data.offsets, data.centroids)
        idx.set_option(st.ST_OPT_ID_OFFSET, base)
        g_ids = torch.empty((world, B, k), dtype=torch.int64, device=dev)
        g_sc = torch.empty((world, B, k), dtype=torch.int32, device=dev)
        m_ids = torch.empty((B, k), dtype=torch.int64, device=dev)
        m_sc = torch.empty((B, k), dtype=torch.int32, device=dev)
    else:
        idx = st.Index(data.items, data.sigs, data.offsets, data.centroids)
    ids = torch.empty((B, k), dtype=torch.int64, device=dev)
    scores = torch.empty((B, k), dtype=torch.int32, device=dev)

    # per-batch eligible counts and byte model (untimed)
    elig = torch.empty((pool, B), dtype=torch.int64, device=dev)
    probe = torch.empty((pool, B, P), dtype=torch.int32, device=dev)
    for b in range(pool):
        idx.search(q[b], m[b], P, k, out_ids=ids, out_scores=scores, eligible=elig[b], probe=probe[b])
    assert idx.check() == st.ST_OK
    models = [byte_model(data, probe[b], m[b], W, d) for b in range(pool)]
    fp_stats = None
    if hasattr(data, "lang"):  # the generator's exact attributes (not kept for a shard's arrays)
        r0 = rank_query_rows(rank, B, pool)[0]
        fp_stats = np.array([bloom_fp(data, probe[b], r0 + b * B) for b in range(pool)]).sum(0)
    elig_per_batch = elig.sum(1).double().cpu().numpy()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(data, q, m, wl, args.cpu_seconds)
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
    # stage events on every `stride`-th timed step only: an event between two
    # kernels ends the programmatic dependent launch across it, so the other
    # steps run exactly as a caller's searches do. The stride is coprime with
    # the batch pool, so the sampled steps cover every batch equally.
    stride = next(s_ for s_ in range(3, 1000) if math.gcd(s_, pool) == 1)
    sampled = list(range(0, K, stride))
    evs = {i: [torch.cuda.Event(enable_timing=True) for _ in range(5)] for i in sampled}
    for row in evs.values():
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
        step(i, evs.get(i))
    end.record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    assert idx.check() == st.ST_OK
    ms_local = start.elapsed_time(end)
    ms = allreduce_max(ms_local, world)

    stage_ms = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(4)] for i in sampled])
    stage_mean = stage_ms.mean(0)
    scan_ms = stage_mean[2]
    method_bytes = np.array([models[i % pool][0] for i in sampled], dtype=np.float64)
    full_bytes = np.array([models[i % pool][1] for i in sampled], dtype=np.float64)
    scan_gbs = float(method_bytes.sum() / (stage_ms[:, 2].sum() * 1e-3) / 1e9)
    peak, peak_kind = peaks()

    # shards share one batch per step (their eligible counts add up); replicas each run their own
    total_q = float(B * K) if shard else allreduce_sum(float(B * K), world)
    elig_total = allreduce_sum(float(sum(elig_per_batch[i % pool] for i in range(K))), world)
    value = total_q / (ms * 1e-3)

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

    for i in range(3 if Ke else 0):
        e2e_step(i)
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
    e2e = allreduce_sum(float(B * Ke), world) / (ems * 1e-3) if Ke else None
    idx.close()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True,
            "scaling": "strong" if shard else "weak",
            "vs_baseline": None, "dtype": "int8/int32", "data": "synthetic",
            "config": {"workload": wl.name, "n": wl.n, "d": d, "nlist": wl.nlist, "B": B, "nprobe": P,
                       "k": k, "sig_bits": wl.sig_bits, "mask_mode": "head",
                       "l2": f"inputs larger than L2 (index {wl.n * (d + 8 * W) / 1e9:.1f} GB); steps cycle {pool} distinct query batches",
                       "parallelism": (f"document shards x{world} (NCCL all-gather of the shards' top-k, exact merge)"
                                       if shard else f"replicas x{world} (independent query batches)")},
            "item_scores_per_s": elig_total / (ms * 1e-3),
            "stage_ms": {"probe": stage_mean[0], "plan": stage_mean[1], "scan": stage_mean[2],
                         "select": stage_mean[3]},
            "roofline": {"bound": "hbm", "kernel": "scan_kernel", "achieved": scan_gbs, "peak": peak,
                         "unit": "GB/s", "frac": scan_gbs / peak,
                         "traffic": scan_traffic() if wl.name == "ivf_80m" else None,
                         "peak_kind": peak_kind,
                         "bytes_per_launch": float(method_bytes.mean()),
                         "signature_plane_bytes_per_launch": float(np.mean([x[6] for x in models])),
                         "rowmajor_model_bytes_per_launch": float(np.mean([x[5] for x in models])),
                         "full_scan_bytes_per_launch": float(full_bytes.mean()),
                         "step_frac": float(method_bytes.mean() / (ms / K * 1e-3) / 1e9 / peak)},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e, "unit": "queries/s", "h2d_bytes_per_step": B * (d + 8 * W),
                    "d2h_bytes_per_step": B * k * 12,
                    "call": f"st_search_host_async, page-locked buffers, {E2E_INFLIGHT} batches in flight"},
            "device_inflight": None if inflight is None else {
                "value": inflight, "unit": "queries/s",
                "note": f"device-resident searches, {E2E_INFLIGHT} batches in flight on {E2E_INFLIGHT} streams"},
            "stage_sampling": f"stage events on one timed step in {stride} ({len(sampled)} of {K})",
            "gpu_launches": (KERNELS_PER_SEARCH + (1 if shard else 0)) * K,  # memset node not counted
            "clocks": clk,
            "workload_stats": {"scanned_items": float(np.mean([x[2] for x in models])),
                               "survivor_rows": float(np.mean([x[3] for x in models])),
                               "distinct_lists": float(np.mean([x[4] for x in models])),
                               "eligible_per_query": float(elig_per_batch.mean() / B),
                               "bloom_false_positive_rate": (None if fp_stats is None or fp_stats[0] == 0
                                                             else float(fp_stats[1] / fp_stats[0])),
                               "bloom_false_negatives": None if fp_stats is None else int(fp_stats[2])},
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
