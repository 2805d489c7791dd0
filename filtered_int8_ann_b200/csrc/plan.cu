// Plan: cut every probed list into work units of kWarpItems rows x a group of
// the queries probing it, so the scan reads each probed list once per batch
// however many queries probe it. One self-contained 16-byte entry per unit:
// {first row, chunk, first query slot, rows << 16 | queries}. Lists probed by
// fewer than tc_min_q queries get groups of up to kQMax queries, scanned by
// one warp each (scan.cu); lists probed by more, or whose queries expect many
// eligible rows (dense_by_selectivity), get groups of up to kTcQMax queries in
// a second table, scanned as dense tensor-core tiles (scan_tc.cu).
//
// The probe kernel already filed each query into the slot row of every list it
// chose (slots L*B .. L*B + count-1), so no scan over lists or scatter of pairs
// is needed here. Two small balanced kernels:
//   * units_alloc: one thread per list; a warp-wide scan of the lists' unit
//     counts and one atomic per warp give every probed list its block of the
//     unit table (blocks land in completion order, which the scan ignores);
//   * units_write: one thread per list chunk (the index's chunk table, list by
//     list: a list's creation chunks, then its append chunks), so a list of
//     millions of rows is written by thousands of threads: the thread writes
//     its chunk's entry for each query group of the list.
#include "st_internal.cuh"

namespace st {

constexpr int kUnitsBlock = 256;

__global__ void __launch_bounds__(kUnitsBlock)
units_alloc_kernel(SearchArgs a)
{
    const int lane = threadIdx.x & 31;
    const int L = blockIdx.x * kUnitsBlock + threadIdx.x;
    // the index's chunk table is read before waiting for the probe
    const int nch = L < a.nlist ? a.chunk_start[L + 1] - a.chunk_start[L] : 0;
    dep_enter();
    uint32_t u = 0;
    bool dense = false;
    if (L < a.nlist) {
        const int cnt = a.list_cnt[L];
        if (cnt > 0) {
            dense = dense_list(a, cnt) || dense_by_selectivity(a, L, cnt);
            const int qg = dense ? kTcQMax : kQMax;
            u = uint32_t(nch) * uint32_t((cnt + qg - 1) / qg);
        }
    }
    // one warp-wide scan per table (sparse, dense)
    const uint32_t us = dense ? 0u : u, ud = dense ? u : 0u;
    uint32_t is = us, id = ud;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t ts = __shfl_up_sync(0xffffffffu, is, off), td = __shfl_up_sync(0xffffffffu, id, off);
        if (lane >= off) {
            is += ts;
            id += td;
        }
    }
    const uint32_t tot_s = __shfl_sync(0xffffffffu, is, 31), tot_d = __shfl_sync(0xffffffffu, id, 31);
    if (tot_s + tot_d == 0u) return;  // warp-uniform
    uint32_t bs = 0, bd = 0;
    if (lane == 31) {
        if (tot_s) {
            bs = atomicAdd(reinterpret_cast<unsigned int*>(&a.ctl->n_units), tot_s);
            if (uint64_t(bs) + tot_s > uint64_t(a.max_units)) set_error(a.err, kErrUnitTable);
        }
        if (tot_d) {
            bd = atomicAdd(reinterpret_cast<unsigned int*>(&a.ctl->n_dense), tot_d);
            if (uint64_t(bd) + tot_d > uint64_t(a.max_units)) set_error(a.err, kErrUnitTable);
        }
    }
    bs = __shfl_sync(0xffffffffu, bs, 31);
    bd = __shfl_sync(0xffffffffu, bd, 31);
    // a dense list's first unit is stored bit-inverted, so units_write reads
    // the choice made here instead of repeating it
    if (u > 0) a.list_ustart[L] = dense ? ~int32_t(bd + id - ud) : int32_t(bs + is - us);
}

__global__ void __launch_bounds__(kUnitsBlock)
units_write_kernel(SearchArgs a)
{
    const int t = blockIdx.x * kUnitsBlock + threadIdx.x;  // chunk table entry
    // the index's chunk table is read before waiting for the unit blocks
    int4 c = make_int4(0, 0, 0, -1);  // {first row, plane block, rows, list}
    int c0 = 0, nch = 0;
    if (t < a.n_chunks) {
        c = a.chunk_desc[t];
        if (c.w >= 0 && c.w < a.nlist) {
            c0 = a.chunk_start[c.w];
            nch = a.chunk_start[c.w + 1] - c0;
        }
    }
    dep_enter();
    if (t >= a.n_chunks) return;
    const int L = c.w;
    if (L < 0 || L >= a.nlist) {
        set_error(a.err, kErrUnitDecode);
        return;
    }
    const int cnt = a.list_cnt[L];
    if (cnt <= 0) return;
    const int ci = t - c0;
    if (ci < 0 || ci >= nch) {  // the list's block of units does not cover this entry
        set_error(a.err, kErrUnitDecode);
        return;
    }
    int4 unit = make_int4(c.x, c.y, 0, c.z);
    if (c.z < 1 || c.z > kWarpItems || c.x < 0 || int64_t(c.x) + c.z > a.n_rows || c.y < 0 ||
        c.y >= a.n_plane_chunks) {
        // a unit the scan can run but that finds nothing
        set_error(a.err, kErrUnitDecode);
        unit = make_int4(0, 0, 0, 0);
    }
    const int32_t us = a.list_ustart[L];
    const bool dense = us < 0;
    const int64_t base = dense ? int64_t(~us) : int64_t(us);
    const int qg = dense ? kTcQMax : kQMax;
    int4* table = dense ? a.units_tc : a.units;
    const int groups = (cnt + qg - 1) / qg;
    for (int g = 0; g < groups; ++g) {
        const int64_t idx = base + int64_t(g) * nch + ci;
        if (idx < a.max_units)
            table[idx] = make_int4(unit.x, unit.y, L * a.B + g * qg, (unit.w << 16) | min(qg, cnt - g * qg));
    }
}

cudaError_t launch_plan(const SearchArgs& a, int num_sms, cudaStream_t s)
{
    (void)num_sms;
    cudaError_t e = launch_dep(units_alloc_kernel, dim3((a.nlist + kUnitsBlock - 1) / kUnitsBlock), dim3(kUnitsBlock), 0, s, a);
    if (e != cudaSuccess) return e;
    return launch_dep(units_write_kernel, dim3((a.n_chunks + kUnitsBlock - 1) / kUnitsBlock), dim3(kUnitsBlock), 0, s, a);
}

}  // namespace st
