// Plan: cut every probed list into work units of kWarpItems rows x a group of
// the queries probing it, so the scan reads each probed list once per batch
// however many queries probe it. One self-contained 16-byte entry per unit:
// {first row, chunk, first query slot, rows << 16 | queries}. Lists probed by
// fewer than tc_min_q queries get groups of up to kQMax queries, scanned by
// one warp each (scan.cu); lists probed by more get groups of up to kTcQMax
// queries in a second table, scanned as dense tensor-core tiles (scan_tc.cu).
//
// The probe kernel already filed each query into the slot row of every list it
// chose (slots L*B .. L*B + count-1), so no scan over lists or scatter of pairs
// is needed here. The last probe CTA to finish sizes every list's block of
// the unit tables (size_units, one CTA: a scan of the lists' unit counts), and
// one small balanced kernel writes the entries:
//   * units_write: one thread per list chunk (the index's chunk table, list by
//     list: a list's creation chunks, then its append chunks), so a list of
//     millions of rows is written by thousands of threads: the thread writes
//     its chunk's entry for each query group of the list.
#include "st_internal.cuh"

namespace st {

constexpr int kUnitsBlock = 256;


__global__ void __launch_bounds__(kUnitsBlock)
units_write_kernel(SearchArgs a)
{
    dep_enter();
    const int t = blockIdx.x * kUnitsBlock + threadIdx.x;  // chunk table entry
    if (t >= a.n_chunks) return;
    const int4 c = a.chunk_desc[t];  // {first row, plane block, rows, list}
    const int L = c.w;
    if (L < 0 || L >= a.nlist) {
        set_error(a.err, kErrUnitDecode);
        return;
    }
    const int cnt = a.list_cnt[L];
    if (cnt <= 0) return;
    const int c0 = a.chunk_start[L];
    const int nch = a.chunk_start[L + 1] - c0;
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
    const int64_t base = a.list_ustart[L];
    const bool dense = dense_list(a, cnt);
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
    return launch_dep(units_write_kernel, dim3((a.n_chunks + kUnitsBlock - 1) / kUnitsBlock), dim3(kUnitsBlock), 0, s, a);
}

}  // namespace st
