// Host side of the C ABI declared in include/st.h: argument validation, the
// library-owned index copy, stream-ordered scratch, and the kernel sequence
// memset -> probe -> plan -> scan -> select of one search.
#include <algorithm>
#include <cuda.h>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "index_map.h"
#include "st_internal.cuh"

namespace st {
// the union merge (merge.cu)
cudaError_t launch_merge_union(const int64_t* ids, const int32_t* scores, int G, int B, int k, int64_t* out_ids,
                               int32_t* out_scores, cudaStream_t s);
}  // namespace st


// Rows: [0, n) the creation lists (list c: offsets[c] .. offsets[c+1]-1), then
// append chunks of kWarpItems rows, chunk a at rows n + kWarpItems * a, each
// owned by one list and filled in order. An item's id is its row.
struct st_index {
    int device = 0;
    int num_sms = 0;
    int64_t n = 0;                   // creation rows
    int32_t d = 0, nlist = 0, W = 0;
    int8_t* items = nullptr;         // [rows_alloc][d]
    uint64_t* sigs = nullptr;        // [rows_alloc][W]
    int64_t rows_alloc = 0;          // n + kWarpItems * app_cap
    int64_t* offsets = nullptr;      // [nlist+1] creation lists
    int32_t* base_chunk_start = nullptr;  // [nlist+1] first creation chunk (plane block) of each list
    int32_t* chunk_list = nullptr;   // [n_base_chunks] list of each creation chunk
    int32_t n_base_chunks = 0;
    uint32_t* planes = nullptr;      // [n_base_chunks + app_cap][64W][16] signature bit-planes
    int4* chunk_desc = nullptr;      // [desc_cap] chunk table, list by list: {first row, plane block, rows, list}
    int32_t* chunk_start = nullptr;  // [nlist+1] first chunk table entry of each list
    int32_t n_desc = 0, desc_cap = 0;
    int32_t* app_len = nullptr;      // [app_cap] rows filled in each append chunk
    int32_t app_used = 0, app_cap = 0;
    st::rowmap::Layout layout;       // host copy of where every row lives (creation lists, append chunks)
    int8_t* centroids = nullptr;
    uint32_t* err = nullptr;
    std::vector<int64_t> top_prefix;  // [p] = rows in the p largest lists
    std::vector<int64_t> top_chunks;  // [p] = chunk table entries of the p lists with the most
    cudaMemPool_t pool = nullptr;
    int64_t cand_bytes = int64_t(2) << 30;
    int64_t cand_cap_override = 0;
    int64_t id_offset = 0;
    uint32_t* dead = nullptr;        // [ceil(rows_alloc / 32)] deletion bitmap, allocated at the first deletion
    CUtensorMap tmap[2];             // the item rows as a 2-D tensor (TMA tiles of 32 and 128 rows, dense scan)
    bool tmap_ok = false;
    int32_t tc_min_q = st::kTcMinQDefault;  // queries per list from which its units are dense
    uint64_t* sig_sample = nullptr;  // [n_sample][W] signatures of creation rows 0, s, 2s, ... (s = n / kSelSample)
    int32_t n_sample = 0;
};

namespace st {

cudaError_t ensure_smem_attr(const void* func, int bytes)
{
    // kernels whose limit has been raised, per device, with the size set
    struct Entry {
        int dev;
        const void* func;
        int bytes;
    };
    static std::mutex mu;
    static std::vector<Entry> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry& x : done)
        if (x.dev == dev && x.func == func && x.bytes >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    // every large-shared-memory kernel asks for the same (largest) carveout, so
    // an SM need not reconfigure its L1 / shared split between them
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(func, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess) done.push_back(Entry{dev, func, bytes});
    return e;
}

}  // namespace st

namespace {

using st::SearchArgs;

struct DeviceGuard {
    int prev = -1;
    explicit DeviceGuard(int dev)
    {
        if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
        if (prev != dev) cudaSetDevice(dev);
    }
    ~DeviceGuard()
    {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

bool is_device_ptr(const void* p, int device)
{
    if (p == nullptr) return false;
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (attr.type == cudaMemoryTypeManaged) return true;
    return attr.type == cudaMemoryTypeDevice && attr.device == device;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

st_status cuda_status(cudaError_t e)
{
    if (e == cudaSuccess) return ST_OK;
    if (e == cudaErrorMemoryAllocation) return ST_ERR_OOM;
    return ST_ERR_CUDA;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

constexpr int64_t kIdLimit = int64_t(1) << 31;  // ids (with the offset) stay below this

size_t plane_block_bytes(int W) { return size_t(64) * W * 16 * 4; }

st::RowMap row_map(const st_index* idx)
{
    st::RowMap m;
    m.offsets = idx->offsets;
    m.base_chunk_start = idx->base_chunk_start;
    m.nlist = idx->nlist;
    m.n = idx->n;
    m.n_base_chunks = idx->n_base_chunks;
    m.app_len = idx->app_len;
    m.n_app = idx->app_used;
    return m;
}

// The item rows [rows_alloc][d] as 2-D uint8 tensors for TMA tile loads of
// 32 and of 128 rows x d bytes into the dense scan's swizzled layout (128-byte
// swizzle for d = 128, 64-byte for d = 64). Other d have no dense scan.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool make_items_tmap(st_index* idx)
{
    idx->tmap_ok = false;
    if (!st::scan_tc_supported(idx->d)) return false;
    static EncodeTiledFn encode = nullptr;
    if (encode == nullptr) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr) {
            cudaGetLastError();
            return false;
        }
        encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    const cuuint64_t dims[2] = {cuuint64_t(idx->d), cuuint64_t(idx->rows_alloc)};
    const cuuint64_t strides[1] = {cuuint64_t(idx->d)};
    const cuuint32_t estr[2] = {1, 1};
    bool ok = true;
    for (int t = 0; t < 2; ++t) {
        const cuuint32_t box[2] = {cuuint32_t(idx->d), t == 0 ? 32u : 128u};
        const CUresult r = encode(&idx->tmap[t], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, idx->items, dims, strides, box,
                                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                  idx->d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        ok = ok && r == CUDA_SUCCESS;
    }
    idx->tmap_ok = ok;
    return idx->tmap_ok;
}

// Copy the chunk table to the device (a larger array when it outgrew the old
// one: the device is drained first, since earlier searches may still read it).
cudaError_t upload_tables(st_index* idx, const st::rowmap::Tables& t, cudaStream_t stream)
{
    const int32_t nd = int32_t(t.desc.size());
    std::vector<int4> desc(t.desc.size());
    for (size_t i = 0; i < desc.size(); ++i)
        desc[i] = make_int4(t.desc[i].first_row, t.desc[i].plane_block, t.desc[i].rows, t.desc[i].list);
    if (nd > idx->desc_cap || idx->chunk_desc == nullptr) {
        const int32_t cap = std::max<int32_t>(std::max<int32_t>(nd, 1), idx->desc_cap + idx->desc_cap / 2);
        int4* fresh = nullptr;
        cudaError_t e = cudaMalloc(&fresh, size_t(cap) * sizeof(int4));
        if (e != cudaSuccess) return e;
        e = cudaDeviceSynchronize();
        if (e != cudaSuccess) {
            cudaFree(fresh);
            return e;
        }
        cudaFree(idx->chunk_desc);
        idx->chunk_desc = fresh;
        idx->desc_cap = cap;
    }
    cudaError_t e = cudaSuccess;
    if (nd > 0) e = cudaMemcpyAsync(idx->chunk_desc, desc.data(), size_t(nd) * sizeof(int4), cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(idx->chunk_start, t.start.data(), t.start.size() * 4, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);  // the host vectors may go after this
    if (e == cudaSuccess) {
        idx->n_desc = nd;
        idx->top_prefix = t.top_rows;
        idx->top_chunks = t.top_chunks;
    }
    return e;
}

// Room for app_cap append chunks: new item, signature, plane, fill-count and
// deletion arrays, the old contents copied in, the rest zeroed. All or nothing.
st_status grow_rows(st_index* idx, int32_t app_cap, cudaStream_t stream)
{
    if (app_cap <= idx->app_cap) return ST_OK;
    const int64_t rows = idx->n + int64_t(st::kWarpItems) * app_cap;
    if (rows + idx->id_offset >= kIdLimit) return ST_ERR_UNSUPPORTED;
    const int64_t old_rows = idx->rows_alloc;
    const size_t pb = plane_block_bytes(idx->W);
    const size_t old_planes = size_t(idx->n_base_chunks + idx->app_cap) * pb;
    const size_t new_planes = size_t(idx->n_base_chunks + app_cap) * pb;
    const size_t old_words = size_t((old_rows + 31) / 32), new_words = size_t((rows + 31) / 32);
    int8_t* items = nullptr;
    uint64_t* sigs = nullptr;
    uint32_t* planes = nullptr;
    int32_t* app_len = nullptr;
    uint32_t* dead = nullptr;
    auto release = [&]() {
        cudaFree(items);
        cudaFree(sigs);
        cudaFree(planes);
        cudaFree(app_len);
        cudaFree(dead);
        cudaGetLastError();
    };
    if (cudaMalloc(&items, size_t(rows) * idx->d + 256) != cudaSuccess ||
        cudaMalloc(&sigs, size_t(rows) * idx->W * 8 + 256) != cudaSuccess ||
        cudaMalloc(&planes, new_planes) != cudaSuccess ||
        cudaMalloc(&app_len, size_t(app_cap) * 4) != cudaSuccess ||
        (idx->dead && cudaMalloc(&dead, new_words * 4) != cudaSuccess)) {
        release();
        return ST_ERR_OOM;
    }
    cudaError_t e = cudaMemcpyAsync(items, idx->items, size_t(old_rows) * idx->d, cudaMemcpyDeviceToDevice, stream);
    if (e == cudaSuccess) e = cudaMemcpyAsync(sigs, idx->sigs, size_t(old_rows) * idx->W * 8, cudaMemcpyDeviceToDevice, stream);
    if (e == cudaSuccess) e = cudaMemcpyAsync(planes, idx->planes, old_planes, cudaMemcpyDeviceToDevice, stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(reinterpret_cast<char*>(planes) + old_planes, 0, new_planes - old_planes, stream);
    if (e == cudaSuccess && idx->app_cap > 0)
        e = cudaMemcpyAsync(app_len, idx->app_len, size_t(idx->app_cap) * 4, cudaMemcpyDeviceToDevice, stream);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(app_len + idx->app_cap, 0, size_t(app_cap - idx->app_cap) * 4, stream);
    if (e == cudaSuccess && dead) {
        e = cudaMemcpyAsync(dead, idx->dead, old_words * 4, cudaMemcpyDeviceToDevice, stream);
        if (e == cudaSuccess) e = cudaMemsetAsync(dead + old_words, 0, (new_words - old_words) * 4, stream);
    }
    if (e == cudaSuccess) e = cudaDeviceSynchronize();  // also drains searches on other streams
    if (e != cudaSuccess) {
        release();
        return ST_ERR_CUDA;
    }
    std::swap(items, idx->items);
    std::swap(sigs, idx->sigs);
    std::swap(planes, idx->planes);
    std::swap(app_len, idx->app_len);
    if (dead) std::swap(dead, idx->dead);
    release();  // the old arrays
    idx->app_cap = app_cap;
    idx->rows_alloc = rows;
    make_items_tmap(idx);  // the rows moved
    return ST_OK;
}

// Carves one scratch allocation into the per-search arrays. The arrays that
// must start at zero come first, so one memset clears them.
struct ScratchLayout {
    size_t total = 0;
    size_t off_list_cnt, off_cand_cnt, off_elig, off_rng, off_sel_hist, off_sel_cursor, off_ctl, off_tc_hist, zero_bytes;
    size_t off_units_tc, off_qscale, off_qsel;
    size_t off_sel_out, off_sel_tie;
    size_t off_probe, off_probe_keys, off_list_ustart, off_qbits, off_qnbits, off_qlist, off_qmask, off_slot_bits, off_units, off_cand;
    size_t add(size_t bytes)
    {
        const size_t o = total;
        total = align_up(total + bytes, 256);
        return o;
    }
};

int64_t candidate_capacity(const st_index* idx, int32_t B, int32_t P, int32_t k)
{
    if (k > ST_SMALL_K) {
        // the global-memory final top-k has no overflow path: room for the key
        // of every row of the nprobe largest lists, so the scan cannot overflow
        int64_t cap = std::max<int64_t>(idx->top_prefix[std::min<int64_t>(P, idx->nlist)], int64_t(k) + st::kSelectBlock);
        cap += 1;
        return (cap + 31) / 32 * 32;
    }
    int64_t cap = idx->top_prefix[std::min<int64_t>(P, idx->nlist)];
    const int64_t budget = idx->cand_bytes / 8 / B;
    if (cap > budget) cap = budget;
    if (idx->cand_cap_override > 0) cap = idx->cand_cap_override;
    const int64_t floor_cap = int64_t(k) + st::kSelectBlock;
    if (cap < floor_cap) cap = floor_cap;
    cap += 1;  // one spare key so a pairwise copy of an odd count stays inside the buffer
    return (cap + 31) / 32 * 32;  // keeps every query's buffer 256-byte aligned
}

// Units = sum over probed lists of chunks(list) x query groups(list): at most
// every chunk for every group, and at most each query's P lists with the most
// chunks for each query.
int64_t max_units_bound(const st_index* idx, int32_t B, int32_t P)
{
    const int64_t groups = (B + st::kQMax - 1) / st::kQMax;
    const int64_t b1 = int64_t(idx->n_desc) * groups;
    const int64_t b2 = int64_t(B) * idx->top_chunks[std::min<int64_t>(P, idx->nlist)];
    return std::max<int64_t>(1, std::min(b1, b2));
}

st_status search_impl(const st_index* idx, const int8_t* queries, const uint64_t* qmasks, int32_t B,
                      int32_t nprobe, int32_t k, int64_t* out_ids, int32_t* out_scores,
                      const st_search_extras* extras, cudaStream_t stream)
{
    const int64_t cap = candidate_capacity(idx, B, nprobe, k);
    const int64_t max_units = max_units_bound(idx, B, nprobe);
    if (max_units >= (int64_t(1) << 31)) return ST_ERR_UNSUPPORTED;
    if (int64_t(idx->nlist) * B >= (int64_t(1) << 31)) return ST_ERR_UNSUPPORTED;
    const size_t nl4 = size_t(idx->nlist + 3) / 4 * 4;
    const size_t slots = size_t(idx->nlist) * size_t(B);

    ScratchLayout L;
    L.off_list_cnt = L.add(nl4 * 4);
    L.off_cand_cnt = L.add(size_t(B) * st::kCntStride * 4);
    L.off_elig = L.add(size_t(B) * st::kCntStride * 4);
    L.off_rng = L.add(size_t(B) * st::kCntStride * 4);
    // the chunked final top-k's per-query histograms (the cluster final top-k
    // has no use for them, so they are not cleared then)
    const size_t sel_bytes = st::select_reads_bins(B, k) ? 0 : size_t(B) * st::kSelBins * 4;
    L.off_sel_hist = L.add(sel_bytes);
    L.off_sel_cursor = L.add(sel_bytes);
    L.off_ctl = L.add(sizeof(st::PlanCtl));
    const int tc_min_q = (idx->tmap_ok && idx->tc_min_q > 0 && B >= idx->tc_min_q) ? idx->tc_min_q : 0;
    L.off_tc_hist = L.add(size_t(B) * st::kTcBins * 4);
    L.zero_bytes = L.total;
    L.off_probe = L.add(size_t(B) * nprobe * 4);
    L.off_probe_keys = L.add(size_t(B) * size_t(st::probe_keys_ld(idx->nlist)) * 8);
    L.off_list_ustart = L.add(nl4 * 4);
    const int n_alt = 1 + (extras ? extras->n_or : 0);  // masks per query
    L.off_qbits = L.add(size_t(B) * n_alt * st::kMaskBitsMax);
    L.off_qnbits = L.add(size_t(B) * n_alt * 4);
    L.off_qlist = L.add(slots * 4);
    L.off_qmask = L.add(slots * 16);
    L.off_slot_bits = L.add(slots * st::kSlotBits);
    L.off_units = L.add(size_t(max_units) * 16);
    L.off_units_tc = L.add(tc_min_q ? size_t(max_units) * 16 : 0);
    L.off_qscale = L.add(size_t(B) * 8);
    // lists of fewer than tc_min_q queries may go dense by their queries'
    // selectivity once the batch is large enough to fill the dense pipeline
    // (tc_min_q = 1 already sends every list there)
    const bool sel_route = tc_min_q > 1 && idx->n_sample > 0 && int64_t(B) * nprobe >= st::kSelMinProbes;
    L.off_qsel = L.add(sel_route ? size_t(B) * 2 : 0);
    L.off_cand = L.add(size_t(B) * size_t(cap) * 8);
    L.off_sel_out = L.add(size_t(B) * size_t(k) * 8);
    L.off_sel_tie = L.add(size_t(B) * st::kSelTieCap * 8);

    unsigned char* base = nullptr;
    cudaError_t e = cudaMallocFromPoolAsync(reinterpret_cast<void**>(&base), L.total, idx->pool, stream);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return e == cudaErrorMemoryAllocation ? ST_ERR_OOM : ST_ERR_CUDA;
    }

    SearchArgs a;
    std::memset(&a, 0, sizeof(a));
    a.items = idx->items;
    a.sigs = idx->sigs;
    a.planes = idx->planes;
    a.chunk_desc = idx->chunk_desc;
    a.chunk_start = idx->chunk_start;
    a.n_chunks = idx->n_desc;
    a.n_plane_chunks = idx->n_base_chunks + idx->app_cap;
    a.n_rows = idx->rows_alloc;
    a.centroids = idx->centroids;
    a.d = idx->d;
    a.nlist = idx->nlist;
    a.W = idx->W;
    a.queries = queries;
    a.qmasks = qmasks;
    a.B = B;
    a.P = nprobe;
    a.k = k;
    a.out_ids = out_ids;
    a.out_scores = out_scores;
    a.out_eligible = extras ? extras->eligible : nullptr;
    a.out_cands = extras ? extras->candidates : nullptr;
    a.list_cnt = reinterpret_cast<int32_t*>(base + L.off_list_cnt);
    a.cand_cnt = reinterpret_cast<uint32_t*>(base + L.off_cand_cnt);
    a.eligible_cnt = reinterpret_cast<unsigned long long*>(base + L.off_elig);
    a.score_rng = reinterpret_cast<uint32_t*>(base + L.off_rng);
    a.sel_hist = reinterpret_cast<uint32_t*>(base + L.off_sel_hist);
    a.sel_cursor = reinterpret_cast<uint32_t*>(base + L.off_sel_cursor);
    a.ctl = reinterpret_cast<st::PlanCtl*>(base + L.off_ctl);
    a.probe = reinterpret_cast<int32_t*>(base + L.off_probe);
    a.probe_keys = reinterpret_cast<uint64_t*>(base + L.off_probe_keys);
    a.list_ustart = reinterpret_cast<int32_t*>(base + L.off_list_ustart);
    a.qbits = reinterpret_cast<uint8_t*>(base + L.off_qbits);
    a.qnbits = reinterpret_cast<int32_t*>(base + L.off_qnbits);
    a.qlist = reinterpret_cast<int32_t*>(base + L.off_qlist);
    a.qmask_slot = reinterpret_cast<uint64_t*>(base + L.off_qmask);
    a.slot_bits = reinterpret_cast<uint8_t*>(base + L.off_slot_bits);
    a.units = reinterpret_cast<int4*>(base + L.off_units);
    a.max_units = int32_t(max_units);
    a.tc_min_q = tc_min_q;
    if (tc_min_q) a.units_tc = reinterpret_cast<int4*>(base + L.off_units_tc);
    if (sel_route) {
        a.sig_sample = idx->sig_sample;
        a.n_sample = idx->n_sample;
        a.qsel = reinterpret_cast<uint16_t*>(base + L.off_qsel);
    }
    a.qscale = reinterpret_cast<int2*>(base + L.off_qscale);
    a.qhist = reinterpret_cast<uint32_t*>(base + L.off_tc_hist);
    a.count_bins = st::select_reads_bins(B, k) ? 1 : 0;
    a.cand = reinterpret_cast<uint64_t*>(base + L.off_cand);
    a.cap = cap;
    a.id_offset = idx->id_offset;
    a.dead = idx->dead;
    a.qexclude = extras ? extras->exclude_masks : nullptr;
    a.n_or = extras ? extras->n_or : 0;
    a.or_masks = a.n_or > 0 ? extras->or_masks : nullptr;
    a.sel_out = reinterpret_cast<uint64_t*>(base + L.off_sel_out);
    a.sel_tie = reinterpret_cast<uint64_t*>(base + L.off_sel_tie);
    a.err = idx->err;

    auto mark = [&](int i) {
        if (e == cudaSuccess && extras && extras->stage_events[i]) e = cudaEventRecord(extras->stage_events[i], stream);
    };
    e = cudaMemsetAsync(base, 0, L.zero_bytes, stream);
    mark(0);
    if (e == cudaSuccess) e = st::launch_probe_search(a, idx->num_sms, stream);
    mark(1);
    if (e == cudaSuccess) e = st::launch_plan(a, idx->num_sms, stream);
    mark(2);
    if (e == cudaSuccess) e = st::launch_scan(a, idx->num_sms, stream);
    if (e == cudaSuccess && tc_min_q) e = st::launch_scan_tc(a, idx->tmap, idx->num_sms, stream);
    mark(3);
    if (e == cudaSuccess) e = st::launch_select(a, idx->num_sms, stream);
    mark(4);
    if (e == cudaSuccess && extras && extras->probe)
        e = cudaMemcpyAsync(extras->probe, a.probe, size_t(B) * nprobe * 4, cudaMemcpyDeviceToDevice, stream);
    cudaError_t ef = cudaFreeAsync(base, stream);
    if (e == cudaSuccess) e = ef;
    return cuda_status(e);
}

st_status check_search_args(const st_index* idx, int32_t B, int32_t nprobe, int32_t k)
{
    if (idx == nullptr) return ST_ERR_INVALID_ARG;
    if (B < 1 || k < 1 || nprobe < 1 || nprobe > idx->nlist) return ST_ERR_INVALID_ARG;
    if (k > ST_MAX_K || nprobe > ST_MAX_NPROBE || B > ST_MAX_B) return ST_ERR_UNSUPPORTED;
    if (int64_t(B) * nprobe >= (int64_t(1) << 31)) return ST_ERR_UNSUPPORTED;
    return ST_OK;
}

}  // namespace

extern "C" {

const char* st_status_string(st_status s)
{
    switch (s) {
    case ST_OK: return "ok";
    case ST_ERR_INVALID_ARG: return "invalid argument";
    case ST_ERR_UNSUPPORTED: return "unsupported size";
    case ST_ERR_OOM: return "out of device memory";
    case ST_ERR_CUDA: return "CUDA error";
    case ST_ERR_DEVICE: return "device-side error recorded by a kernel";
    case ST_ERR_SCRATCH_LIMIT: return "request needs more than the fixed scratch of the allocation-free call";
    }
    return "unknown status";
}

st_status st_index_create(const int8_t* items, const uint64_t* sigs, const int64_t* list_offsets,
                          const int8_t* centroids, int64_t n, int32_t d, int32_t nlist,
                          int32_t sig_words, cudaStream_t stream, st_index** out)
{
    if (out == nullptr) return ST_ERR_INVALID_ARG;
    *out = nullptr;
    if (!items || !sigs || !list_offsets || !centroids) return ST_ERR_INVALID_ARG;
    if (n < 1 || nlist < 1 || d < 1) return ST_ERR_INVALID_ARG;
    if (d % 16 != 0 || d > ST_MAX_D || (sig_words != 1 && sig_words != 2)) return ST_ERR_UNSUPPORTED;
    if (n >= (int64_t(1) << 31)) return ST_ERR_UNSUPPORTED;

    st_index* idx = new (std::nothrow) st_index();
    if (!idx) return ST_ERR_OOM;
    auto fail = [&](st_status s) {
        st_index_destroy(idx);
        return s;
    };
    cudaError_t e = cudaGetDevice(&idx->device);
    if (e != cudaSuccess) return fail(ST_ERR_CUDA);
    e = cudaDeviceGetAttribute(&idx->num_sms, cudaDevAttrMultiProcessorCount, idx->device);
    if (e != cudaSuccess) return fail(ST_ERR_CUDA);
    idx->n = n;
    idx->d = d;
    idx->nlist = nlist;
    idx->W = sig_words;

    // offsets: validate on the host
    std::vector<int64_t> off(size_t(nlist) + 1);
    e = cudaMemcpyAsync(off.data(), list_offsets, off.size() * 8, cudaMemcpyDefault, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(ST_ERR_INVALID_ARG);
    }
    if (off[0] != 0 || off[nlist] != n) return fail(ST_ERR_INVALID_ARG);
    for (int32_t c = 0; c < nlist; ++c)
        if (off[c + 1] < off[c]) return fail(ST_ERR_INVALID_ARG);
    idx->rows_alloc = n;

    // library-owned copies (a little slack past the end of the row arrays)
    const size_t items_bytes = size_t(n) * d, sig_bytes = size_t(n) * sig_words * 8;
    if (cudaMalloc(&idx->items, items_bytes + 256) != cudaSuccess ||
        cudaMalloc(&idx->sigs, sig_bytes + 256) != cudaSuccess ||
        cudaMalloc(&idx->offsets, off.size() * 8) != cudaSuccess ||
        cudaMalloc(&idx->centroids, size_t(nlist) * d + 256) != cudaSuccess ||
        cudaMalloc(&idx->base_chunk_start, size_t(nlist + 1) * 4) != cudaSuccess ||
        cudaMalloc(&idx->chunk_start, size_t(nlist + 1) * 4) != cudaSuccess ||
        cudaMalloc(&idx->err, 256) != cudaSuccess) {
        cudaGetLastError();
        return fail(ST_ERR_OOM);
    }
    e = cudaMemcpyAsync(idx->items, items, items_bytes, cudaMemcpyDefault, stream);
    if (e == cudaSuccess) e = cudaMemcpyAsync(idx->sigs, sigs, sig_bytes, cudaMemcpyDefault, stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(idx->offsets, off.data(), off.size() * 8, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(idx->centroids, centroids, size_t(nlist) * d, cudaMemcpyDefault, stream);
    // creation chunks: list c owns plane blocks cstart[c] .. cstart[c+1]-1
    idx->layout = st::rowmap::make_layout(off, st::kWarpItems);
    const std::vector<int32_t>& cstart = idx->layout.base_cstart;
    idx->n_base_chunks = idx->layout.n_base_chunks;
    std::vector<int32_t> clist(size_t(idx->n_base_chunks > 0 ? idx->n_base_chunks : 1), 0);
    for (int32_t c = 0; c < nlist; ++c)
        for (int32_t t = cstart[c]; t < cstart[c + 1]; ++t) clist[t] = c;
    if (cudaMalloc(&idx->chunk_list, clist.size() * 4) != cudaSuccess) {
        cudaGetLastError();
        return fail(ST_ERR_OOM);
    }
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(idx->base_chunk_start, cstart.data(), cstart.size() * 4, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = cudaMemcpyAsync(idx->chunk_list, clist.data(), clist.size() * 4, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) {
        const size_t pbytes = size_t(idx->n_base_chunks > 0 ? idx->n_base_chunks : 1) * plane_block_bytes(sig_words);
        if (cudaMalloc(&idx->planes, pbytes) != cudaSuccess) {
            cudaGetLastError();
            return fail(ST_ERR_OOM);
        }
        e = st::launch_build_planes(idx->sigs, idx->offsets, idx->base_chunk_start, idx->chunk_list,
                                    idx->n_base_chunks, sig_words, idx->planes, stream);
    }
    // a fixed sample of the rows' signatures, for each search's selectivity
    // estimates (they choose between the two scans only; not updated when
    // rows are inserted, updated or deleted)
    if (e == cudaSuccess) {
        const int64_t stride = std::max<int64_t>(1, n / st::kSelSample);
        idx->n_sample = int32_t(std::min<int64_t>(st::kSelSample, (n + stride - 1) / stride));
        if (cudaMalloc(&idx->sig_sample, size_t(idx->n_sample) * sig_words * 8) != cudaSuccess) {
            cudaGetLastError();
            return fail(ST_ERR_OOM);
        }
        e = cudaMemcpy2DAsync(idx->sig_sample, size_t(sig_words) * 8, idx->sigs, size_t(stride) * sig_words * 8,
                              size_t(sig_words) * 8, size_t(idx->n_sample), cudaMemcpyDeviceToDevice, stream);
    }
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess) make_items_tmap(idx);
    if (e == cudaSuccess) e = upload_tables(idx, st::rowmap::build_tables(idx->layout), stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(idx->err, 0, 256, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(e == cudaErrorInvalidValue ? ST_ERR_INVALID_ARG
                    : e == cudaErrorMemoryAllocation ? ST_ERR_OOM : ST_ERR_CUDA);
    }

    cudaMemPoolProps props;
    std::memset(&props, 0, sizeof(props));
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = idx->device;
    if (cudaMemPoolCreate(&idx->pool, &props) != cudaSuccess) {
        cudaGetLastError();
        idx->pool = nullptr;
        return fail(ST_ERR_CUDA);
    }
    uint64_t keep = ~uint64_t(0);
    cudaMemPoolSetAttribute(idx->pool, cudaMemPoolAttrReleaseThreshold, &keep);
    *out = idx;
    return ST_OK;
}

st_status st_search_ex(const st_index* idx, const int8_t* queries, const uint64_t* qmasks, int32_t B,
                       int32_t nprobe, int32_t k, int64_t* out_ids, int32_t* out_scores,
                       const st_search_extras* extras, cudaStream_t stream)
{
    st_status s = check_search_args(idx, B, nprobe, k);
    if (s != ST_OK) return s;
    DeviceGuard g(idx->device);
    if (!is_device_ptr(queries, idx->device) || !is_device_ptr(qmasks, idx->device) ||
        !is_device_ptr(out_ids, idx->device) || !is_device_ptr(out_scores, idx->device))
        return ST_ERR_INVALID_ARG;
    if (!aligned(queries, 16) || !aligned(qmasks, 8) || !aligned(out_ids, 8) || !aligned(out_scores, 4))
        return ST_ERR_INVALID_ARG;
    if (extras) {
        if (extras->eligible && (!is_device_ptr(extras->eligible, idx->device) || !aligned(extras->eligible, 8)))
            return ST_ERR_INVALID_ARG;
        if (extras->probe && (!is_device_ptr(extras->probe, idx->device) || !aligned(extras->probe, 4)))
            return ST_ERR_INVALID_ARG;
        if (extras->exclude_masks &&
            (!is_device_ptr(extras->exclude_masks, idx->device) || !aligned(extras->exclude_masks, 8)))
            return ST_ERR_INVALID_ARG;
        if (extras->n_or < 0 || extras->n_or > ST_MAX_OR ||
            (extras->n_or > 0 && (!is_device_ptr(extras->or_masks, idx->device) || !aligned(extras->or_masks, 8))))
            return ST_ERR_INVALID_ARG;
    }
    return search_impl(idx, queries, qmasks, B, nprobe, k, out_ids, out_scores, extras, stream);
}

st_status st_search(const st_index* idx, const int8_t* queries, const uint64_t* qmasks, int32_t B,
                    int32_t nprobe, int32_t k, int64_t* out_ids, int32_t* out_scores, cudaStream_t stream)
{
    return st_search_ex(idx, queries, qmasks, B, nprobe, k, out_ids, out_scores, nullptr, stream);
}

}  // extern "C"

namespace {

bool is_pinned_host(const void* p)
{
    if (p == nullptr) return false;
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return attr.type == cudaMemoryTypeHost;
}

// Host-buffer search: stage the inputs in pool memory, search, copy the
// outputs back; optionally wait for the stream.
st_status search_host_impl(const st_index* idx, const int8_t* queries, const uint64_t* qmasks, int32_t B,
                           int32_t nprobe, int32_t k, int64_t* out_ids, int32_t* out_scores, cudaStream_t stream,
                           bool wait)
{
    const size_t qb = align_up(size_t(B) * idx->d, 256), mb = align_up(size_t(B) * idx->W * 8, 256);
    const size_t ib = align_up(size_t(B) * k * 8, 256), sb = align_up(size_t(B) * k * 4, 256);
    unsigned char* buf = nullptr;
    cudaError_t e = cudaMallocFromPoolAsync(reinterpret_cast<void**>(&buf), qb + mb + ib + sb, idx->pool, stream);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return e == cudaErrorMemoryAllocation ? ST_ERR_OOM : ST_ERR_CUDA;
    }
    int8_t* dq = reinterpret_cast<int8_t*>(buf);
    uint64_t* dm = reinterpret_cast<uint64_t*>(buf + qb);
    int64_t* dids = reinterpret_cast<int64_t*>(buf + qb + mb);
    int32_t* dsc = reinterpret_cast<int32_t*>(buf + qb + mb + ib);
    e = cudaMemcpyAsync(dq, queries, size_t(B) * idx->d, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = cudaMemcpyAsync(dm, qmasks, size_t(B) * idx->W * 8, cudaMemcpyHostToDevice, stream);
    st_status rs = ST_OK;
    if (e == cudaSuccess) {
        rs = search_impl(idx, dq, dm, B, nprobe, k, dids, dsc, nullptr, stream);
        if (rs == ST_OK) {
            e = cudaMemcpyAsync(out_ids, dids, size_t(B) * k * 8, cudaMemcpyDeviceToHost, stream);
            if (e == cudaSuccess) e = cudaMemcpyAsync(out_scores, dsc, size_t(B) * k * 4, cudaMemcpyDeviceToHost, stream);
        }
    }
    cudaError_t ef = cudaFreeAsync(buf, stream);
    cudaError_t es = wait ? cudaStreamSynchronize(stream) : cudaSuccess;
    if (rs != ST_OK) return rs;
    if (e == cudaSuccess) e = ef;
    if (e == cudaSuccess) e = es;
    return cuda_status(e);
}

}  // namespace

extern "C" {

st_status st_search_host(const st_index* idx, const int8_t* queries, const uint64_t* qmasks, int32_t B,
                         int32_t nprobe, int32_t k, int64_t* out_ids, int32_t* out_scores,
                         cudaStream_t stream)
{
    st_status s = check_search_args(idx, B, nprobe, k);
    if (s != ST_OK) return s;
    if (!queries || !qmasks || !out_ids || !out_scores) return ST_ERR_INVALID_ARG;
    DeviceGuard g(idx->device);
    return search_host_impl(idx, queries, qmasks, B, nprobe, k, out_ids, out_scores, stream, true);
}

st_status st_search_host_async(const st_index* idx, const int8_t* queries, const uint64_t* qmasks, int32_t B,
                               int32_t nprobe, int32_t k, int64_t* out_ids, int32_t* out_scores,
                               cudaStream_t stream)
{
    st_status s = check_search_args(idx, B, nprobe, k);
    if (s != ST_OK) return s;
    DeviceGuard g(idx->device);
    if (!is_pinned_host(queries) || !is_pinned_host(qmasks) || !is_pinned_host(out_ids) ||
        !is_pinned_host(out_scores))
        return ST_ERR_INVALID_ARG;
    return search_host_impl(idx, queries, qmasks, B, nprobe, k, out_ids, out_scores, stream, false);
}

st_status st_probe_noalloc(const st_index* idx, const int8_t* queries, int32_t B, int32_t nprobe,
                           int32_t* out_probe, cudaStream_t stream)
{
    if (idx == nullptr) return ST_ERR_INVALID_ARG;
    if (B < 1 || nprobe < 1 || nprobe > idx->nlist) return ST_ERR_INVALID_ARG;
    if (nprobe > ST_MAX_NPROBE || int64_t(B) * nprobe >= (int64_t(1) << 31)) return ST_ERR_UNSUPPORTED;
    DeviceGuard g(idx->device);
    if (!is_device_ptr(queries, idx->device) || !is_device_ptr(out_probe, idx->device)) return ST_ERR_INVALID_ARG;
    if (!aligned(queries, 16) || !aligned(out_probe, 4)) return ST_ERR_INVALID_ARG;
    SearchArgs a;
    std::memset(&a, 0, sizeof(a));
    a.centroids = idx->centroids;
    a.d = idx->d;
    a.nlist = idx->nlist;
    a.W = idx->W;
    a.queries = queries;
    a.B = B;
    a.P = nprobe;
    a.probe = out_probe;
    a.err = idx->err;
    const int S = st::probe_slices(a, idx->num_sms);
    const bool keys_in_smem = (idx->nlist + S - 1) / S + 1 <= st::kProbeSmemKeys;
    if (st::probe_noalloc_scratch_bytes(B, S, nprobe, idx->nlist, keys_in_smem) > ST_PROBE_NOALLOC_SCRATCH_BYTES)
        return ST_ERR_SCRATCH_LIMIT;
    // any non-null value asks for the keys in global scratch; the launcher
    // points it into the fixed array
    a.probe_keys = keys_in_smem ? nullptr : reinterpret_cast<uint64_t*>(uintptr_t(1));
    return cuda_status(st::launch_probe_noalloc(a, S, stream));
}

st_status st_merge_topk(const int64_t* ids, const int32_t* scores, int32_t G, int32_t B, int32_t k,
                        int64_t* out_ids, int32_t* out_scores, cudaStream_t stream)
{
    if (G < 1 || B < 1 || k < 1) return ST_ERR_INVALID_ARG;
    if (k > ST_SMALL_K || int64_t(G) * k > ST_MERGE_MAX_KEYS) return ST_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ST_ERR_CUDA;
    if (!is_device_ptr(ids, dev) || !is_device_ptr(scores, dev) || !is_device_ptr(out_ids, dev) ||
        !is_device_ptr(out_scores, dev))
        return ST_ERR_INVALID_ARG;
    if (!aligned(ids, 8) || !aligned(scores, 4) || !aligned(out_ids, 8) || !aligned(out_scores, 4))
        return ST_ERR_INVALID_ARG;
    return cuda_status(st::launch_merge(ids, scores, G, B, k, out_ids, out_scores, stream));
}

st_status st_merge_topk_union(const int64_t* ids, const int32_t* scores, int32_t G, int32_t B, int32_t k,
                              int64_t* out_ids, int32_t* out_scores, cudaStream_t stream)
{
    if (G < 1 || B < 1 || k < 1) return ST_ERR_INVALID_ARG;
    if (k > ST_SMALL_K || int64_t(G) * k > ST_MERGE_MAX_KEYS) return ST_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ST_ERR_CUDA;
    if (!is_device_ptr(ids, dev) || !is_device_ptr(scores, dev) || !is_device_ptr(out_ids, dev) ||
        !is_device_ptr(out_scores, dev))
        return ST_ERR_INVALID_ARG;
    if (!aligned(ids, 8) || !aligned(scores, 4) || !aligned(out_ids, 8) || !aligned(out_scores, 4))
        return ST_ERR_INVALID_ARG;
    return cuda_status(st::launch_merge_union(ids, scores, G, B, k, out_ids, out_scores, stream));
}

st_status st_merge_check(cudaStream_t stream)
{
    if (cudaStreamSynchronize(stream) != cudaSuccess) return ST_ERR_CUDA;
    uint32_t word = 0;
    if (st::merge_error_word(&word, true) != cudaSuccess) return ST_ERR_CUDA;
    return word ? ST_ERR_DEVICE : ST_OK;
}

st_status st_index_update(st_index* idx, const int64_t* ids, const int8_t* items, const uint64_t* sigs,
                          int64_t m, cudaStream_t stream)
{
    if (idx == nullptr || m < 0 || (items == nullptr && sigs == nullptr)) return ST_ERR_INVALID_ARG;
    if (m == 0) return ST_OK;
    DeviceGuard g(idx->device);
    if (!is_device_ptr(ids, idx->device) || !aligned(ids, 8)) return ST_ERR_INVALID_ARG;
    if (items && (!is_device_ptr(items, idx->device) || !aligned(items, 16))) return ST_ERR_INVALID_ARG;
    if (sigs && (!is_device_ptr(sigs, idx->device) || !aligned(sigs, 8))) return ST_ERR_INVALID_ARG;
    return cuda_status(st::launch_update(idx->items, idx->sigs, idx->planes, row_map(idx), idx->d, idx->W, ids,
                                         items, sigs, m, idx->err, stream));
}

st_status st_index_delete(st_index* idx, const int64_t* ids, int64_t m, cudaStream_t stream)
{
    if (idx == nullptr || m < 0) return ST_ERR_INVALID_ARG;
    if (m == 0) return ST_OK;
    DeviceGuard g(idx->device);
    if (!is_device_ptr(ids, idx->device) || !aligned(ids, 8)) return ST_ERR_INVALID_ARG;
    if (idx->dead == nullptr) {
        const size_t bytes = size_t((idx->rows_alloc + 31) / 32) * 4;
        if (cudaMalloc(&idx->dead, bytes) != cudaSuccess) {
            cudaGetLastError();
            idx->dead = nullptr;
            return ST_ERR_OOM;
        }
        if (cudaMemsetAsync(idx->dead, 0, bytes, stream) != cudaSuccess) return ST_ERR_CUDA;
    }
    return cuda_status(st::launch_delete(idx->dead, row_map(idx), ids, m, idx->err, stream));
}

st_status st_index_check(const st_index* idx, cudaStream_t stream)
{
    if (idx == nullptr) return ST_ERR_INVALID_ARG;
    DeviceGuard g(idx->device);
    uint32_t word = 0;
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess) e = cudaMemcpy(&word, idx->err, 4, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return ST_ERR_CUDA;
    if (word != 0) {
        cudaMemset(idx->err, 0, 4);
        return ST_ERR_DEVICE;
    }
    return ST_OK;
}

st_status st_index_set_option(st_index* idx, st_option opt, int64_t value)
{
    if (idx == nullptr || value < 0) return ST_ERR_INVALID_ARG;
    switch (opt) {
    case ST_OPT_CANDIDATE_BYTES:
        idx->cand_bytes = value > 0 ? value : (int64_t(2) << 30);
        return ST_OK;
    case ST_OPT_CANDIDATE_CAPACITY:
        idx->cand_cap_override = value;
        return ST_OK;
    case ST_OPT_ID_OFFSET:
        if (value >= kIdLimit || value + idx->rows_alloc >= kIdLimit) return ST_ERR_UNSUPPORTED;
        idx->id_offset = value;
        return ST_OK;
    case ST_OPT_DENSE_MIN_QUERIES:
        if (value > ST_MAX_B) return ST_ERR_INVALID_ARG;
        idx->tc_min_q = int32_t(value);
        return ST_OK;
    case ST_OPT_INSERT_RESERVE: {
        if (value == 0) return ST_OK;
        const int64_t chunks = (value + st::kWarpItems - 1) / st::kWarpItems;
        if (idx->n + (idx->app_used + chunks) * st::kWarpItems + idx->id_offset >= kIdLimit) return ST_ERR_UNSUPPORTED;
        DeviceGuard g(idx->device);
        return grow_rows(idx, int32_t(idx->app_used + chunks), nullptr);
    }
    }
    return ST_ERR_INVALID_ARG;
}

st_status st_index_insert(st_index* idx, const int32_t* lists, const int8_t* items, const uint64_t* sigs,
                          int64_t m, int64_t* out_ids, cudaStream_t stream)
{
    if (idx == nullptr || m < 0) return ST_ERR_INVALID_ARG;
    if (m == 0) return ST_OK;
    if (lists == nullptr || out_ids == nullptr) return ST_ERR_INVALID_ARG;
    DeviceGuard g(idx->device);
    if (!is_device_ptr(items, idx->device) || !aligned(items, 16) || !is_device_ptr(sigs, idx->device) ||
        !aligned(sigs, 8))
        return ST_ERR_INVALID_ARG;
    for (int64_t j = 0; j < m; ++j)
        if (lists[j] < 0 || lists[j] >= idx->nlist) return ST_ERR_INVALID_ARG;
    if (m >= kIdLimit) return ST_ERR_UNSUPPORTED;

    // place the items on the host: each fills its list's last append chunk,
    // then a fresh chunk (on a copy of the layout, kept only on success)
    st::rowmap::Layout lay = idx->layout;
    std::vector<int64_t> ids;
    if (!st::rowmap::place(lay, lists, m, idx->id_offset, kIdLimit, ids)) return ST_ERR_UNSUPPORTED;
    const int64_t used = lay.app_used();
    if (used > idx->app_cap) {
        // at least double the append room, within the id limit
        int64_t cap = std::max<int64_t>(used, 2 * int64_t(idx->app_cap));
        const int64_t cap_max = (kIdLimit - 1 - idx->id_offset - idx->n) / st::kWarpItems;
        cap = std::min(cap, cap_max);
        const st_status gs = grow_rows(idx, int32_t(cap), stream);
        if (gs != ST_OK) return gs;
    }
    const st::rowmap::Tables t = st::rowmap::build_tables(lay);

    int64_t* dids = nullptr;
    cudaError_t e = cudaMallocFromPoolAsync(reinterpret_cast<void**>(&dids), size_t(m) * 8, idx->pool, stream);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return e == cudaErrorMemoryAllocation ? ST_ERR_OOM : ST_ERR_CUDA;
    }
    e = cudaMemcpyAsync(dids, ids.data(), size_t(m) * 8, cudaMemcpyHostToDevice, stream);
    // the fill counts cover the new rows before the rows are written
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(idx->app_len, lay.app_len.data(), lay.app_len.size() * 4, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) {
        st::RowMap map = row_map(idx);
        map.n_app = int32_t(used);
        e = st::launch_update(idx->items, idx->sigs, idx->planes, map, idx->d, idx->W, dids, items, sigs, m, idx->err,
                              stream);
    }
    // the chunk table last: searches enqueued after this call see the new rows
    if (e == cudaSuccess) e = upload_tables(idx, t, stream);
    cudaError_t ef = cudaFreeAsync(dids, stream);
    if (e == cudaSuccess) e = ef;
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return e == cudaErrorMemoryAllocation ? ST_ERR_OOM : ST_ERR_CUDA;
    }
    idx->layout = std::move(lay);
    idx->app_used = int32_t(used);
    std::memcpy(out_ids, ids.data(), size_t(m) * 8);
    return ST_OK;
}

void st_index_destroy(st_index* idx)
{
    if (idx == nullptr) return;
    {
        DeviceGuard g(idx->device);
        cudaDeviceSynchronize();
        cudaFree(idx->items);
        cudaFree(idx->sigs);
        cudaFree(idx->offsets);
        cudaFree(idx->centroids);
        cudaFree(idx->chunk_start);
        cudaFree(idx->base_chunk_start);
        cudaFree(idx->chunk_desc);
        cudaFree(idx->app_len);
        cudaFree(idx->chunk_list);
        cudaFree(idx->planes);
        cudaFree(idx->err);
        cudaFree(idx->dead);
        cudaFree(idx->sig_sample);
        if (idx->pool) cudaMemPoolDestroy(idx->pool);
        cudaGetLastError();
    }
    delete idx;
}

}  // extern "C"
