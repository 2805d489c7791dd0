// Host-side bookkeeping of where an index's rows live: the creation lists,
// the append chunks that insertions fill, and the chunk table the search walks
// list by list. Plain C++ with no CUDA types, so the same code is compiled into
// the library and into a host-only unit test.
//
// Rows [0, n) are the creation lists (list c: off[c] .. off[c+1]-1, cut into
// chunks of `chunk` rows whose plane blocks start at base_cstart[c]). Append
// chunk a covers rows n + chunk * a .. n + chunk * (a + 1) - 1, belongs to one
// list, is filled in insertion order, and has plane block n_base_chunks + a.
// An item's id is its row.
#pragma once

#include <algorithm>
#include <cstdint>
#include <functional>
#include <vector>

namespace st {
namespace rowmap {

struct Layout {
    int64_t n = 0;                               // creation rows
    int32_t chunk = 0;                           // rows per chunk
    int32_t n_base_chunks = 0;                   // chunks of the creation lists
    std::vector<int64_t> off;                    // [nlist+1] creation offsets
    std::vector<int32_t> base_cstart;            // [nlist+1] first creation chunk of each list
    std::vector<std::vector<int32_t>> list_app;  // append chunks of each list, in fill order
    std::vector<int32_t> app_len;                // rows filled in each append chunk handed out

    int32_t nlist() const { return int32_t(off.size()) - 1; }
    int32_t app_used() const { return int32_t(app_len.size()); }
};

// The creation part of a layout from the list offsets (off[0] = 0, off[nlist] = n).
inline Layout make_layout(const std::vector<int64_t>& off, int32_t chunk)
{
    Layout L;
    L.chunk = chunk;
    L.off = off;
    const int32_t nl = int32_t(off.size()) - 1;
    L.n = off[nl];
    L.base_cstart.assign(size_t(nl) + 1, 0);
    for (int32_t c = 0; c < nl; ++c)
        L.base_cstart[c + 1] = L.base_cstart[c] + int32_t((off[c + 1] - off[c] + chunk - 1) / chunk);
    L.n_base_chunks = L.base_cstart[nl];
    L.list_app.assign(size_t(nl), std::vector<int32_t>());
    return L;
}

// Give m new items (item j joins list lists[j], each in [0, nlist)) their
// rows: each fills its list's last append chunk, then a fresh chunk. Writes
// the ids and returns true; returns false, leaving L as it was, when an id
// plus id_offset would reach id_limit.
inline bool place(Layout& L, const int32_t* lists, int64_t m, int64_t id_offset, int64_t id_limit,
                  std::vector<int64_t>& ids)
{
    std::vector<std::vector<int32_t>> list_app = L.list_app;
    std::vector<int32_t> app_len = L.app_len;
    ids.assign(size_t(m), 0);
    for (int64_t j = 0; j < m; ++j) {
        std::vector<int32_t>& own = list_app[lists[j]];
        if (own.empty() || app_len[own.back()] == L.chunk) {
            const int64_t a = int64_t(app_len.size());
            if (L.n + (a + 1) * L.chunk + id_offset >= id_limit) return false;
            own.push_back(int32_t(a));
            app_len.push_back(0);
        }
        const int32_t a = own.back();
        ids[j] = L.n + int64_t(L.chunk) * a + app_len[a];
        ++app_len[a];
    }
    L.list_app = std::move(list_app);
    L.app_len = std::move(app_len);
    return true;
}

// One chunk table entry: up to `chunk` consecutive rows of one list.
struct ChunkDesc {
    int32_t first_row, plane_block, rows, list;
};

// The chunk table (list by list: creation chunks, then append chunks in fill
// order), each list's first entry, and the size prefixes the search sizes its
// scratch with: top_rows[p] / top_chunks[p] = rows / entries of the p lists
// with the most of them.
struct Tables {
    std::vector<ChunkDesc> desc;
    std::vector<int32_t> start;
    std::vector<int64_t> top_rows, top_chunks;
};

inline Tables build_tables(const Layout& L)
{
    Tables t;
    const int32_t nl = L.nlist();
    const int64_t C = L.chunk;
    t.start.assign(size_t(nl) + 1, 0);
    std::vector<int64_t> rows(nl), chunks(nl);
    for (int32_t c = 0; c < nl; ++c) {
        t.start[c] = int32_t(t.desc.size());
        const int64_t o0 = L.off[c], nc = L.off[c + 1] - o0;
        int64_t r = nc;
        for (int64_t j = 0; j * C < nc; ++j)
            t.desc.push_back(ChunkDesc{int32_t(o0 + j * C), L.base_cstart[c] + int32_t(j),
                                       int32_t(std::min(C, nc - j * C)), c});
        for (int32_t a : L.list_app[c]) {
            t.desc.push_back(ChunkDesc{int32_t(L.n + C * a), L.n_base_chunks + a, L.app_len[a], c});
            r += L.app_len[a];
        }
        rows[c] = r;
        chunks[c] = int64_t(t.desc.size()) - t.start[c];
    }
    t.start[nl] = int32_t(t.desc.size());
    std::sort(rows.begin(), rows.end(), std::greater<int64_t>());
    std::sort(chunks.begin(), chunks.end(), std::greater<int64_t>());
    t.top_rows.assign(size_t(nl) + 1, 0);
    t.top_chunks.assign(size_t(nl) + 1, 0);
    for (int32_t c = 0; c < nl; ++c) {
        t.top_rows[c + 1] = t.top_rows[c] + rows[c];
        t.top_chunks[c + 1] = t.top_chunks[c] + chunks[c];
    }
    return t;
}

}  // namespace rowmap
}  // namespace st
