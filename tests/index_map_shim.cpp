// extern "C" wrapper around the library's host-side row map (index_map.h), so
// that the CPU tests can drive it through ctypes without a GPU.
#include <cstring>

#include "../filtered_int8_ann_b200/csrc/index_map.h"

using st::rowmap::Layout;
using st::rowmap::Tables;

struct Handle {
    Layout layout;
    Tables tables;
};

extern "C" {

void* im_create(const int64_t* off, int32_t nlist, int32_t chunk)
{
    Handle* h = new Handle();
    h->layout = st::rowmap::make_layout(std::vector<int64_t>(off, off + nlist + 1), chunk);
    return h;
}

int32_t im_place(void* hp, const int32_t* lists, int64_t m, int64_t id_offset, int64_t id_limit, int64_t* ids)
{
    Handle* h = static_cast<Handle*>(hp);
    std::vector<int64_t> out;
    if (!st::rowmap::place(h->layout, lists, m, id_offset, id_limit, out)) return 0;
    if (m > 0) std::memcpy(ids, out.data(), size_t(m) * 8);
    return 1;
}

int32_t im_app_used(void* hp) { return static_cast<Handle*>(hp)->layout.app_used(); }

int32_t im_build(void* hp)
{
    Handle* h = static_cast<Handle*>(hp);
    h->tables = st::rowmap::build_tables(h->layout);
    return int32_t(h->tables.desc.size());
}

void im_tables(void* hp, int32_t* desc, int32_t* start, int64_t* top_rows, int64_t* top_chunks)
{
    const Tables& t = static_cast<Handle*>(hp)->tables;
    for (size_t i = 0; i < t.desc.size(); ++i) {
        desc[4 * i] = t.desc[i].first_row;
        desc[4 * i + 1] = t.desc[i].plane_block;
        desc[4 * i + 2] = t.desc[i].rows;
        desc[4 * i + 3] = t.desc[i].list;
    }
    std::memcpy(start, t.start.data(), t.start.size() * 4);
    std::memcpy(top_rows, t.top_rows.data(), t.top_rows.size() * 8);
    std::memcpy(top_chunks, t.top_chunks.data(), t.top_chunks.size() * 8);
}

void im_destroy(void* hp) { delete static_cast<Handle*>(hp); }

}  // extern "C"
