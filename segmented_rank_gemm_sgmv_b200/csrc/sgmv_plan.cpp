// Segment builder and size-based dispatch (host).
//
// SGMV groups the batch's tokens by adapter and, per segment, uses tensor
// cores for large segments and a batched gather path for small ones
// ("Multi-LoRA serving: the single translator with a thousand glossaries ...",
// section "SGMV: the kernel that holds it all up", and its figure).  This file
// builds that grouping with a stable counting sort over the distinct adapter
// ids of the batch and cuts the work into items for the two kernel families.
#include <algorithm>
#include <cstring>
#include <vector>

#include "internal.h"

namespace sgmv {
namespace {

int64_t align16(int64_t n) { return (n + 15) & ~int64_t(15); }

struct Layout {
    int64_t token_idx, seg_offsets, seg_adapter, seg_rank, seg_scale, seg_a_pt, seg_b_pt, simt_items, tc_tiles, end;
};

Layout layout_for(int64_t rows, int64_t S, int64_t n_proj, int64_t n_simt, int64_t n_tc) {
    Layout L;
    int64_t o = 0;
    L.token_idx = o;   o = align16(o + rows * 4);
    L.seg_offsets = o; o = align16(o + (S + 1) * 4);
    L.seg_adapter = o; o = align16(o + S * 4);
    L.seg_rank = o;    o = align16(o + S * 4);
    L.seg_scale = o;   o = align16(o + S * 4);
    L.seg_a_pt = o;    o = align16(o + S * n_proj * 8);
    L.seg_b_pt = o;    o = align16(o + S * n_proj * 8);
    L.simt_items = o;  o = align16(o + n_simt * n_proj * 32);
    L.tc_tiles = o;    o = align16(o + n_tc * n_proj * 32);
    L.end = o;
    return L;
}

}  // namespace
}  // namespace sgmv

using namespace sgmv;

extern "C" int64_t sgmv_plan_table_capacity(int32_t T, int32_t n_proj) {
    if (T < 0 || n_proj < 0) return -1;
    // rows <= T, segments <= T, items <= T and tiles <= T (each holds >= 1 row)
    return layout_for(T, T, std::max<int64_t>(n_proj, 1), T, T).end;
}

extern "C" sgmv_status sgmv_build_plan(const int32_t* adapter_ids, int32_t T, const sgmv_pool* pool,
                                       int32_t long_threshold, void* table, int64_t table_capacity,
                                       sgmv_plan* plan) {
    if (!pool || !plan) return fail(SGMV_ERR_INVALID, "build_plan: pool and plan are required");
    if (T < 0) return fail(SGMV_ERR_INVALID, "build_plan: T must be >= 0");
    if (T > 0 && !adapter_ids) return fail(SGMV_ERR_INVALID, "build_plan: adapter_ids is NULL");
    if (!table && table_capacity > 0) return fail(SGMV_ERR_INVALID, "build_plan: table is NULL");
    if (reinterpret_cast<uintptr_t>(table) & 15) return fail(SGMV_ERR_INVALID, "build_plan: table must be 16-byte aligned");
    const bool default_threshold = long_threshold <= 0;
    if (default_threshold) long_threshold = kDefaultLongThreshold;

    // Distinct adapters of the batch, ascending; tokens with id -1 use none.
    std::vector<int32_t> ids;
    ids.reserve(T);
    for (int32_t t = 0; t < T; ++t) {
        const int32_t a = adapter_ids[t];
        if (a < -1) return fail(SGMV_ERR_INVALID, "build_plan: adapter id < -1");
        if (a >= 0) ids.push_back(a);
    }
    std::sort(ids.begin(), ids.end());
    ids.erase(std::unique(ids.begin(), ids.end()), ids.end());
    const int64_t S = (int64_t)ids.size();
    std::vector<const AdapterRec*> recs(S);
    for (int64_t s = 0; s < S; ++s) {
        auto it = pool->adapters.find(ids[s]);
        if (it == pool->adapters.end())
            return fail(SGMV_ERR_NOT_RESIDENT, "build_plan: adapter " + std::to_string(ids[s]) + " is not resident");
        recs[s] = &it->second;
    }

    // Counting sort: segment of each token by binary search, then prefix sums.
    std::vector<int32_t> seg_of(T, -1), count(S + 1, 0);
    for (int32_t t = 0; t < T; ++t) {
        if (adapter_ids[t] < 0) continue;
        const int32_t s = (int32_t)(std::lower_bound(ids.begin(), ids.end(), adapter_ids[t]) - ids.begin());
        seg_of[t] = s;
        ++count[s + 1];
    }
    std::vector<int32_t> offsets(S + 1, 0);
    for (int64_t s = 0; s < S; ++s) offsets[s + 1] = offsets[s] + count[s + 1];
    const int32_t rows = offsets[S];

    // With the default threshold, the tensor-core kernels are used only when the long
    // segments hold at least one full 128-row tile in total: below that their fixed cost
    // (cluster launch, tensor-memory allocation, barrier setup) outweighs the adapter
    // re-reads of the SIMT items they would save.  The plan then reports the threshold
    // as never reached.
    if (default_threshold) {
        int64_t long_rows = 0;
        for (int64_t s = 0; s < S; ++s) {
            const int32_t n = offsets[s + 1] - offsets[s];
            if (recs[s]->rank > 0 && n >= long_threshold) long_rows += n;
        }
        if (long_rows < kTcTileRows) long_threshold = INT32_MAX;
    }

    // Dispatch: long segments -> 128-row tensor-core tiles, the rest -> SIMT items.
    int64_t n_simt = 0, n_tc = 0;
    int32_t max_rank = 0, max_item = 0;
    for (int64_t s = 0; s < S; ++s) {
        const int32_t n = offsets[s + 1] - offsets[s], r = recs[s]->rank;
        max_rank = std::max(max_rank, r);
        if (r == 0 || n == 0) continue;
        if (n >= long_threshold) n_tc += (n + kTcTileRows - 1) / kTcTileRows;
        else n_simt += (n + kSimtMaxItemRows - 1) / kSimtMaxItemRows;
    }
    const int64_t n_proj = pool->n_proj;
    const Layout L = layout_for(rows, S, n_proj, n_simt, n_tc);
    if (L.end > table_capacity) return fail(SGMV_ERR_CAPACITY, "build_plan: table capacity too small");

    uint8_t* base = static_cast<uint8_t*>(table);
    if (L.end > 0) std::memset(base, 0, (size_t)L.end);
    int32_t* token_idx = reinterpret_cast<int32_t*>(base + L.token_idx);
    int32_t* seg_offsets = reinterpret_cast<int32_t*>(base + L.seg_offsets);
    int32_t* seg_adapter = reinterpret_cast<int32_t*>(base + L.seg_adapter);
    int32_t* seg_rank = reinterpret_cast<int32_t*>(base + L.seg_rank);
    float* seg_scale = reinterpret_cast<float*>(base + L.seg_scale);
    int64_t* seg_a_pt = reinterpret_cast<int64_t*>(base + L.seg_a_pt);
    int64_t* seg_b_pt = reinterpret_cast<int64_t*>(base + L.seg_b_pt);
    auto recs_rank = [&](int32_t s) { return recs[s]->rank; };
    auto recs_pt = [&](int32_t s, int64_t p, int m) { return m == 0 ? recs[s]->a_pt[p] : recs[s]->b_pt[p]; };
    ItemRec* simt = reinterpret_cast<ItemRec*>(base + L.simt_items);
    ItemRec* tc = reinterpret_cast<ItemRec*>(base + L.tc_tiles);
    auto put = [&](ItemRec* recs, int64_t idx, int32_t s, int32_t r0, int32_t r1) {
        for (int64_t p = 0; p < n_proj; ++p)
            recs[idx * n_proj + p] = ItemRec{s, r0, r1, recs_rank(s), recs_pt(s, p, 0), recs_pt(s, p, 1)};
    };

    std::vector<int32_t> fill(offsets.begin(), offsets.end() - 1);
    for (int32_t t = 0; t < T; ++t)  // ascending t keeps each segment in batch order
        if (seg_of[t] >= 0) token_idx[fill[seg_of[t]]++] = t;
    if (S > 0 || L.end > 0) std::memcpy(seg_offsets, offsets.data(), (S + 1) * sizeof(int32_t));
    // SIMT items are emitted largest rank first (stable): their CTAs are then
    // scheduled first, and the smaller items fill in behind them
    struct Simt {
        int32_t rank, s, r0, r1;
    };
    std::vector<Simt> simt_list;
    simt_list.reserve(n_simt);
    int64_t i_simt = 0, i_tc = 0;
    for (int64_t s = 0; s < S; ++s) {
        seg_adapter[s] = ids[s];
        seg_rank[s] = recs[s]->rank;
        const auto sc = pool->adapter_scale.find(ids[s]);
        seg_scale[s] = sc == pool->adapter_scale.end() ? 1.0f : sc->second;
        for (int64_t p = 0; p < n_proj; ++p) {
            seg_a_pt[s * n_proj + p] = recs[s]->a_pt[p];
            seg_b_pt[s * n_proj + p] = recs[s]->b_pt[p];
        }
        const int32_t b = offsets[s], e = offsets[s + 1], n = e - b;
        if (recs[s]->rank == 0 || n == 0) continue;
        if (n >= long_threshold) {
            for (int32_t r0 = b; r0 < e; r0 += kTcTileRows) put(tc, i_tc++, (int32_t)s, r0, std::min(e, r0 + kTcTileRows));
        } else {
            for (int32_t r0 = b; r0 < e; r0 += kSimtMaxItemRows) {
                const int32_t r1 = std::min(e, r0 + kSimtMaxItemRows);
                max_item = std::max(max_item, r1 - r0);
                simt_list.push_back(Simt{recs[s]->rank, (int32_t)s, r0, r1});
            }
        }
    }
    std::stable_sort(simt_list.begin(), simt_list.end(), [](const Simt& x, const Simt& y) { return x.rank > y.rank; });
    for (const Simt& it : simt_list) put(simt, i_simt++, it.s, it.r0, it.r1);

    std::memset(plan, 0, sizeof(*plan));
    plan->T = T;
    plan->num_segments = (int32_t)S;
    plan->num_rows = rows;
    plan->max_rank = max_rank;
    plan->n_proj = (int32_t)n_proj;
    plan->num_simt_items = (int32_t)n_simt;
    plan->num_tc_tiles = (int32_t)n_tc;
    plan->long_threshold = long_threshold;
    plan->max_item_rows = max_item;
    const int32_t inline_cap = plan->n_proj > 1 ? kInlineItemsMultiProj : kInlineItems;
    plan->needs_device_table = (n_tc > 0 || n_simt > inline_cap) ? 1 : 0;
    plan->host_table = table;
    plan->table_bytes = L.end;
    plan->off_token_idx = L.token_idx;
    plan->off_seg_offsets = L.seg_offsets;
    plan->off_seg_adapter = L.seg_adapter;
    plan->off_seg_rank = L.seg_rank;
    plan->off_seg_scale = L.seg_scale;
    plan->off_seg_a_pt = L.seg_a_pt;
    plan->off_seg_b_pt = L.seg_b_pt;
    plan->off_simt_items = L.simt_items;
    plan->off_tc_tiles = L.tc_tiles;
    return SGMV_OK;
}
