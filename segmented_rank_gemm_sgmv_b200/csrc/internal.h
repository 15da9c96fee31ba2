// Library-internal declarations shared by the translation units.
#pragma once
#include <cstdint>
#include <map>
#include <algorithm>
#include <string>
#include <unordered_map>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/sgmv.h"

namespace sgmv {

// --------------------------------------------------------------- status text
sgmv_status fail(sgmv_status s, const std::string& msg);
sgmv_status cuda_fail(cudaError_t e, const char* what);
#define SGMV_CUDA_TRY(call)                                     \
    do {                                                        \
        cudaError_t e__ = (call);                               \
        if (e__ != cudaSuccess) return ::sgmv::cuda_fail(e__, #call); \
    } while (0)

// ---------------------------------------------------------------------- pool
struct AdapterRec {
    int32_t rank = 0;
    int64_t pt_begin = 0, pt_count = 0;      // contiguous page-table range
    std::vector<int64_t> a_pt, b_pt;         // per projection, first entry of A / B^T
};

}  // namespace sgmv

struct sgmv_pool {
    int device = -1;
    int64_t num_pages = 0;
    int32_t page_elems = 0, page_log2 = 0;
    int32_t n_proj = 0, max_rank = 0;
    std::vector<int32_t> d_in, d_out;
    int32_t wfmt = 0;                // sgmv_weight_format
    int64_t page_bytes = 0;          // page_elems values: x2 (bf16), x1 (E4M3), x1/2 (INT4)
    void* pages_dev = nullptr;       // [num_pages][page_bytes]
    float* scale_dev = nullptr;      // quantised pools: fp32 [pt_capacity], scale of a rank row
                                     // at the page-table entry of its first chunk
    int32_t* pt_dev = nullptr;       // int32 [pt_capacity]
    int64_t pt_capacity = 0;
    std::vector<int32_t> pt_host;    // mirror of the page table
    std::vector<int64_t> free_pages; // stack of free page ids
    std::map<int64_t, int64_t> free_pt;  // free page-table ranges: start -> length
    std::unordered_map<int32_t, sgmv::AdapterRec> adapters;
    std::unordered_map<int32_t, float> adapter_scale;  // per-adapter multiplier (1 when absent),
                                                       // kept across evictions and reloads
    void* staging_dev = nullptr;     // device staging for host-source loads
    size_t staging_bytes = 0;
};

namespace sgmv {

// -------------------------------------------------------------- plan tables
// One work item as a kernel sees it for one projection: the rows of a
// segment it covers, its rank, and the first page-table entries of A and B^T
// of its adapter for that projection.  Records are stored [item][projection]
// so that a CTA finds everything about its item with one 32-byte load.
struct ItemRec {
    int32_t seg, row_begin, row_end, rank;
    int64_t a_pt, b_pt;
};
static_assert(sizeof(ItemRec) == 32, "ItemRec must be 32 bytes");

constexpr int kSimtMaxItemRows = 4;    // rows per SIMT work item
constexpr int kInlineItems = 256;      // SIMT items that can travel as launch arguments (13 KB of parameters)
// A plan over a pool of several projections keeps a device table above this many items: a
// launch-argument list carries one projection, and a grouped call over the pool's
// projections (one launch pair for all of them) needs the table.
constexpr int kInlineItemsMultiProj = 64;

// A SIMT work item passed by value in the kernel's parameters: the record for
// the launch's projection plus the item's token rows.
struct InlineItem {
    int32_t seg, row_begin, row_end, rank;
    int64_t a_pt, b_pt;
    int32_t tok[kSimtMaxItemRows];
};
static_assert(sizeof(InlineItem) == 48, "InlineItem must be 48 bytes");
template <int N>
struct InlineTable {
    int32_t count, pad[3];
    InlineItem items[N];
    float scale[N];              // multiplier of each item's adapter
};
constexpr int kTcTileRows = 128;       // rows per tensor-core tile (MMA M)
constexpr int kDefaultLongThreshold = 16;
constexpr int kMaxRank = 128;
constexpr int kMaxGroup = 8;           // projections in one grouped launch

// Device view of everything a kernel needs about the batch.
struct BatchView {
    const int32_t* token_idx;
    const int32_t* seg_offsets;
    const int32_t* seg_rank;
    const int64_t* seg_a_pt;
    const int64_t* seg_b_pt;
    const float* seg_scale;      // [num_segments] multiplier of each segment's adapter
    const ItemRec* simt_items;   // [num_simt_items][n_proj]
    const ItemRec* tc_tiles;     // [num_tc_tiles][n_proj]
    int32_t num_segments, num_rows, n_proj, proj, T;
};

// Weight format of a pool, as the kernels see it: bytes that hold 8 values.
constexpr int kFmtBf16 = 0, kFmtFp8 = 1, kFmtInt4 = 2;
template <int WF>
__host__ __device__ constexpr int bytes_per_8() { return WF == kFmtBf16 ? 16 : WF == kFmtFp8 ? 8 : 4; }

// 40 bytes, part of every kernel's parameters (page ids are int32, so is the page count).
struct PoolView {
    const uint16_t* pages;       // bf16 pages; a quantised pool's code pages as the same buffer
    const int32_t* page_table;
    const float* row_scale;      // quantised pools: scale of each rank row (first-chunk entry)
    int64_t pt_capacity;
    int32_t num_pages;
    int16_t page_log2;
    int16_t wfmt;                // sgmv_weight_format
};
static_assert(sizeof(PoolView) == 40, "PoolView must stay 40 bytes");

// --------------------------------------------------------------- launchers
// Work of the SIMT items, in stages of 8 rank rows: `sum_ng` over the items,
// `max_ng` of the largest (items come largest first).  The launchers size the
// CTA split with it.
struct SimtWork {
    int64_t sum_ng = 0;
    int32_t max_ng = 0;
};
constexpr int kMaxShare = 4;           // projections that share one x in a SIMT shrink pass

// One x of a SIMT shrink launch and the projections computed from it: nsub >= 1
// projections whose A rows are stacked in the same CTAs (their shared x is read
// once per CTA).  A launch takes up to kMaxGroup of them over the same plan
// (launch arguments `inl` only with one job of one projection).
struct ShrinkJob {
    const uint16_t* x;
    int64_t ldx;
    int32_t d_in;
    int32_t nsub;
    int32_t proj[kMaxShare];
    float* v[kMaxShare];
    int64_t ldv[kMaxShare];
};
struct ExpandJob {
    const float* v;
    int64_t ldv;
    int32_t d_out;
    int32_t proj;
    void* y;
    int64_t ldy;
};
// `inl` (may be null) holds the items as launch arguments when they fit.
cudaError_t launch_shrink_simt(const ShrinkJob* jobs, int n_jobs, const BatchView& b, int32_t num_items,
                               int32_t max_item_rows, int32_t max_rank, const SimtWork& work, const PoolView& pool,
                               const InlineTable<kInlineItems>* inl, cudaStream_t stream);
// y_early: y may be read before the preceding kernel completes (that kernel is
// the shrink of the same call, which does not write y).
cudaError_t launch_expand_simt(const ExpandJob* jobs, int n_jobs, const BatchView& b, int32_t num_items,
                               int32_t max_item_rows, int32_t max_rank, const SimtWork& work, const PoolView& pool,
                               float scale, int32_t y_dtype, const InlineTable<kInlineItems>* inl, bool y_early,
                               cudaStream_t stream);
// Both phases of a single projection in one kernel (decode-sized plans without tensor-core
// tiles); *used = false (nothing launched) when the plan does not fit its limits.
cudaError_t launch_fused_simt(const ShrinkJob& sj, const ExpandJob& ej, const BatchView& b, int32_t num_items,
                              int32_t max_item_rows, int32_t max_rank, const PoolView& pool, float scale,
                              int32_t y_dtype, const InlineTable<kInlineItems>* inl, cudaStream_t stream,
                              bool* used, bool dry = false);
// The one-shot slab shrink of one x over a bf16 pool, when it applies (*used = true; with
// `dry` the choice is made and nothing is launched).  launch_shrink_simt tries it first.
cudaError_t slab_shrink_launch(const ShrinkJob& j, const BatchView& b, int32_t num_items, int32_t max_item_rows,
                               int32_t max_rank, const PoolView& pool, const InlineTable<kInlineItems>* inl,
                               cudaStream_t stream, bool* used, bool dry);
cudaError_t launch_shrink_tc(const uint16_t* x, int64_t ldx, int32_t d_in, const BatchView& b, int32_t num_tiles,
                             int32_t max_rank, const PoolView& pool, float* v, int64_t ldv, cudaStream_t stream);
// after_shrink: the preceding kernel of the stream is this call's tensor-core shrink, an
// ordinary launch that wrote v and nothing else this kernel reads; the expand is then a
// programmatic dependent launch that reads the plan, the pool and y at once and waits for
// the shrink's completion only before it reads v.
cudaError_t launch_expand_tc(const float* v, int64_t ldv, int32_t d_out, const BatchView& b, int32_t num_tiles,
                             int32_t max_rank, const PoolView& pool, float scale, void* y, int64_t ldy,
                             int32_t y_dtype, bool after_shrink, cudaStream_t stream);

// Read and clear the device error words of every translation unit.
cudaError_t read_clear_errors_simt(uint32_t* bits, cudaStream_t stream);
cudaError_t read_clear_errors_tc(uint32_t* bits, cudaStream_t stream);

// Store a bf16 matrix (rank rows x cols; `transpose`: stored as cols x rows) into the
// pool's pages from page-table entry pt_base on, quantising it in a quantised pool
// (sgmv_pool.cu).
cudaError_t write_matrix(sgmv_pool* p, const uint16_t* src, int64_t rows, int64_t cols, bool transpose,
                         int64_t pt_base, cudaStream_t stream);

}  // namespace sgmv
