// C ABI entry points: argument validation, the size-based dispatch between
// the SIMT and the tensor-core kernels, and error reporting.
#include <algorithm>
#include <cstdio>
#include <mutex>
#include <string>

#include "internal.h"
#include "ptx.cuh"

namespace sgmv {

namespace {
thread_local std::string t_last_error;
}

sgmv_status fail(sgmv_status s, const std::string& msg) {
    t_last_error = msg;
    return s;
}

sgmv_status cuda_fail(cudaError_t e, const char* what) {
    t_last_error = std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")";
    return SGMV_ERR_CUDA;
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

sgmv_status make_views(const sgmv_plan* plan, const void* table, const sgmv_pool* pool, int32_t T, int32_t proj,
                       BatchView* bv, PoolView* pv, const char* who) {
    const std::string w(who);
    if (!plan || !pool) return fail(SGMV_ERR_INVALID, w + ": plan and pool are required");
    if (pool->device < 0 || !pool->pages_dev) return fail(SGMV_ERR_INVALID, w + ": pool has no device memory");
    if (plan->T != T) return fail(SGMV_ERR_INVALID, w + ": T differs from the plan's T");
    if (plan->n_proj != pool->n_proj) return fail(SGMV_ERR_INVALID, w + ": plan was built for another pool");
    if (proj < 0 || proj >= pool->n_proj) return fail(SGMV_ERR_INVALID, w + ": projection index out of range");
    if (plan->needs_device_table && (!table || !aligned16(table)))
        return fail(SGMV_ERR_INVALID, w + ": this plan needs its table as a 16-byte aligned device pointer");
    if (!plan->needs_device_table && !table && !plan->host_table)
        return fail(SGMV_ERR_INVALID, w + ": plan->host_table is NULL and no device table was given");
    const uint8_t* base = static_cast<const uint8_t*>(table);
    *bv = BatchView{};
    if (base) {
        bv->token_idx = reinterpret_cast<const int32_t*>(base + plan->off_token_idx);
        bv->seg_offsets = reinterpret_cast<const int32_t*>(base + plan->off_seg_offsets);
        bv->seg_rank = reinterpret_cast<const int32_t*>(base + plan->off_seg_rank);
        bv->seg_a_pt = reinterpret_cast<const int64_t*>(base + plan->off_seg_a_pt);
        bv->seg_b_pt = reinterpret_cast<const int64_t*>(base + plan->off_seg_b_pt);
        bv->seg_scale = reinterpret_cast<const float*>(base + plan->off_seg_scale);
        bv->simt_items = reinterpret_cast<const ItemRec*>(base + plan->off_simt_items);
        bv->tc_tiles = reinterpret_cast<const ItemRec*>(base + plan->off_tc_tiles);
    }
    bv->num_segments = plan->num_segments;
    bv->num_rows = plan->num_rows;
    bv->n_proj = plan->n_proj;
    bv->proj = proj;
    bv->T = T;
    pv->pages = static_cast<const uint16_t*>(pool->pages_dev);
    pv->page_table = pool->pt_dev;
    pv->num_pages = (int32_t)pool->num_pages;
    pv->pt_capacity = pool->pt_capacity;
    pv->page_log2 = (int16_t)pool->page_log2;
    pv->row_scale = pool->scale_dev;
    pv->wfmt = (int16_t)pool->wfmt;
    return SGMV_OK;
}

// The SIMT items of `plan` for projection `proj` as launch arguments, read from
// the host table; false when they do not fit (the kernels then read the
// device table).
bool inline_items(const sgmv_plan* plan, int32_t proj, InlineTable<kInlineItems>* t) {
    if (!plan->host_table || plan->num_simt_items <= 0 || plan->num_simt_items > kInlineItems) return false;
    const uint8_t* base = static_cast<const uint8_t*>(plan->host_table);
    const ItemRec* recs = reinterpret_cast<const ItemRec*>(base + plan->off_simt_items);
    const int32_t* tix = reinterpret_cast<const int32_t*>(base + plan->off_token_idx);
    const float* ssc = reinterpret_cast<const float*>(base + plan->off_seg_scale);
    t->count = plan->num_simt_items;
    for (int i = 0; i < plan->num_simt_items; ++i) {
        const ItemRec& r = recs[(int64_t)i * plan->n_proj + proj];
        InlineItem& it = t->items[i];
        it.seg = r.seg;
        it.row_begin = r.row_begin;
        it.row_end = r.row_end;
        it.rank = r.rank;
        it.a_pt = r.a_pt;
        it.b_pt = r.b_pt;
        t->scale[i] = (r.seg >= 0 && r.seg < plan->num_segments) ? ssc[r.seg] : 1.0f;
        for (int j = 0; j < kSimtMaxItemRows; ++j) {
            const int row = r.row_begin + j;
            it.tok[j] = (row < r.row_end && row >= 0 && row < plan->num_rows) ? tix[row] : -1;
        }
    }
    return true;
}

// Stage counts of the SIMT items, read from the host table (which the plan's
// contract keeps valid until the calls); uniform by the plan's max rank if absent.
SimtWork simt_work(const sgmv_plan* plan) {
    SimtWork w;
    const int32_t n = plan->num_simt_items;
    w.max_ng = (std::max(plan->max_rank, 1) + 7) / 8;
    if (n <= 0) return w;
    if (!plan->host_table) {
        w.sum_ng = (int64_t)n * w.max_ng;
        return w;
    }
    const ItemRec* recs = reinterpret_cast<const ItemRec*>(static_cast<const uint8_t*>(plan->host_table) +
                                                           plan->off_simt_items);
    int32_t mx = 1;
    for (int32_t i = 0; i < n; ++i) {
        const int32_t ng = (std::max(recs[(int64_t)i * plan->n_proj].rank, 1) + 7) / 8;
        w.sum_ng += ng;
        mx = std::max(mx, ng);
    }
    w.max_ng = mx;
    return w;
}

}  // namespace

sgmv_status shrink_impl(const void* x, int64_t ldx, int32_t T, int32_t d_in, int32_t proj, const sgmv_plan* plan,
                        const void* table, const sgmv_pool* pool, float* v, int64_t ldv, cudaStream_t stream);
sgmv_status expand_impl(const float* v, int64_t ldv, int32_t T, int32_t d_out, int32_t proj, const sgmv_plan* plan,
                        const void* table, const sgmv_pool* pool, float scale, void* y, int64_t ldy, int32_t y_dtype,
                        bool y_early, cudaStream_t stream);
sgmv_status delta_impl(const sgmv_delta_entry* entries, int32_t n, int32_t T, const sgmv_plan* plan,
                       const void* table, const sgmv_pool* pool, float scale, int32_t y_dtype, cudaStream_t stream);

}  // namespace sgmv

using namespace sgmv;

extern "C" const char* sgmv_status_string(sgmv_status s) {
    switch (s) {
        case SGMV_OK: return "SGMV_OK";
        case SGMV_ERR_INVALID: return "SGMV_ERR_INVALID";
        case SGMV_ERR_UNSUPPORTED: return "SGMV_ERR_UNSUPPORTED";
        case SGMV_ERR_NOT_RESIDENT: return "SGMV_ERR_NOT_RESIDENT";
        case SGMV_ERR_OUT_OF_PAGES: return "SGMV_ERR_OUT_OF_PAGES";
        case SGMV_ERR_CUDA: return "SGMV_ERR_CUDA";
        case SGMV_ERR_BOUNDS: return "SGMV_ERR_BOUNDS";
        case SGMV_ERR_TIMEOUT: return "SGMV_ERR_TIMEOUT";
        case SGMV_ERR_CAPACITY: return "SGMV_ERR_CAPACITY";
    }
    return "SGMV_ERR_UNKNOWN";
}

extern "C" const char* sgmv_last_error(void) { return t_last_error.c_str(); }

extern "C" sgmv_status sgmv_shrink(const void* x, int64_t ldx, int32_t T, int32_t d_in, int32_t proj,
                                   const sgmv_plan* plan, const void* table, const sgmv_pool* pool, float* v,
                                   int64_t ldv, sgmv_stream_t stream) {
    return shrink_impl(x, ldx, T, d_in, proj, plan, table, pool, v, ldv, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" sgmv_status sgmv_expand(const float* v, int64_t ldv, int32_t T, int32_t d_out, int32_t proj,
                                   const sgmv_plan* plan, const void* table, const sgmv_pool* pool, float scale,
                                   void* y, int64_t ldy, int32_t y_dtype, sgmv_stream_t stream) {
    return expand_impl(v, ldv, T, d_out, proj, plan, table, pool, scale, y, ldy, y_dtype, false,
                       reinterpret_cast<cudaStream_t>(stream));
}

namespace {

// Argument checks of the shrink phase; fills the views.  Returns SGMV_OK with
// *nothing = true when the batch has no work.
sgmv_status check_shrink(const void* x, int64_t ldx, int32_t T, int32_t d_in, int32_t proj, const sgmv_plan* plan,
                         const void* table, const sgmv_pool* pool, const float* v, int64_t ldv, BatchView* bv,
                         PoolView* pv, bool* nothing) {
    sgmv_status st = make_views(plan, table, pool, T, proj, bv, pv, "shrink");
    if (st != SGMV_OK) return st;
    if (d_in != pool->d_in[proj]) return fail(SGMV_ERR_INVALID, "shrink: d_in differs from the pool's projection");
    *nothing = plan->num_rows == 0 || (plan->num_simt_items == 0 && plan->num_tc_tiles == 0);
    if (*nothing) return SGMV_OK;
    if (!x || !v) return fail(SGMV_ERR_INVALID, "shrink: x and v are required");
    if (ldx < d_in || (ldx % 8) || !aligned16(x)) return fail(SGMV_ERR_INVALID, "shrink: x rows must be 16-byte aligned, ldx >= d_in");
    if (ldv < plan->max_rank || ldv < 1 || (ldv % 4) || !aligned16(v))
        return fail(SGMV_ERR_INVALID, "shrink: v needs ldv >= max_rank, ldv % 4 == 0, 16-byte alignment");
    if (plan->num_simt_items > 0 && pool->page_elems > 1024)
        return fail(SGMV_ERR_UNSUPPORTED, "shrink: the SIMT path takes page_elems <= 1024");
    return SGMV_OK;
}

// Argument checks of the expand phase; fills the views.
sgmv_status check_expand(const float* v, int64_t ldv, int32_t T, int32_t d_out, int32_t proj, const sgmv_plan* plan,
                         const void* table, const sgmv_pool* pool, const void* y, int64_t ldy, int32_t y_dtype,
                         BatchView* bv, PoolView* pv, bool* nothing) {
    sgmv_status st = make_views(plan, table, pool, T, proj, bv, pv, "expand");
    if (st != SGMV_OK) return st;
    if (d_out != pool->d_out[proj]) return fail(SGMV_ERR_INVALID, "expand: d_out differs from the pool's projection");
    if (y_dtype != 0 && y_dtype != 1) return fail(SGMV_ERR_INVALID, "expand: y_dtype must be 0 (bf16) or 1 (fp32)");
    *nothing = plan->num_rows == 0 || (plan->num_simt_items == 0 && plan->num_tc_tiles == 0);
    if (*nothing) return SGMV_OK;
    if (!v || !y) return fail(SGMV_ERR_INVALID, "expand: v and y are required");
    const int64_t esz = y_dtype == 0 ? 2 : 4;
    if (ldy < d_out || ((ldy * esz) % 16) || !aligned16(y))
        return fail(SGMV_ERR_INVALID, "expand: y rows must be 16-byte aligned, ldy >= d_out");
    if (ldv < plan->max_rank || ldv < 1 || (ldv % 4) || !aligned16(v))
        return fail(SGMV_ERR_INVALID, "expand: v needs ldv >= max_rank, ldv % 4 == 0, 16-byte alignment");
    if (plan->num_simt_items > 0 && pool->page_elems > 1024)
        return fail(SGMV_ERR_UNSUPPORTED, "expand: the SIMT path takes page_elems <= 1024");
    return SGMV_OK;
}

}  // namespace

sgmv_status sgmv::shrink_impl(const void* x, int64_t ldx, int32_t T, int32_t d_in, int32_t proj,
                              const sgmv_plan* plan, const void* table, const sgmv_pool* pool, float* v,
                              int64_t ldv, cudaStream_t stream) {
    BatchView bv;
    PoolView pv;
    bool nothing = false;
    sgmv_status st = check_shrink(x, ldx, T, d_in, proj, plan, table, pool, v, ldv, &bv, &pv, &nothing);
    if (st != SGMV_OK || nothing) return st;
    const uint16_t* xb = static_cast<const uint16_t*>(x);
    InlineTable<kInlineItems> inl;
    const bool use_inl = inline_items(plan, proj, &inl);
    const ShrinkJob job{xb, ldx, d_in, 1, {proj}, {v}, {ldv}};
    SGMV_CUDA_TRY(launch_shrink_simt(&job, 1, bv, plan->num_simt_items, plan->max_item_rows, plan->max_rank,
                                     simt_work(plan), pv, use_inl ? &inl : nullptr, stream));
    SGMV_CUDA_TRY(launch_shrink_tc(xb, ldx, d_in, bv, plan->num_tc_tiles, plan->max_rank, pv, v, ldv, stream));
    return SGMV_OK;
}

sgmv_status sgmv::expand_impl(const float* v, int64_t ldv, int32_t T, int32_t d_out, int32_t proj,
                              const sgmv_plan* plan, const void* table, const sgmv_pool* pool, float scale, void* y,
                              int64_t ldy, int32_t y_dtype, bool y_early, cudaStream_t stream) {
    BatchView bv;
    PoolView pv;
    bool nothing = false;
    sgmv_status st = check_expand(v, ldv, T, d_out, proj, plan, table, pool, y, ldy, y_dtype, &bv, &pv, &nothing);
    if (st != SGMV_OK || nothing) return st;
    InlineTable<kInlineItems> inl;
    const bool use_inl = inline_items(plan, proj, &inl);
    const ExpandJob job{v, ldv, d_out, proj, y, ldy};
    SGMV_CUDA_TRY(launch_expand_simt(&job, 1, bv, plan->num_simt_items, plan->max_item_rows, plan->max_rank,
                                     simt_work(plan), pv, scale, y_dtype, use_inl ? &inl : nullptr, y_early, stream));
    SGMV_CUDA_TRY(launch_expand_tc(v, ldv, d_out, bv, plan->num_tc_tiles, plan->max_rank, pv, scale, y, ldy, y_dtype,
                                   false, stream));
    return SGMV_OK;
}

// Both phases of every entry (projections over one plan), arguments checked
// before anything is launched: the SIMT shrink of all entries, the tensor-core
// shrinks, then the SIMT expand of all entries as a programmatic dependent
// launch (its adapter pages and y rows stream in while the shrinks run) and the
// tensor-core expands.  Launch-argument work lists carry one projection, so a
// group over a plan without a device table runs entry by entry.
sgmv_status sgmv::delta_impl(const sgmv_delta_entry* entries, int32_t n, int32_t T, const sgmv_plan* plan,
                             const void* table, const sgmv_pool* pool, float scale, int32_t y_dtype,
                             cudaStream_t stream) {
    if (!entries || n < 1 || n > kMaxGroup)
        return fail(SGMV_ERR_INVALID, "lora_delta: 1 to " + std::to_string(kMaxGroup) + " entries are required");
    BatchView bv;
    PoolView pv;
    bool nothing = false;
    for (int32_t i = 0; i < n; ++i) {
        const sgmv_delta_entry& e = entries[i];
        if (plan && plan->num_rows > 0 && (plan->num_simt_items > 0 || plan->num_tc_tiles > 0) && !e.v)
            return fail(SGMV_ERR_INVALID, "lora_delta: the workspace v is required");
        for (int32_t k = 0; k < i; ++k)
            if (entries[k].v == e.v && e.v)
                return fail(SGMV_ERR_INVALID, "lora_delta: the entries of a group need distinct workspaces v");
        sgmv_status st = check_shrink(e.x, e.ldx, T, e.d_in, e.proj, plan, table, pool, e.v, e.ldv, &bv, &pv, &nothing);
        if (st != SGMV_OK) return st;
        st = check_expand(e.v, e.ldv, T, e.d_out, e.proj, plan, table, pool, e.y, e.ldy, y_dtype, &bv, &pv, &nothing);
        if (st != SGMV_OK) return st;
    }
    if (nothing) return SGMV_OK;
    InlineTable<kInlineItems> inl;
    const bool use_inl = n == 1 && inline_items(plan, entries[0].proj, &inl);
    if (n > 1 && !table && plan->num_simt_items > 0) {  // items only as launch arguments: one entry at a time
        for (int32_t i = 0; i < n; ++i) {
            const sgmv_status st = delta_impl(&entries[i], 1, T, plan, table, pool, scale, y_dtype, stream);
            if (st != SGMV_OK) return st;
        }
        return SGMV_OK;
    }
    const SimtWork work = simt_work(plan);
    // entries that read the same x (same pointer, row stride and d_in) share one SIMT
    // shrink pass: their A rows are stacked in the same CTAs and x is read once per CTA
    ShrinkJob sj[kMaxGroup];
    ExpandJob ej[kMaxGroup];
    int n_sj = 0;
    for (int32_t i = 0; i < n; ++i) {
        const sgmv_delta_entry& e = entries[i];
        ej[i] = ExpandJob{e.v, e.ldv, e.d_out, e.proj, e.y, e.ldy};
        int g = 0;
        while (g < n_sj && !(sj[g].x == e.x && sj[g].ldx == e.ldx && sj[g].d_in == e.d_in && sj[g].nsub < kMaxShare))
            ++g;
        if (g == n_sj) sj[n_sj++] = ShrinkJob{static_cast<const uint16_t*>(e.x), e.ldx, e.d_in, 0, {}, {}, {}};
        ShrinkJob& j = sj[g];
        j.proj[j.nsub] = e.proj;
        j.v[j.nsub] = e.v;
        j.ldv[j.nsub] = e.ldv;
        ++j.nsub;
    }
    if (use_inl && sj[0].nsub > 1) return fail(SGMV_ERR_INVALID, "lora_delta: internal: shared x with inline items");
    if (n == 1 && plan->num_tc_tiles == 0) {  // decode-sized: both phases in one kernel when it fits
        bool used = false;
        SGMV_CUDA_TRY(launch_fused_simt(sj[0], ej[0], bv, plan->num_simt_items, plan->max_item_rows, plan->max_rank,
                                        pv, scale, y_dtype, use_inl ? &inl : nullptr, stream, &used));
        if (used) return SGMV_OK;
    }
    SGMV_CUDA_TRY(launch_shrink_simt(sj, n_sj, bv, plan->num_simt_items, plan->max_item_rows, plan->max_rank, work, pv,
                                     use_inl ? &inl : nullptr, stream));
    for (int32_t i = 0; i < n; ++i) {
        const sgmv_delta_entry& e = entries[i];
        bv.proj = e.proj;
        SGMV_CUDA_TRY(launch_shrink_tc(static_cast<const uint16_t*>(e.x), e.ldx, e.d_in, bv, plan->num_tc_tiles,
                                       plan->max_rank, pv, e.v, e.ldv, stream));
    }
    // the expand's predecessors are this call's shrinks, which do not write y: y may be read early
    SGMV_CUDA_TRY(launch_expand_simt(ej, n, bv, plan->num_simt_items, plan->max_item_rows, plan->max_rank, work, pv,
                                     scale, y_dtype, use_inl ? &inl : nullptr, true, stream));
    // the first tensor-core expand directly follows a tensor-core shrink when there are no
    // SIMT items: it may then start while that shrink finishes
    for (int32_t i = 0; i < n; ++i) {
        bv.proj = entries[i].proj;
        SGMV_CUDA_TRY(launch_expand_tc(ej[i].v, ej[i].ldv, ej[i].d_out, bv, plan->num_tc_tiles, plan->max_rank, pv,
                                       scale, ej[i].y, ej[i].ldy, y_dtype, i == 0 && plan->num_simt_items == 0,
                                       stream));
    }
    return SGMV_OK;
}

extern "C" sgmv_status sgmv_lora_delta(const void* x, int64_t ldx, int32_t T, int32_t d_in, int32_t d_out,
                                       int32_t proj, const sgmv_plan* plan, const void* table, const sgmv_pool* pool,
                                       float scale, void* y, int64_t ldy, int32_t y_dtype, float* v, int64_t ldv,
                                       sgmv_stream_t stream) {
    if (plan && plan->num_rows > 0 && (plan->num_simt_items > 0 || plan->num_tc_tiles > 0) && !v)
        return fail(SGMV_ERR_INVALID, "lora_delta: the workspace v is required");
    const sgmv_delta_entry e{proj, d_in, d_out, 0, x, ldx, y, ldy, v, ldv};
    return delta_impl(&e, 1, T, plan, table, pool, scale, y_dtype, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" sgmv_status sgmv_lora_delta_grouped(const sgmv_delta_entry* entries, int32_t n_entries, int32_t T,
                                               const sgmv_plan* plan, const void* table, const sgmv_pool* pool,
                                               float scale, int32_t y_dtype, sgmv_stream_t stream) {
    return delta_impl(entries, n_entries, T, plan, table, pool, scale, y_dtype, reinterpret_cast<cudaStream_t>(stream));
}

namespace sgmv {
namespace {
// The plan table from pinned host memory to the device: coalesced 16-byte loads through
// unified addressing (the host buffer is read across the bus by the kernel), stores to the
// device copy.  Four granules a thread, loads before stores.
constexpr int kUploadThreads = 256, kUploadPer = 4;
__global__ void __launch_bounds__(kUploadThreads) table_upload_kernel(const uint4* __restrict__ src,
                                                                      uint4* __restrict__ dst, int64_t n16) {
    const int64_t base = (int64_t)blockIdx.x * kUploadThreads * kUploadPer + threadIdx.x;
    uint4 r[kUploadPer];
#pragma unroll
    for (int i = 0; i < kUploadPer; ++i) {
        const int64_t g = base + (int64_t)i * kUploadThreads;
        if (g < n16) r[i] = src[g];
    }
#pragma unroll
    for (int i = 0; i < kUploadPer; ++i) {
        const int64_t g = base + (int64_t)i * kUploadThreads;
        if (g < n16) dst[g] = r[i];
    }
}
}  // namespace
}  // namespace sgmv

extern "C" sgmv_status sgmv_upload_table(const sgmv_plan* plan, void* device_table, sgmv_stream_t stream) {
    if (!plan || !device_table) return fail(SGMV_ERR_INVALID, "upload_table: plan and device_table are required");
    if (!plan->host_table) return fail(SGMV_ERR_INVALID, "upload_table: plan->host_table is NULL");
    if (!aligned16(device_table) || !aligned16(plan->host_table))
        return fail(SGMV_ERR_INVALID, "upload_table: both tables must be 16-byte aligned");
    const int64_t bytes = plan->table_bytes;
    if (bytes <= 0) return SGMV_OK;
    if (bytes % 16) return fail(SGMV_ERR_INVALID, "upload_table: table_bytes is not a multiple of 16");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaPointerAttributes at{};
    const void* src = nullptr;
    if (cudaPointerGetAttributes(&at, plan->host_table) == cudaSuccess && at.type == cudaMemoryTypeHost)
        src = at.devicePointer;
    cudaGetLastError();  // (an unregistered pointer is not an error here)
    if (!src) {  // pageable host memory: a copy-engine transfer
        SGMV_CUDA_TRY(cudaMemcpyAsync(device_table, plan->host_table, (size_t)bytes, cudaMemcpyHostToDevice, s));
        return SGMV_OK;
    }
    const int64_t n16 = bytes / 16;
    const int64_t per_cta = (int64_t)kUploadThreads * kUploadPer;
    table_upload_kernel<<<(unsigned)((n16 + per_cta - 1) / per_cta), kUploadThreads, 0, s>>>(
        static_cast<const uint4*>(src), static_cast<uint4*>(device_table), n16);
    SGMV_CUDA_TRY(cudaGetLastError());
    return SGMV_OK;
}

// Which kernels sgmv_lora_delta / sgmv_lora_delta_grouped launch for a plan, pool and set of
// projections: the same choices the calls make (including the one-wave test of the fused
// kernel, an occupancy query), with nothing launched.
extern "C" sgmv_status sgmv_lora_delta_kernels(const sgmv_plan* plan, const sgmv_pool* pool, const int32_t* projs,
                                               int32_t n_entries, const void* table, int32_t y_dtype,
                                               int32_t* kinds, int32_t* launches) {
    if (!plan || !pool || !projs || !kinds || !launches)
        return fail(SGMV_ERR_INVALID, "lora_delta_kernels: plan, pool, projs, kinds and launches are required");
    if (pool->device < 0 || !pool->pages_dev)
        return fail(SGMV_ERR_INVALID, "lora_delta_kernels: pool has no device memory");
    if (n_entries < 1 || n_entries > kMaxGroup)
        return fail(SGMV_ERR_INVALID, "lora_delta_kernels: 1 to " + std::to_string(kMaxGroup) + " entries are required");
    if (y_dtype != 0 && y_dtype != 1) return fail(SGMV_ERR_INVALID, "lora_delta_kernels: y_dtype must be 0 or 1");
    if (plan->n_proj != pool->n_proj) return fail(SGMV_ERR_INVALID, "lora_delta_kernels: plan was built for another pool");
    for (int32_t i = 0; i < n_entries; ++i)
        if (projs[i] < 0 || projs[i] >= pool->n_proj)
            return fail(SGMV_ERR_INVALID, "lora_delta_kernels: projection index out of range");
    *kinds = 0;
    *launches = 0;
    if (plan->num_rows <= 0 || (plan->num_simt_items <= 0 && plan->num_tc_tiles <= 0)) return SGMV_OK;
    const bool simt = plan->num_simt_items > 0, tc = plan->num_tc_tiles > 0;
    if (tc) {
        *kinds |= SGMV_KERNELS_TC;
        *launches += 2 * n_entries;  // a shrink and an expand per entry
    }
    if (!simt) return SGMV_OK;
    SGMV_CUDA_TRY(cudaSetDevice(pool->device));
    const bool per_entry = n_entries > 1 && !table;  // the calls then run the entries one at a time
    const int32_t calls = per_entry ? n_entries : 1;
    for (int32_t c = 0; c < calls; ++c) {
        bool fused = false;
        if ((per_entry || n_entries == 1) && !tc) {
            const int32_t p = projs[c];
            PoolView pv{};
            pv.page_log2 = (int16_t)pool->page_log2;
            pv.wfmt = (int16_t)pool->wfmt;
            const ShrinkJob sj{nullptr, 0, pool->d_in[p], 1, {p}, {}, {}};
            const ExpandJob ej{nullptr, 0, pool->d_out[p], p, nullptr, 0};
            InlineTable<kInlineItems> inl;
            const bool use_inl = inline_items(plan, p, &inl);
            SGMV_CUDA_TRY(launch_fused_simt(sj, ej, BatchView{}, plan->num_simt_items, plan->max_item_rows,
                                            plan->max_rank, pv, 1.0f, y_dtype, use_inl ? &inl : nullptr, nullptr,
                                            &fused, true));
        }
        *kinds |= fused ? SGMV_KERNELS_FUSED : SGMV_KERNELS_SIMT;
        *launches += fused ? 1 : 2;
        if (!fused && (per_entry || n_entries == 1)) {  // one x, one projection: the slab shrink may run
            const int32_t p = projs[c];
            PoolView pv{};
            pv.page_log2 = (int16_t)pool->page_log2;
            pv.wfmt = (int16_t)pool->wfmt;
            const ShrinkJob sj{nullptr, 0, pool->d_in[p], 1, {p}, {}, {}};
            InlineTable<kInlineItems> inl;
            const bool use_inl = inline_items(plan, p, &inl);
            bool slab = false;
            SGMV_CUDA_TRY(slab_shrink_launch(sj, BatchView{}, plan->num_simt_items, plan->max_item_rows,
                                             plan->max_rank, pv, use_inl ? &inl : nullptr, nullptr, &slab, true));
            if (slab) *kinds |= SGMV_KERNELS_SLAB;
        }
    }
    return SGMV_OK;
}

// ---------------------------------------------------------------------------
// The step from host buffers: plan, copies in, grouped delta, copy out.

namespace {

int64_t align256(int64_t n) { return (n + 255) & ~int64_t(255); }

// Device workspace layout of sgmv_lora_delta_host: the table, every distinct x,
// every y, then every v (rows x ldv fp32); `rows` and `ldv` may be upper bounds.
struct HostLayout {
    int64_t table = 0, x[kMaxGroup] = {}, y[kMaxGroup] = {}, v[kMaxGroup] = {}, end = 0;
    int x_of[kMaxGroup] = {};  // entry -> first entry with the same x
};

bool host_layout(const sgmv_host_entry* e, int32_t n, int32_t T, int64_t table_bytes, int64_t rows, int64_t ldv,
                 int32_t y_dtype, HostLayout* L) {
    const int64_t esz = y_dtype == 0 ? 2 : 4;
    int64_t o = 0;
    L->table = o;
    o = align256(o + std::max<int64_t>(table_bytes, 16));
    for (int32_t i = 0; i < n; ++i) {
        L->x_of[i] = i;
        for (int32_t k = 0; k < i; ++k)
            if (e[k].x_host == e[i].x_host && e[k].d_in == e[i].d_in) {
                L->x_of[i] = L->x_of[k];
                break;
            }
        if (L->x_of[i] == i) {
            L->x[i] = o;
            o = align256(o + (int64_t)T * e[i].d_in * 2);
        } else {
            L->x[i] = L->x[L->x_of[i]];
        }
    }
    for (int32_t i = 0; i < n; ++i) {
        L->y[i] = o;
        o = align256(o + (int64_t)T * e[i].d_out * esz);
    }
    for (int32_t i = 0; i < n; ++i) {
        L->v[i] = o;
        o = align256(o + std::max<int64_t>(rows, 1) * ldv * 4);
    }
    L->end = o;
    return true;
}

sgmv_status check_host_entries(const sgmv_host_entry* e, int32_t n, const sgmv_pool* pool, int32_t y_dtype) {
    if (!pool) return fail(SGMV_ERR_INVALID, "lora_delta_host: pool is NULL");
    if (!e || n < 1 || n > kMaxGroup)
        return fail(SGMV_ERR_INVALID, "lora_delta_host: 1 to " + std::to_string(kMaxGroup) + " entries are required");
    if (y_dtype != 0 && y_dtype != 1) return fail(SGMV_ERR_INVALID, "lora_delta_host: y_dtype must be 0 or 1");
    for (int32_t i = 0; i < n; ++i) {
        if (e[i].proj < 0 || e[i].proj >= pool->n_proj) return fail(SGMV_ERR_INVALID, "lora_delta_host: bad projection");
        if (e[i].d_in != pool->d_in[e[i].proj] || e[i].d_out != pool->d_out[e[i].proj])
            return fail(SGMV_ERR_INVALID, "lora_delta_host: d_in / d_out differ from the pool's projection");
        if (!e[i].x_host || !e[i].y_host) return fail(SGMV_ERR_INVALID, "lora_delta_host: x_host and y_host are required");
        for (int32_t k = 0; k < i; ++k)
            if (e[k].y_host == e[i].y_host) return fail(SGMV_ERR_INVALID, "lora_delta_host: two entries name one y_host");
    }
    return SGMV_OK;
}

}  // namespace

extern "C" int64_t sgmv_host_workspace_bytes(int32_t T, const sgmv_pool* pool, const sgmv_host_entry* entries,
                                             int32_t n_entries, int32_t y_dtype) {
    if (T < 0 || check_host_entries(entries, n_entries, pool, y_dtype) != SGMV_OK) return -1;
    HostLayout L;
    const int64_t ldv = std::max<int64_t>(4, ((int64_t)pool->max_rank + 3) / 4 * 4);
    host_layout(entries, n_entries, T, sgmv_plan_table_capacity(T, pool->n_proj), T, ldv, y_dtype, &L);
    return L.end;
}

extern "C" sgmv_status sgmv_lora_delta_host(const int32_t* adapter_ids, int32_t T, const sgmv_pool* pool,
                                            const sgmv_host_entry* entries, int32_t n_entries, float scale,
                                            int32_t y_dtype, void* host_table, int64_t host_table_bytes,
                                            void* workspace, int64_t workspace_bytes, sgmv_plan* plan_out,
                                            int64_t* h2d_bytes, int64_t* d2h_bytes, sgmv_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    sgmv_status st = check_host_entries(entries, n_entries, pool, y_dtype);
    if (st != SGMV_OK) return st;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return fail(SGMV_ERR_INVALID, "lora_delta_host: workspace must be a 256-byte aligned device pointer");
    sgmv_plan plan;
    st = sgmv_build_plan(adapter_ids, T, pool, 0, host_table, host_table_bytes, &plan);
    if (st != SGMV_OK) return st;
    const int64_t esz = y_dtype == 0 ? 2 : 4;
    const int64_t ldv = std::max<int64_t>(4, ((int64_t)plan.max_rank + 3) / 4 * 4);
    HostLayout L;
    host_layout(entries, n_entries, T, plan.table_bytes, plan.num_rows, ldv, y_dtype, &L);
    if (L.end > workspace_bytes) return fail(SGMV_ERR_CAPACITY, "lora_delta_host: workspace too small");
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    sgmv_delta_entry de[kMaxGroup];
    for (int32_t i = 0; i < n_entries; ++i) {
        const sgmv_host_entry& e = entries[i];
        de[i] = sgmv_delta_entry{e.proj, e.d_in, e.d_out, 0, ws + L.x[i], e.d_in, ws + L.y[i], e.d_out,
                                 reinterpret_cast<float*>(ws + L.v[i]), ldv};
    }
    const void* table = plan.needs_device_table ? ws + L.table : nullptr;
    // every argument of the kernels is checked before the first copy is enqueued
    BatchView bv;
    PoolView pv;
    bool nothing = false;
    for (int32_t i = 0; i < n_entries; ++i) {
        const sgmv_delta_entry& e = de[i];
        st = check_shrink(e.x, e.ldx, T, e.d_in, e.proj, &plan, table ? table : ws + L.table, pool, e.v, e.ldv, &bv,
                          &pv, &nothing);
        if (st != SGMV_OK) return st;
        st = check_expand(e.v, e.ldv, T, e.d_out, e.proj, &plan, table ? table : ws + L.table, pool, e.y, e.ldy,
                          y_dtype, &bv, &pv, &nothing);
        if (st != SGMV_OK) return st;
    }
    int64_t in = 0, out = 0;
    if (plan.needs_device_table) {
        const sgmv_status st_up = sgmv_upload_table(&plan, ws + L.table, stream_);
        if (st_up != SGMV_OK) return st_up;
        in += plan.table_bytes;
    }
    for (int32_t i = 0; i < n_entries; ++i) {
        const sgmv_host_entry& e = entries[i];
        if (L.x_of[i] == i && T > 0) {
            SGMV_CUDA_TRY(cudaMemcpyAsync(ws + L.x[i], e.x_host, (size_t)T * e.d_in * 2, cudaMemcpyHostToDevice,
                                          stream));
            in += (int64_t)T * e.d_in * 2;
        }
        if (T > 0) {
            SGMV_CUDA_TRY(cudaMemcpyAsync(ws + L.y[i], e.y_host, (size_t)T * e.d_out * esz, cudaMemcpyHostToDevice,
                                          stream));
            in += (int64_t)T * e.d_out * esz;
        }
    }
    st = delta_impl(de, n_entries, T, &plan, table, pool, scale, y_dtype, stream);
    if (st != SGMV_OK) return st;
    for (int32_t i = 0; i < n_entries && T > 0; ++i) {
        SGMV_CUDA_TRY(cudaMemcpyAsync(entries[i].y_host, ws + L.y[i], (size_t)T * entries[i].d_out * esz,
                                      cudaMemcpyDeviceToHost, stream));
        out += (int64_t)T * entries[i].d_out * esz;
    }
    if (plan_out) *plan_out = plan;
    if (h2d_bytes) *h2d_bytes = in;
    if (d2h_bytes) *d2h_bytes = out;
    return SGMV_OK;
}

// ---------------------------------------------------------------------------
// sgmv_lora_delta without a caller workspace.
//
// Some callers cannot hand this library a device buffer for the intermediate
// v: their device memory is owned by another runtime's fixed arena, or the
// library is not allowed to grow the process's device footprint or to pay for
// cudaMalloc's device-wide synchronisation.  For them the workspace lives in
// the fixed array below, which every GPU that loads this library holds until
// the process exits.  All calls on a device share it: calls whose kernels
// overlap on that device race on it, and it keeps whatever the last call left
// (nothing in it has to start at zero -- the shrink writes every entry the
// expand then reads).
constexpr int64_t kNoAllocScratchFloats = int64_t(1) << 19;  // 2 MiB of fp32
static __device__ __align__(256) float g_noalloc_v[kNoAllocScratchFloats];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
float* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_v on the current device (looked up once per device).
sgmv_status noalloc_scratch(float** out) {
    int dev = 0;
    SGMV_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return fail(SGMV_ERR_UNSUPPORTED, "lora_delta_noalloc: device ordinal too large");
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_v);
        if (e != cudaSuccess || !p) return cuda_fail(e, "lora_delta_noalloc: cudaGetSymbolAddress");
        g_noalloc_ptr[dev] = static_cast<float*>(p);
    }
    *out = g_noalloc_ptr[dev];
    return SGMV_OK;
}
}  // namespace

extern "C" sgmv_status sgmv_lora_delta_noalloc(const void* x, int64_t ldx, int32_t T, int32_t d_in, int32_t d_out,
                                               int32_t proj, const sgmv_plan* plan, const void* table,
                                               const sgmv_pool* pool, float scale, void* y, int64_t ldy,
                                               int32_t y_dtype, sgmv_stream_t stream) {
    if (!plan) return fail(SGMV_ERR_INVALID, "lora_delta_noalloc: plan is required");
    const int64_t ldv = std::max<int64_t>(4, ((int64_t)plan->max_rank + 3) / 4 * 4);
    if ((int64_t)plan->num_rows * ldv > kNoAllocScratchFloats)
        return fail(SGMV_ERR_CAPACITY, "lora_delta_noalloc: the batch needs " +
                                           std::to_string((int64_t)plan->num_rows * ldv) +
                                           " fp32 of workspace, above the fixed " +
                                           std::to_string(kNoAllocScratchFloats) + "; use sgmv_lora_delta");
    float* v = nullptr;
    const sgmv_status st = noalloc_scratch(&v);
    if (st != SGMV_OK) return st;
    return sgmv_lora_delta(x, ldx, T, d_in, d_out, proj, plan, table, pool, scale, y, ldy, y_dtype, v, ldv, stream);
}

extern "C" sgmv_status sgmv_check_errors(sgmv_stream_t stream_, uint32_t* flags) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    uint32_t bits = 0;
    SGMV_CUDA_TRY(read_clear_errors_simt(&bits, stream));
    SGMV_CUDA_TRY(read_clear_errors_tc(&bits, stream));
    if (flags) *flags = bits;
    if (bits & kErrTimeout) return fail(SGMV_ERR_TIMEOUT, "a device-side wait timed out");
    if (bits) return fail(SGMV_ERR_BOUNDS, "a device-side bounds check failed");
    return SGMV_OK;
}
