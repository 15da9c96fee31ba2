// SIMT path of SGMV-shrink and SGMV-expand for short segments (decode).
//
// "Multi-LoRA serving: the single translator with a thousand glossaries ..."
// (blog.lo0.es), section "SGMV: the kernel that holds it all up": phase 1
// projects d_in -> r with A_{a(t)}, phase 2 projects r -> d_out with B_{a(t)};
// small segments take a batched gather path.  One launch per phase covers
// every short segment of the batch, whatever its rank, with no padded work.
//
// Decode batches move a few MB per phase, so the kernels are built around
// latency: a CTA first reads the page ids of everything it will touch in one
// round of independent loads, then keeps three or four 16 KB stages of adapter
// rows in flight with 16-byte cp.async copies issued by all threads (pages are
// 1 KiB and scattered, too fine-grained for one bulk copy per page); the token
// rows' x slices travel in the same stages.  Grids are sized to one wave of
// resident CTAs.
//
// shrink:  a thread-block cluster of C CTAs per work item (<= 4 rows of one
//          segment); CTA q owns a page-aligned share of d_in.  Stages are 8
//          rank rows x up to 1024 columns; each thread owns 8 columns; partial
//          dot products are reduced with warp shuffles and shared memory; the
//          other CTAs of the cluster push their partial tiles into rank 0's
//          shared memory, which sums them in a fixed order and writes v.
//          Deterministic, no atomics, no scratch memory.
// expand:  CTAs per work item each cover one or more 1024-column passes of
//          d_out.  Launched as a programmatic dependent of the shrink: B^T rank
//          rows are staged (and, inside sgmv_lora_delta, the first y rows read)
//          before the kernel waits for the shrink; then v of the item is read,
//          each thread accumulates its 8 output columns for up to 4 tokens and
//          updates y with one rounding, pass by pass.
// Quantised pools (template parameter WF): the stages hold E4M3 / INT4 codes
// (8 or 4 KB, filled with 16-byte copies) and each thread converts its 8
// values in registers; a rank row's scale multiplies v_k once, at the end of
// the shrink, and v_k as the expand reads it.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <type_traits>

#include "internal.h"
#include "ptx.cuh"

namespace sgmv {
namespace {

__device__ unsigned int g_err_simt;

constexpr int kThreads = 128;
constexpr int kVec = 8;                    // columns per thread
constexpr int kPass = kThreads * kVec;     // 1024 columns per stage
constexpr int kRowGroup = 8;               // rank rows per stage
// shrink ring depth by token group: 1-token items stream long adapter rows with
// 4 stages; items of 2-4 tokens carry larger x slices and keep 3 CTAs per SM
// with 3 stages
template <int MAXG>
__host__ __device__ constexpr int shrink_stages() { return MAXG == 1 ? 4 : 3; }
constexpr int kExpandStages = 3;
constexpr int kStageElems = kRowGroup * kPass;
// bytes of one stage in weight format WF (bf16 16 KB, E4M3 8 KB, INT4 4 KB)
template <int WF>
__host__ __device__ constexpr int stage_bytes() { return kStageElems / 8 * bytes_per_8<WF>(); }

// One x of a shrink launch and the nsub projections computed from it.  A launch
// covers up to kMaxGroup entries over the same batch plan (sgmv_lora_delta_grouped);
// every entry gets the same number of CTAs per item.  The A rows of an entry's
// projections are stacked in its CTAs: row group g of a CTA is row group g % NG of
// projection g / NG (NG = row groups of one projection), so the shared x slices are
// staged by one CTA for all of them.
struct ShrinkEntry {
    const uint16_t* x;
    int64_t ldx;
    float* v[kMaxShare];
    int64_t ldv[kMaxShare];
    int32_t d_in;
    int32_t kc;          // columns of d_in per CTA (multiple of the page size)
    int32_t proj[kMaxShare];
    int32_t nsub;        // projections stacked over this x (1 .. kMaxShare)
    int32_t pad;
};

template <int NE>  // entry capacity: 1 (one projection) or kMaxGroup
struct ShrinkArgs {
    ShrinkEntry ent[NE];
    int32_t n_entries;
    int32_t items;       // SIMT items of the plan (each entry's CTAs: items x cluster)
    BatchView b;         // b.proj unused: every entry names its projection
    PoolView pool;
    int32_t cluster;     // C
    int32_t stages;
    int32_t max_rank;
    int32_t ring_offset; // byte offset of the stage ring in shared memory
    int32_t nsub_max;    // largest nsub of the launch (sizes the partial tiles and page ids)
    int32_t pad;
};

struct ExpandEntry {
    const float* v;
    int64_t ldv;
    void* y;
    int64_t ldy;
    int32_t d_out;
    int32_t npass;       // 1024-column passes per CTA
    int32_t cpi;         // CTAs per item
    int32_t cta_base;    // first CTA of this entry in the grid
    int32_t proj;
    int32_t pad[3];
};

template <int NE>
struct ExpandArgs {
    ExpandEntry ent[NE];
    int32_t n_entries;
    int32_t items;
    BatchView b;
    PoolView pool;
    float scale;
    int32_t y_dtype;
    int32_t y_early;        // y may be read before the preceding kernel (the shrink) completes
    int32_t stages;
    int32_t max_rank;
    int32_t ring_offset;    // byte offset of the stage ring in shared memory
};

struct ItemInfo {
    int i0, n, r;
    int64_t pt;          // first page-table entry of the matrix for this projection
    float sc;            // multiplier of the item's adapter (read for the expand only)
    bool ok;
    int tok[kSimtMaxItemRows];  // token rows of the item (-1 past n or when out of range)
};

__device__ __forceinline__ void check_item(const BatchView& b, ItemInfo& m, int seg, int row_end, int max_rows,
                                           int max_rank) {
    m.ok = seg >= 0 && seg < b.num_segments && m.i0 >= 0 && m.n > 0 && m.n <= max_rows && row_end <= b.num_rows &&
           m.r > 0 && m.r <= max_rank;
    if (!m.ok) {
        m.n = 0;
        m.r = 0;
    }
}

__device__ __forceinline__ void finish_tokens(const BatchView& b, ItemInfo& m) {
#pragma unroll
    for (int j = 0; j < kSimtMaxItemRows; ++j) {
        if (j >= m.n) {
            m.tok[j] = -1;
        } else if (m.tok[j] < 0 || m.tok[j] >= b.T) {
            if (threadIdx.x == 0) atomicOr(&g_err_simt, kErrToken);
            m.tok[j] = -1;
        }
    }
}

// Work item `idx` from the device table: one 32-byte record, then the token rows.
__device__ __forceinline__ ItemInfo load_item(const BatchView& b, int proj, int idx, int max_rows, int max_rank,
                                              int matrix) {
    ItemInfo m;
    const int4* rp = reinterpret_cast<const int4*>(b.simt_items + ((int64_t)idx * b.n_proj + proj));
    const int4 h = rp[0], t = rp[1];  // {seg, row_begin, row_end, rank}, {a_pt, b_pt}
    m.i0 = h.y;
    m.n = h.z - h.y;
    m.r = h.w;
    check_item(b, m, h.x, h.z, max_rows, max_rank);
    m.pt = matrix == 0 ? (int64_t)(((uint64_t)(uint32_t)t.y << 32) | (uint32_t)t.x)
                       : (int64_t)(((uint64_t)(uint32_t)t.w << 32) | (uint32_t)t.z);
    m.sc = (matrix == 1 && m.ok) ? b.seg_scale[h.x] : 1.f;  // (segment checked above)
#pragma unroll
    for (int j = 0; j < kSimtMaxItemRows; ++j) m.tok[j] = j < m.n ? b.token_idx[m.i0 + j] : -1;
    finish_tokens(b, m);
    return m;
}

// Work item `idx` from the launch arguments.
template <int N>
__device__ __forceinline__ ItemInfo load_item(const BatchView& b, const InlineTable<N>& t, int idx, int max_rows,
                                              int max_rank, int matrix) {
    ItemInfo m;
    const InlineItem& it = t.items[idx];
    m.i0 = it.row_begin;
    m.n = it.row_end - it.row_begin;
    m.r = it.rank;
    check_item(b, m, it.seg, it.row_end, max_rows, max_rank);
    m.pt = matrix == 0 ? it.a_pt : it.b_pt;
    m.sc = t.scale[idx];
#pragma unroll
    for (int j = 0; j < kSimtMaxItemRows; ++j) m.tok[j] = it.tok[j];
    finish_tokens(b, m);
    return m;
}

__device__ __forceinline__ float dot8(const float (&a)[8], const float (&b)[8]) {
    float s = a[0] * b[0];
#pragma unroll
    for (int e = 1; e < 8; ++e) s = fmaf(a[e], b[e], s);
    return s;
}

// Sum N values per thread over the CTA.  Thread t < N gets the CTA-wide sum of
// value index t.  N is 8, 16, 32 or 64.
template <int N>
__device__ __forceinline__ float block_reduce(float (&vals)[N], float* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int LOGN = (N == 8) ? 3 : (N == 16) ? 4 : (N == 32) ? 5 : 6;
    constexpr int STEPS = LOGN < 5 ? LOGN : 5;
#pragma unroll
    for (int step = 0; step < STEPS; ++step) {  // transpose-reduce: halve the values a lane keeps
        const int o = 16 >> step;
        const int half = N >> (step + 1);
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = upper ? vals[i] : vals[i + half];
            const float keep = upper ? vals[i + half] : vals[i];
            vals[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, o);
        }
    }
    if constexpr (N < 32) {
#pragma unroll
        for (int o = (16 >> LOGN); o >= 1; o >>= 1) vals[0] += __shfl_xor_sync(0xFFFFFFFFu, vals[0], o);
    }
    if constexpr (N <= 32) {
        constexpr int SPAN = 32 / N;  // lanes sharing one value index
        if ((lane & (SPAN - 1)) == 0) red[warp * N + (lane >> (5 - LOGN))] = vals[0];
    } else {
        // after five steps lane l holds values i < N/32 of index l * (N/32) + i
#pragma unroll
        for (int i = 0; i < N / 32; ++i) red[warp * N + lane * (N / 32) + i] = vals[i];
    }
    __syncthreads();
    float s = 0.f;
    if (threadIdx.x < N)
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) s += red[w * N + threadIdx.x];
    __syncthreads();
    return s;
}

// Stage u of a CTA holds rank rows [8 g, 8 g + 8) x columns [c, c + W) of one
// matrix (W <= 1024), row-major with row stride W.  All 128 threads fill it
// with 16-byte cp.async copies: consecutive threads take consecutive 16-byte
// granules of a row (512 contiguous bytes per warp instruction, conflict-free
// shared-memory writes), each granule's page found in the CTA's page-id table.
// Every stage is one commit group; the prologue commits kStages groups and
// each consumed stage commits one more (possibly empty), so waiting for all but
// the newest kStages - 1 groups always means "this stage has landed".
struct StageGeom {  // rows and columns of the CTA's stages
    int NG, npass, span, col_base, rank, pages_per_row;
    int NGs;             // row groups of one stacked projection (NG = nsub * NGs; the expand: NG)
    int64_t pt;
    const int32_t* pid;  // page ids of the CTA's span, [row group][8 rank rows][chunk], in shared memory
    int span_pages;
};

// The ring: stage `issued` goes to slot `islot`, its row group / pass advance
// incrementally (row group outer for the shrink, pass outer for the expand).
template <int kStages, int WF>
struct Pipe {
    uint8_t* data;
    int issued = 0, total = 0;
    int islot = 0, cslot = 0;  // slots of the next issued / consumed stage
    int ig = 0, is = 0;        // row group and pass of the next issued stage
};

// x slices that travel with the shrink's stages: token row j's columns of the
// stage's pass go to ring[slot][j] (maxg rows per slot), so their latency is
// hidden by the same ring as the adapter rows.
struct XStage {
    uint16_t* ring;                              // null: no x slices (expand)
    const uint16_t* rows[kSimtMaxItemRows];      // start of the CTA's chunk of each token row, or null
    const uint16_t* any;                         // a valid address for zero-filled copies
    int maxg;
};

template <int kStages, int WF>
__device__ __forceinline__ void pipe_issue(const PoolView& pool, Pipe<kStages, WF>& pp, const StageGeom& sg,
                                           bool pass_outer, const XStage& xs) {
    constexpr int VB = bytes_per_8<WF>();  // bytes of 8 stored values
    const uint8_t* pages = reinterpret_cast<const uint8_t*>(pool.pages);
    if (pp.issued < pp.total) {
        const int P_log2 = pool.page_log2, P = 1 << P_log2;
        const int g = pp.ig, c = pp.is * kPass;
        const int W = min(kPass, sg.span - c);
        if (xs.ring && kVec * (int)threadIdx.x < W) {
            uint16_t* xd = xs.ring + (size_t)pp.islot * xs.maxg * kPass + kVec * threadIdx.x;
#pragma unroll
            for (int j = 0; j < kSimtMaxItemRows; ++j)
                if (j < xs.maxg)
                    cp_async16(xd + j * kPass, xs.rows[j] ? xs.rows[j] + c + kVec * threadIdx.x : xs.any,
                               xs.rows[j] != nullptr);
        }
        const int gl = g - (g / sg.NGs) * sg.NGs;  // row group within its projection
        const int rows = min(kRowGroup, sg.rank - kRowGroup * gl);
        uint8_t* dst0 = pp.data + (size_t)pp.islot * stage_bytes<WF>();
        const int32_t* pidg = sg.pid + kRowGroup * g * sg.span_pages;
        // a page is (1 << P_log2) values, (1 << page_shift) bytes; column c of it at byte c * VB / 8
        const int page_shift = P_log2 + (VB == 16 ? 1 : VB == 8 ? 0 : -1);
        if constexpr (WF != kFmtBf16) {
            // codes: 16-byte copies (16 E4M3 / 32 INT4 values; a row of the stage is W * VB / 8
            // bytes, a multiple of 32 since W is a multiple of 64), consecutive threads on
            // consecutive granules of a row; the consumers read the same bytes 8 values a thread
            constexpr int kVals16 = 128 / VB;                  // values per 16-byte granule
            const int gpr = W / kVals16;                       // granules per row
#pragma unroll
            for (int i = 0; i < stage_bytes<WF>() / 16 / kThreads; ++i) {
                const int gi = threadIdx.x + kThreads * i;
                const int kk = gi / gpr, cg = gi - kk * gpr;
                if (kk < rows) {
                    const int col = c + cg * kVals16;
                    const int32_t page = pidg[kk * sg.span_pages + (col >> P_log2)];
                    cp_async16(dst0 + (size_t)kk * (W / 8 * VB) + cg * 16,
                               pages + ((int64_t)page << page_shift) + (col & (P - 1)) / 8 * VB, true);
                }
            }
        } else if (W == kPass) {  // full pass: thread t copies granule t of each of the stage's rows
            const int col = c + kVec * threadIdx.x;
            const int32_t* pidc = pidg + (col >> P_log2);
            const uint16_t* src0 = pool.pages + (col & (P - 1));
            uint16_t* dst = reinterpret_cast<uint16_t*>(dst0) + kVec * threadIdx.x;
#pragma unroll
            for (int kk = 0; kk < kRowGroup; ++kk)
                if (kk < rows)
                    cp_async16(dst + kk * kPass, src0 + ((int64_t)pidc[kk * sg.span_pages] << P_log2), true);
        } else {
            const int gpr = W >> 3;  // granules (8 values) per row
            uint16_t* d0 = reinterpret_cast<uint16_t*>(dst0);
#pragma unroll
            for (int i = 0; i < kStageElems / 8 / kThreads; ++i) {
                const int gi = threadIdx.x + kThreads * i;
                const int kk = gi / gpr, cg = gi - kk * gpr;
                if (kk < rows) {
                    const int col = c + cg * 8;
                    const int32_t page = pidg[kk * sg.span_pages + (col >> P_log2)];
                    cp_async16(d0 + (size_t)kk * W + cg * 8, pool.pages + ((int64_t)page << P_log2) + (col & (P - 1)),
                               true);
                }
            }
        }
        if (pass_outer) {
            if (++pp.ig == sg.NG) { pp.ig = 0; ++pp.is; }
        } else {
            if (++pp.is == sg.npass) { pp.is = 0; ++pp.ig; }
        }
        pp.islot = pp.islot + 1 == kStages ? 0 : pp.islot + 1;
    }
    ++pp.issued;
    cp_async_commit();
}

template <int kStages, int WF>
__device__ __forceinline__ const uint8_t* pipe_acquire(Pipe<kStages, WF>& pp) {
    cp_async_wait<kStages - 1>();
    __syncthreads();
    return pp.data + (size_t)pp.cslot * stage_bytes<WF>();
}

template <int kStages, int WF>
__device__ __forceinline__ void pipe_release(const PoolView& pool, Pipe<kStages, WF>& pp, const StageGeom& sg,
                                             bool pass_outer, const XStage& xs) {
    __syncthreads();  // every thread is done with the slot before it is refilled
    pp.cslot = pp.cslot + 1 == kStages ? 0 : pp.cslot + 1;
    pipe_issue(pool, pp, sg, pass_outer, xs);
}

// All threads: fetch the page ids of every rank row over the CTA's column span
// into shared memory in one round of independent loads; with nsub stacked
// projections (first page-table entries pt_sub[p]), projection p's rows start at
// row p * 8 * NGs.  Out-of-range ids are flagged and replaced by page 0 (in
// bounds; the result is flagged).
__device__ void load_page_ids(const PoolView& pool, StageGeom& sg, int32_t* pid, unsigned int* err,
                              const int64_t* pt_sub = nullptr, int nsub = 1) {
    const int P_log2 = pool.page_log2;
    sg.span_pages = sg.span > 0 ? (sg.span + (1 << P_log2) - 1) >> P_log2 : 0;
    const int per = sg.rank * sg.span_pages;  // ids of one projection
    for (int i = threadIdx.x; i < nsub * per; i += kThreads) {
        const int p = i / per, ip = i - p * per;
        const int k = ip / sg.span_pages, pc = ip - k * sg.span_pages;
        const int64_t base = pt_sub ? pt_sub[p] : sg.pt;
        const int64_t e = base + (int64_t)k * sg.pages_per_row + (sg.col_base >> P_log2) + pc;
        int32_t page = (e >= 0 && e < pool.pt_capacity) ? pool.page_table[e] : -1;
        if (page < 0 || page >= pool.num_pages) {
            atomicOr(err, kErrPage);
            page = 0;
        }
        pid[(p * kRowGroup * sg.NGs + k) * sg.span_pages + pc] = page;
    }
    sg.pid = pid;
}

// Threads k < r: the scale of rank row k of a quantised matrix (kept at the
// page-table entry of the row's first chunk) into rsc[k].  An entry outside
// the table is flagged and reads as 0.
__device__ __forceinline__ void load_row_scales(const PoolView& pool, int64_t pt, int pages_per_row, int r,
                                                float* rsc, unsigned int* err) {
    for (int k = threadIdx.x; k < r; k += kThreads) {
        const int64_t e = pt + (int64_t)k * pages_per_row;
        float v = 0.f;
        if (e >= 0 && e < pool.pt_capacity) v = pool.row_scale[e];
        else atomicOr(err, kErrPage);
        rsc[k] = v;
    }
}

// ------------------------------------------------------------------ shrink
template <int G, int kStages, int WF>
__device__ void shrink_item(const PoolView& pool, const ItemInfo& m, Pipe<kStages, WF>& pp, const StageGeom& sg,
                            const XStage& xs, float* part, float* red, int nsub) {
    constexpr int VB = bytes_per_8<WF>();
    const int tid = threadIdx.x, col = kVec * tid;
    for (int g = 0; g < sg.NG; ++g) {
        const int ps = g / sg.NGs, gl = g - ps * sg.NGs;  // stacked projection, its row group
        float p[kRowGroup * G];
#pragma unroll
        for (int i = 0; i < kRowGroup * G; ++i) p[i] = 0.f;
        for (int s = 0; s < sg.npass; ++s) {
            const int c = s * kPass, W = min(kPass, sg.span - c);
            const bool active = col < W;
            const uint8_t* st = pipe_acquire(pp);
            const uint16_t* xst = xs.ring + (size_t)pp.cslot * xs.maxg * kPass + col;
            if (active) {
                float xf[G][8];
#pragma unroll
                for (int j = 0; j < G; ++j) unpack8(*reinterpret_cast<const uint4*>(xst + j * kPass), xf[j]);
                if constexpr (WF == kFmtInt4) {  // INT4 codes arrive scaled by 16^(e % 4): x takes the inverse
#pragma unroll
                    for (int j = 0; j < G; ++j)
#pragma unroll
                        for (int e = 0; e < 8; ++e) xf[j][e] *= int4_pos_unscale(e);
                }
#pragma unroll
                for (int kk = 0; kk < kRowGroup; ++kk) {
                    float af[8];
                    if constexpr (WF == kFmtBf16)
                        unpack8(*reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(st) + (size_t)kk * W + col), af);
                    else if constexpr (WF == kFmtInt4)
                        int4x8_to_f32_pos(*reinterpret_cast<const uint32_t*>(st + ((size_t)kk * (W >> 3) + tid) * VB), af);
                    else
                        load_w8<WF>(st + ((size_t)kk * (W >> 3) + tid) * VB, af);
#pragma unroll
                    for (int j = 0; j < G; ++j) p[kk * G + j] += dot8(af, xf[j]);
                }
            }
            pipe_release(pool, pp, sg, false, xs);
        }
        const float sum = block_reduce<kRowGroup * G>(p, red);
        if (tid < kRowGroup * G) {  // partial tile [token j][projection ps][rank row]
            const int kk = tid / G, j = tid - (tid / G) * G;
            if (kRowGroup * gl + kk < m.r && j < m.n) part[(j * nsub + ps) * m.r + kRowGroup * gl + kk] = sum;
        }
    }
}

template <int MAXG, int NI, int NE, int WF>
__global__ void __launch_bounds__(kThreads, 3)
    shrink_simt_kernel(const __grid_constant__ ShrinkArgs<NE> a, const __grid_constant__ InlineTable<NI> inl) {
    extern __shared__ __align__(128) uint8_t smem[];
    pdl_launch_dependents();  // the expand may start staging its B^T pages now
    const int C = a.cluster;
    // First cluster phase: every CTA has started.  Its wait, just before the
    // partial tiles are pushed, makes rank 0's shared memory a valid target.
    if (C > 1) cluster_arrive_relaxed();
    const int per_entry = a.items * C;  // a multiple of C: no cluster straddles two entries
    const int ei = NE == 1 ? 0 : (int)blockIdx.x / per_entry;
    const ShrinkEntry& en = a.ent[ei];
    const int item_idx = ((int)blockIdx.x - ei * per_entry) / C;
    const uint32_t q = cluster_ctarank();
    const int nsub = NI > 1 ? 1 : en.nsub;                 // projections stacked over this x
    const int slot = kSimtMaxItemRows * a.max_rank * a.nsub_max;  // floats of one partial tile
    float* part = reinterpret_cast<float*>(smem);     // [C slots][slot]; slot 0 is this CTA's own
    float* red = part + C * slot;                      // [4 warps][64]
    float* rsc = red + 4 * 64;                         // [nsub][kMaxRank] row scales (quantised pools only)
    int32_t* pid = reinterpret_cast<int32_t*>(rsc + (WF == kFmtBf16 ? 0 : a.nsub_max * kMaxRank));
    __shared__ int64_t pt_sub[kMaxShare];              // first page-table entry of A, per stacked projection

    // the stacked projections' A bases come from their own records of this item (loaded
    // alongside the item's first record; every projection of an item has its rows and rank)
    if (NI == 1 && (int)threadIdx.x < nsub) {
        const int4 t = reinterpret_cast<const int4*>(
            a.b.simt_items + ((int64_t)item_idx * a.b.n_proj + en.proj[threadIdx.x]))[1];
        pt_sub[threadIdx.x] = (int64_t)(((uint64_t)(uint32_t)t.y << 32) | (uint32_t)t.x);
    }
    const ItemInfo m = NI > 1 ? load_item(a.b, inl, item_idx, MAXG, a.max_rank, 0)
                              : load_item(a.b, en.proj[0], item_idx, MAXG, a.max_rank, 0);
    if (NI > 1 && threadIdx.x == 0) pt_sub[0] = m.pt;
    if (!m.ok && threadIdx.x == 0) atomicOr(&g_err_simt, kErrRows);
    StageGeom sg;
    sg.NGs = (m.r + kRowGroup - 1) / kRowGroup;
    sg.NG = nsub * sg.NGs;
    sg.span = en.kc;
    sg.npass = (en.kc + kPass - 1) / kPass;
    sg.col_base = (int)q * en.kc;
    sg.rank = m.r;
    sg.pages_per_row = en.d_in >> a.pool.page_log2;
    sg.pt = m.pt;
    constexpr int kShrinkStages = shrink_stages<MAXG>();
    Pipe<kShrinkStages, WF> pp;
    pp.data = smem + a.ring_offset;
    pp.total = m.ok ? sg.NG * sg.npass : 0;
    XStage xs;
    xs.ring = reinterpret_cast<uint16_t*>(pp.data + (size_t)kShrinkStages * stage_bytes<WF>());
    xs.maxg = MAXG;
    xs.any = en.x;
#pragma unroll
    for (int j = 0; j < kSimtMaxItemRows; ++j)
        xs.rows[j] = (j < MAXG && m.tok[j] >= 0) ? en.x + (int64_t)m.tok[j] * en.ldx + (int64_t)q * en.kc : nullptr;
    __syncthreads();  // pt_sub
    if (m.ok) load_page_ids(a.pool, sg, pid, &g_err_simt, pt_sub, nsub);
    if (WF != kFmtBf16 && m.ok && q == 0)
        for (int ps = 0; ps < nsub; ++ps)
            load_row_scales(a.pool, pt_sub[ps], sg.pages_per_row, m.r, rsc + ps * kMaxRank, &g_err_simt);
    __syncthreads();
#pragma unroll 1
    for (int i = 0; i < kShrinkStages; ++i) pipe_issue(a.pool, pp, sg, false, xs);
    if (m.ok) {  // MAXG bounds the token group, and with it the registers of the launch
        if (MAXG == 1 || m.n == 1) shrink_item<1, kShrinkStages>(a.pool, m, pp, sg, xs, part, red, nsub);
        else if (MAXG == 2 || m.n == 2)
            shrink_item<(MAXG < 2 ? MAXG : 2), kShrinkStages>(a.pool, m, pp, sg, xs, part, red, nsub);
        else shrink_item<MAXG, kShrinkStages>(a.pool, m, pp, sg, xs, part, red, nsub);
    }
    cp_async_wait<0>();

    // Sum the C partial tiles in a fixed order.  Every CTA but rank 0 pushes its
    // tile into slot q of rank 0's shared memory and arrives on the cluster
    // barrier without waiting (it may then exit: nobody reads its memory); rank 0
    // arrives, waits for all, sums slots 0..C-1 and writes v.  Slot 0 is rank 0's
    // own tile, so the order of the sum is fixed.
    const int RS = nsub * m.r;  // values of one token row of the tile: [projection][rank row]
    const int E = m.n * RS;
    __syncthreads();  // part[] complete in this CTA
    if (C > 1) {
        cluster_wait_acquire();
        if (q != 0) {
            if (m.ok) {
                const uint32_t dst = map_cluster(smem_u32(part + (size_t)q * slot), 0u);
                for (int e = threadIdx.x; e < E; e += kThreads) st_cluster_f32(dst + 4u * (uint32_t)e, part[e]);
            }
            cluster_arrive_release();
            return;
        }
        cluster_arrive_release();
        cluster_wait_acquire();
    }
    if (m.ok) {
        for (int e = threadIdx.x; e < E; e += kThreads) {
            float s = 0.f;
            for (int qq = 0; qq < C; ++qq) s += part[(size_t)qq * slot + e];
            const int jrow = e / RS, rem = e - jrow * RS;
            const int ps = rem / m.r, k = rem - ps * m.r;
            // a quantised row's scale leaves the sum: v_k = s_k * sum_c q_kc x_c
            en.v[ps][(int64_t)(m.i0 + jrow) * en.ldv[ps] + k] = WF == kFmtBf16 ? s : s * rsc[ps * kMaxRank + k];
        }
    }
}

// ------------------------------------------------------------------ expand
template <int G, int NE, int WF, int YT>  // YT: y type, 0 = bf16, 1 = fp32
__device__ void expand_item(const ExpandArgs<NE>& a, const ExpandEntry& en, const ItemInfo& m,
                            Pipe<kExpandStages, WF>& pp, const StageGeom& sg, float* vs, const float* rsc) {
    constexpr int VB = bytes_per_8<WF>();
    const int tid = threadIdx.x, col = kVec * tid;
    const float sc = a.scale * m.sc;  // the call's scale times the adapter's
    int trow[G];
#pragma unroll
    for (int j = 0; j < G; ++j) trow[j] = m.tok[j];
    // y of a pass is loaded one pass ahead of its update (two buffers)
    // (bf16 y: the 16 bytes live in the first float4; the second is used for fp32 y only)
    float4 y0[G], y1[G], n0[G], n1[G];
    auto load_y = [&](int s, float4 (&d0)[G], float4 (&d1)[G]) {
        const int c = s * kPass, jcol = sg.col_base + c + col;
        const bool active = col < min(kPass, sg.span - c);
#pragma unroll
        for (int j = 0; j < G; ++j) {
            if (active && trow[j] >= 0) {
                if constexpr (YT == 0) {
                    d0[j] = *reinterpret_cast<const float4*>(static_cast<const uint16_t*>(en.y) +
                                                             (int64_t)trow[j] * en.ldy + jcol);
                } else {
                    const float* yp = static_cast<const float*>(en.y) + (int64_t)trow[j] * en.ldy + jcol;
                    d0[j] = *reinterpret_cast<const float4*>(yp);
                    d1[j] = *reinterpret_cast<const float4*>(yp + 4);
                }
            }
        }
    };
    if (a.y_early) load_y(0, y0, y1);
    pdl_wait();  // v (and, unless y_early, y) are final once the preceding kernel has completed
    for (int e = tid; e < m.n * m.r; e += kThreads) {
        const int jrow = e / m.r, k = e - jrow * m.r;
        const float vk = en.v[(int64_t)(m.i0 + jrow) * en.ldv + k];
        vs[e] = WF == kFmtBf16 ? vk : vk * rsc[k];  // a quantised B^T row's scale goes onto v_k
    }
    // (the first pipe_acquire's barrier publishes vs)
    for (int s = 0; s < sg.npass; ++s) {
        const int c = s * kPass, W = min(kPass, sg.span - c);
        const bool active = col < W;
        const int jcol = sg.col_base + c + col;
        if (s == 0 && !a.y_early) load_y(0, y0, y1);
        if (s + 1 < sg.npass) load_y(s + 1, n0, n1);
        float acc[G][8];
#pragma unroll
        for (int j = 0; j < G; ++j)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[j][e] = 0.f;
        for (int g = 0; g < sg.NG; ++g) {
            const uint8_t* st = pipe_acquire(pp);
            if (active) {
#pragma unroll
                for (int kk = 0; kk < kRowGroup; ++kk) {
                    const int k = kRowGroup * g + kk;
                    if (k < m.r) {
                        float bf[8];
                        if constexpr (WF == kFmtBf16)
                            unpack8(*reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(st) + (size_t)kk * W + col), bf);
                        else if constexpr (WF == kFmtInt4)  // scaled by 16^(e % 4), undone on the sums
                            int4x8_to_f32_pos(*reinterpret_cast<const uint32_t*>(st + ((size_t)kk * (W >> 3) + tid) * VB), bf);
                        else
                            load_w8<WF>(st + ((size_t)kk * (W >> 3) + tid) * VB, bf);
#pragma unroll
                        for (int j = 0; j < G; ++j) {
                            const float w = vs[min(j, m.n - 1) * m.r + k];
#pragma unroll
                            for (int e = 0; e < 8; ++e) acc[j][e] = fmaf(w, bf[e], acc[j][e]);
                        }
                    }
                }
            }
            pipe_release(a.pool, pp, sg, true, XStage{});
        }
        if constexpr (WF == kFmtInt4) {
#pragma unroll
            for (int j = 0; j < G; ++j)
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[j][e] *= int4_pos_unscale(e);
        }
#pragma unroll
        for (int j = 0; j < G; ++j) {
            if (!active || trow[j] < 0) continue;
            if constexpr (YT == 0) {
                float yv[8];
                const float4 q = y0[j];
                unpack8(make_uint4(__float_as_uint(q.x), __float_as_uint(q.y), __float_as_uint(q.z),
                                   __float_as_uint(q.w)), yv);
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float lo = fmaf(sc, acc[j][2 * e], yv[2 * e]);
                    const float hi = fmaf(sc, acc[j][2 * e + 1], yv[2 * e + 1]);
                    w[e] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
                           ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
                }
                *reinterpret_cast<uint4*>(static_cast<uint16_t*>(en.y) + (int64_t)trow[j] * en.ldy + jcol) =
                    make_uint4(w[0], w[1], w[2], w[3]);
            } else {
                float* yp = static_cast<float*>(en.y) + (int64_t)trow[j] * en.ldy + jcol;
                float4 o0 = y0[j], o1 = y1[j];
                o0.x = fmaf(sc, acc[j][0], o0.x); o0.y = fmaf(sc, acc[j][1], o0.y);
                o0.z = fmaf(sc, acc[j][2], o0.z); o0.w = fmaf(sc, acc[j][3], o0.w);
                o1.x = fmaf(sc, acc[j][4], o1.x); o1.y = fmaf(sc, acc[j][5], o1.y);
                o1.z = fmaf(sc, acc[j][6], o1.z); o1.w = fmaf(sc, acc[j][7], o1.w);
                *reinterpret_cast<float4*>(yp) = o0;
                *reinterpret_cast<float4*>(yp + 4) = o1;
            }
        }
#pragma unroll
        for (int j = 0; j < G; ++j) {
            y0[j] = n0[j];
            if constexpr (YT == 1) y1[j] = n1[j];
        }
    }
}

template <int MAXG, int NI, int NE, int WF, int YT>
__global__ void __launch_bounds__(kThreads, 4)
    expand_simt_kernel(const __grid_constant__ ExpandArgs<NE> a, const __grid_constant__ InlineTable<NI> inl) {
    extern __shared__ __align__(128) uint8_t smem_e[];
    int ei = 0;  // this CTA's entry: the last whose first CTA is at or before it
    if (NE > 1)
        while (ei + 1 < a.n_entries && (int)blockIdx.x >= a.ent[ei + 1].cta_base) ++ei;
    const ExpandEntry& en = a.ent[ei];
    const int local = (int)blockIdx.x - en.cta_base;
    const int part_idx = local % en.cpi, item_idx = local / en.cpi;
    float* vs = reinterpret_cast<float*>(smem_e);
    float* rsc = vs + kSimtMaxItemRows * a.max_rank;  // [kMaxRank] row scales (quantised pools only)
    int32_t* pid = reinterpret_cast<int32_t*>(rsc + (WF == kFmtBf16 ? 0 : kMaxRank));

    const ItemInfo m = NI > 1 ? load_item(a.b, inl, item_idx, MAXG, a.max_rank, 1)
                              : load_item(a.b, en.proj, item_idx, MAXG, a.max_rank, 1);
    const int j0 = part_idx * en.npass * kPass;
    StageGeom sg;
    sg.NG = (m.r + kRowGroup - 1) / kRowGroup;
    sg.NGs = sg.NG;
    sg.span = min(en.npass * kPass, en.d_out - j0);
    sg.npass = (sg.span + kPass - 1) / kPass;
    sg.col_base = j0;
    sg.rank = m.r;
    sg.pages_per_row = en.d_out >> a.pool.page_log2;
    sg.pt = m.pt;
    const bool work = m.ok && sg.span > 0;
    Pipe<kExpandStages, WF> pp;
    pp.data = smem_e + a.ring_offset;
    pp.total = work ? sg.NG * sg.npass : 0;
    if (work) load_page_ids(a.pool, sg, pid, &g_err_simt);
    if (WF != kFmtBf16 && work) load_row_scales(a.pool, m.pt, sg.pages_per_row, m.r, rsc, &g_err_simt);
    __syncthreads();
    // B^T pages do not depend on the shrink: start them before waiting for it
#pragma unroll 1
    for (int i = 0; i < kExpandStages; ++i) pipe_issue(a.pool, pp, sg, true, XStage{});
    if (!work) {
        pdl_wait();
        if (threadIdx.x == 0 && !m.ok) atomicOr(&g_err_simt, kErrRows);
        cp_async_wait<0>();
        return;
    }
    if (MAXG == 1 || m.n == 1) expand_item<1, NE, WF, YT>(a, en, m, pp, sg, vs, rsc);
    else if (MAXG == 2 || m.n == 2) expand_item<(MAXG < 2 ? MAXG : 2), NE, WF, YT>(a, en, m, pp, sg, vs, rsc);
    else expand_item<MAXG, NE, WF, YT>(a, en, m, pp, sg, vs, rsc);
    cp_async_wait<0>();
}

// ------------------------------------------------------------------ one-shot fused decode
// A decode-sized call (one projection; every SIMT item's cluster resident in one wave; a
// CTA's slices of A, x, B^T and y small enough to stage whole) runs both phases in one
// kernel.  A cluster of C CTAs per item: CTA q owns d_in columns [q kc, (q+1) kc) and d_out
// columns [q ko, (q+1) ko).  After one round of page-id loads every CTA issues all of its
// copies at once -- A rows and x slices as one commit group, B^T rows and y rows as a second
// -- so the whole call pays one DRAM round trip for its data.  The shrink's partial tile is
// pushed to every CTA of the cluster (distributed shared memory); after the cluster barrier
// each CTA sums the C tiles in a fixed order and runs its share of the expand from shared
// memory.
//
// Eight warps a CTA:
//   shrink: mma_shrink_slab over the staged A and x slices (XOR-swizzled granules); a quantised
//           pool's A codes land in row order and are converted once into the bf16 slab (exact).
//   expand: thread t owns 4 columns of the slice and runs over every rank row with FMA,
//           converting a quantised B^T row's codes in registers; v is kept transposed,
//           [rank row][4 tokens] (with the B^T row's scale folded in), so one 16-byte load
//           gives the row's weights for every token of the item.  (An mma expand, with v
//           split into bf16 hi + lo, was measured twice as slow: each tile needs two dependent
//           mma, and the legacy warp-level mma's latency dominates a phase this short.)
struct FusedArgs {
    const uint16_t* x;
    int64_t ldx;
    float* v;
    int64_t ldv;
    void* y;
    int64_t ldy;
    BatchView b;
    PoolView pool;
    int32_t d_in, d_out;
    int32_t kc, ko;          // d_in / d_out columns per CTA (multiples of the page size)
    int32_t proj;
    int32_t cluster;         // C
    int32_t max_rank;        // rank capacity of the shared-memory tiles (>= 8)
    int32_t y_dtype;
    float scale;
    // byte offsets in shared memory
    int32_t off_part, off_vs, off_rsc, off_pid_a, off_pid_b, off_a, off_ac, off_x, off_b, off_y, off_wp;
};

// The cells of a rows x cols grid that thread `start` visits with stride `stride` in
// row-major order: (k, c), advanced without a division per step.
struct GridWalk {
    int k, c, dk, dc, cols;
    __device__ __forceinline__ GridWalk(int cols_, int start, int stride) : cols(cols_) {
        k = start / cols;
        c = start - k * cols;
        dk = stride / cols;
        dc = stride - dk * cols;
    }
    __device__ __forceinline__ void next() {
        k += dk;
        c += dc;
        if (c >= cols) {
            c -= cols;
            ++k;
        }
    }
};

// The shrink of a CTA's staged bf16 slab on warp-level bf16 mma (m16n8k16, fp32
// accumulation): A rows [r][kc] and token rows x [MAXG][kc] in shared memory at As_u / xs_u,
// both with 16-byte granule c of row k stored at granule c ^ (k % 8), so that the ldmatrix row
// reads are conflict-free.  M = rank rows (16 a tile, up to MT_MAX tiles), N = tokens (8: the
// item's <= 4 and padding), K = 16 columns; warp w takes K steps w, w + W, ... with two
// accumulator sets, and the W warp tiles are summed in warp order into tile[j * r + k] (j < n,
// k < r).  Three instructions per 16 x 16 block of A replace some thirty FMA, conversion and
// shared-memory instructions.  wpart: W x MAXG x ldw floats of scratch.  Every thread of the
// CTA calls it (it holds a barrier); `ok` false leaves the tile untouched.
template <int MAXG, int W, int MT_MAX>
__device__ __forceinline__ void mma_shrink_slab(uint32_t As_u, uint32_t xs_u, int kc, int r, int n, bool ok,
                                                float* wpart, int ldw, float* tile) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (ok) {
        const int MT = (r + 15) >> 4, ksteps = kc >> 4;
        float d[MT_MAX][4], d1[MT_MAX][4];
#pragma unroll
        for (int mt = 0; mt < MT_MAX; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) d[mt][i] = d1[mt][i] = 0.f;
        // lane addresses: x rows are the tokens (padding lanes read row 0; their columns of D
        // are not used), A rows the rank rows of each tile (rows past r read row 0)
        const int mi = lane >> 3;
        const int xrow = (lane & 7) < MAXG ? (lane & 7) : 0;
        const uint32_t xbase = xs_u + (uint32_t)(xrow * kc * 2);
        uint32_t arow[MT_MAX];
        int asw[MT_MAX];
#pragma unroll
        for (int mt = 0; mt < MT_MAX; ++mt) {
            int row = mt * 16 + ((mi & 1) << 3) + (lane & 7);
            row = row < r ? row : 0;
            arow[mt] = As_u + (uint32_t)(row * kc * 2);
            asw[mt] = row & 7;
        }
        for (int ks = warp; ks < ksteps; ks += 2 * W) {
            const int ks1 = ks + W;
            const bool two = ks1 < ksteps;
            uint32_t xb[2], xb1[2];
            ldsm_x2(xbase + ((((ks << 1) | (mi & 1)) ^ (xrow & 7)) << 4), xb);
            if (two) ldsm_x2(xbase + ((((ks1 << 1) | (mi & 1)) ^ (xrow & 7)) << 4), xb1);
#pragma unroll
            for (int mt = 0; mt < MT_MAX; ++mt) {
                if (mt < MT) {
                    uint32_t af[4], af1[4];
                    ldsm_x4(arow[mt] + ((((ks << 1) | (mi >> 1)) ^ asw[mt]) << 4), af);
                    if (two) ldsm_x4(arow[mt] + ((((ks1 << 1) | (mi >> 1)) ^ asw[mt]) << 4), af1);
                    mma_bf16_16816(d[mt], af, xb[0], xb[1]);
                    if (two) mma_bf16_16816(d1[mt], af1, xb1[0], xb1[1]);
                }
            }
        }
        // warp tiles: d[mt] = {(row 16mt + g, tokens 2t, 2t+1), (row 16mt + g + 8, same tokens)}
        const int g = lane >> 2, t2 = 2 * (lane & 3);
#pragma unroll
        for (int mt = 0; mt < MT_MAX; ++mt) {
            if (mt < MT) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int k = mt * 16 + g + ((i >> 1) << 3), j = t2 + (i & 1);
                    if (j < MAXG && k < r) wpart[(warp * MAXG + j) * ldw + k] = d[mt][i] + d1[mt][i];
                }
            }
        }
    }
    __syncthreads();
    if (ok)
        for (int e = tid; e < n * r; e += W * 32) {
            const int j = e / r, k = e - j * r;
            float sum = 0.f;
#pragma unroll
            for (int w = 0; w < W; ++w) sum += wpart[(w * MAXG + j) * ldw + k];
            tile[e] = sum;
        }
}

// Four stored weights of format WF, values c .. c + 3 of a row (c a multiple of 4), to fp32,
// exactly: bf16 halves, E4M3 pairs through the hardware E4M3x2 -> f16x2 conversion, INT4
// nibbles (two's complement, value i in bits 4i .. 4i + 3 of the pair of bytes).
template <int WF>
__device__ __forceinline__ void load_w4(const uint8_t* row, int c, float (&f)[4]) {
    if constexpr (WF == kFmtBf16) {
        const uint2 w = *reinterpret_cast<const uint2*>(row + (size_t)c * 2);
        f[0] = bf16lo(w.x); f[1] = bf16hi(w.x); f[2] = bf16lo(w.y); f[3] = bf16hi(w.y);
    } else if constexpr (WF == kFmtFp8) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(row + c);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t hh;
            asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(hh) : "h"((uint16_t)(w >> (16 * h))));
            float lo, hi;
            asm("cvt.f32.f16 %0, %1;" : "=f"(lo) : "h"((uint16_t)(hh & 0xFFFFu)));
            asm("cvt.f32.f16 %0, %1;" : "=f"(hi) : "h"((uint16_t)(hh >> 16)));
            f[2 * h] = lo;
            f[2 * h + 1] = hi;
        }
    } else {
        const uint32_t w = (uint32_t)*reinterpret_cast<const uint16_t*>(row + c / 2) ^ 0x8888u;
#pragma unroll
        for (int i = 0; i < 4; ++i) f[i] = __uint_as_float(0x4B000000u | ((w >> (4 * i)) & 0xFu)) - 8388616.0f;
    }
}

constexpr int kFusedThreads = 2 * kThreads;  // eight warps, two a scheduler
constexpr int kFusedMaxRank = 64;             // four 16-row mma tiles

template <int MAXG, int NI, int WF>
__global__ void __launch_bounds__(kFusedThreads, 1)
    fused_simt_kernel(const __grid_constant__ FusedArgs a, const __grid_constant__ InlineTable<NI> inl) {
    extern __shared__ __align__(128) uint8_t smem_f[];
    constexpr int VB = bytes_per_8<WF>();
    constexpr int TPB = kFusedThreads;
    constexpr int kWarps = TPB / 32;
    constexpr int kMT = kFusedMaxRank / 16;  // 16-row tiles of the largest rank
    const int tid = threadIdx.x;
    const int C = a.cluster;
    // every CTA of the cluster is running before any pushes into another's shared memory
    if (C > 1) cluster_arrive_relaxed();
    const int item_idx = (int)blockIdx.x / C;
    const uint32_t q = cluster_ctarank();
    float* part = reinterpret_cast<float*>(smem_f + a.off_part);         // [C][4 x max_rank]
    float* vs = reinterpret_cast<float*>(smem_f + a.off_vs);             // [max_rank][4 tokens]
    float* rsc_a = reinterpret_cast<float*>(smem_f + a.off_rsc);         // [kMaxRank] (quantised)
    float* rsc_b = rsc_a + kMaxRank;
    int32_t* pid_a = reinterpret_cast<int32_t*>(smem_f + a.off_pid_a);  // [r][kc / P]
    int32_t* pid_b = reinterpret_cast<int32_t*>(smem_f + a.off_pid_b);  // [r][ko / P]
    uint16_t* As = reinterpret_cast<uint16_t*>(smem_f + a.off_a);        // [r][kc] bf16, swizzled
    uint8_t* Ac = smem_f + a.off_ac;                                     // [r][kc] codes (quantised)
    uint16_t* xs = reinterpret_cast<uint16_t*>(smem_f + a.off_x);        // [MAXG][kc] bf16, swizzled
    uint8_t* Bs = smem_f + a.off_b;                                      // [r][ko] weights
    uint8_t* ys = smem_f + a.off_y;                                      // [MAXG][ko] of y's type
    float* wpart = reinterpret_cast<float*>(smem_f + a.off_wp);          // [warps][MAXG][max_rank]
    const int slot = kSimtMaxItemRows * a.max_rank;

    ItemInfo ma = NI > 1 ? load_item(a.b, inl, item_idx, MAXG, a.max_rank, 0)
                         : load_item(a.b, a.proj, item_idx, MAXG, a.max_rank, 0);
    const ItemInfo mb = NI > 1 ? load_item(a.b, inl, item_idx, MAXG, a.max_rank, 1)
                               : load_item(a.b, a.proj, item_idx, MAXG, a.max_rank, 1);
    if (!ma.ok && tid == 0) atomicOr(&g_err_simt, kErrRows);
    const int r = ma.r, n = ma.n;
    const int P_log2 = a.pool.page_log2, P = 1 << P_log2;
    const int ppr_a = a.d_in >> P_log2, ppr_b = a.d_out >> P_log2;
    const int cpa = a.kc >> P_log2, cpb = a.ko >> P_log2;  // pages of a row in this CTA's slices
    const int ca0 = (int)q * a.kc, cb0 = (int)q * a.ko;     // first column of the slices

    // page ids of both slices (one round of independent loads), row scales of quantised pools
    if (ma.ok) {
        for (int i = tid; i < r * (cpa + cpb); i += TPB) {
            const bool isa = i < r * cpa;
            const int ii = isa ? i : i - r * cpa, cp = isa ? cpa : cpb;
            const int k = ii / cp, pc = ii - k * cp;
            const int64_t e = isa ? ma.pt + (int64_t)k * ppr_a + (ca0 >> P_log2) + pc
                                  : mb.pt + (int64_t)k * ppr_b + (cb0 >> P_log2) + pc;
            int32_t page = (e >= 0 && e < a.pool.pt_capacity) ? a.pool.page_table[e] : -1;
            if (page < 0 || page >= a.pool.num_pages) {
                atomicOr(&g_err_simt, kErrPage);
                page = 0;
            }
            (isa ? pid_a : pid_b)[ii] = page;
        }
        if (WF != kFmtBf16) {
            load_row_scales(a.pool, ma.pt, ppr_a, r, rsc_a, &g_err_simt);
            load_row_scales(a.pool, mb.pt, ppr_b, r, rsc_b, &g_err_simt);
        }
    }
    __syncthreads();

    // every copy at once: group 1 = A rows + x slices, group 2 = B^T rows + y rows.  Granule c
    // of a bf16 A or x row k lands at granule c ^ (k % 8) of the row; quantised A codes land
    // in row order and are converted into the swizzled bf16 slab below.
    const uint8_t* pages = reinterpret_cast<const uint8_t*>(a.pool.pages);
    const int page_shift = P_log2 + (VB == 16 ? 1 : VB == 8 ? 0 : -1);
    constexpr int kVals16 = 128 / VB;  // values per 16-byte granule
    const int gx = a.kc / 8;           // 16-byte granules of an x row slice (and of a bf16 A row)
    if (ma.ok) {
        const int gpr_a = a.kc / kVals16;
        for (GridWalk w(gpr_a, tid, TPB); w.k < r; w.next()) {
            const int cl = w.c * kVals16;
            const uint8_t* src = pages + ((int64_t)pid_a[w.k * cpa + (cl >> P_log2)] << page_shift) + (cl & (P - 1)) / 8 * VB;
            if constexpr (WF == kFmtBf16)
                cp_async16(As + (size_t)w.k * a.kc + (w.c ^ (w.k & 7)) * 8, src, true);
            else
                cp_async16(Ac + (size_t)w.k * (a.kc / 8 * VB) + w.c * 16, src, true);
        }
#pragma unroll
        for (int j = 0; j < MAXG; ++j) {
            const int t = ma.tok[j];
            for (int cg = tid; cg < gx; cg += TPB)
                cp_async16(xs + (size_t)j * a.kc + (cg ^ (j & 7)) * 8,
                           t >= 0 ? a.x + (int64_t)t * a.ldx + ca0 + cg * 8 : a.x, t >= 0);
        }
    }
    cp_async_commit();
    const int esz = a.y_dtype == 0 ? 2 : 4;
    if (ma.ok) {
        const int gpr_b = a.ko / kVals16;
        for (GridWalk w(gpr_b, tid, TPB); w.k < r; w.next()) {
            const int cl = w.c * kVals16;
            cp_async16(Bs + (size_t)w.k * (a.ko / 8 * VB) + w.c * 16,
                       pages + ((int64_t)pid_b[w.k * cpb + (cl >> P_log2)] << page_shift) + (cl & (P - 1)) / 8 * VB,
                       true);
        }
        const int gy = a.ko * esz / 16;  // granules of one y row slice
        const uint8_t* src = static_cast<const uint8_t*>(a.y);
#pragma unroll
        for (int j = 0; j < MAXG; ++j) {
            const int t = mb.tok[j];
            for (int cg = tid; cg < gy; cg += TPB)
                cp_async16(ys + (size_t)j * a.ko * esz + cg * 16,
                           t >= 0 ? src + ((int64_t)t * a.ldy + cb0) * esz + cg * 16 : src, t >= 0);
        }
    }
    cp_async_commit();

    // ---- shrink over this CTA's d_in slice
    cp_async_wait<1>();
    __syncthreads();
    if constexpr (WF != kFmtBf16) {  // codes -> bf16 (exact for E4M3 and INT4), 8 values a granule
        if (ma.ok)
            for (GridWalk w(gx, tid, TPB); w.k < r; w.next()) {
                float f[8];
                const uint8_t* cp = Ac + (size_t)w.k * (a.kc / 8 * VB) + (size_t)w.c * VB;
                if constexpr (WF == kFmtFp8) fp8x8_to_f32(*reinterpret_cast<const uint2*>(cp), f);
                else int4x8_to_f32(*reinterpret_cast<const uint32_t*>(cp), f);
                *reinterpret_cast<uint4*>(As + (size_t)w.k * a.kc + (w.c ^ (w.k & 7)) * 8) =
                    make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                               pack_bf16x2(f[6], f[7]));
            }
        __syncthreads();
    }
    float* mine = part + (size_t)q * slot;  // this CTA's partial tile [token][rank row]
    mma_shrink_slab<MAXG, kWarps, kMT>(smem_u32(As), smem_u32(xs), a.kc, r, n, ma.ok, wpart, a.max_rank, mine);
    __syncthreads();  // this CTA's partial tile is complete

    // ---- push the tile to every other CTA of the cluster, then sum the C tiles in order
    const int E = n * r;
    if (C > 1) {
        cluster_wait_acquire();  // (first phase: every CTA of the cluster has started)
        for (int qq = 0; qq < C; ++qq) {
            if (qq == (int)q) continue;
            const uint32_t dst = map_cluster(smem_u32(mine), (uint32_t)qq);
            for (int e = tid; e < E; e += TPB) st_cluster_f32(dst + 4u * (uint32_t)e, mine[e]);
        }
        cluster_arrive_release();
        cluster_wait_acquire();
    }
    if (ma.ok) {
        for (int e = tid; e < E; e += TPB) {
            float s = 0.f;
            for (int qq = 0; qq < C; ++qq) s += part[(size_t)qq * slot + e];
            const int k = e - (e / r) * r;
            const float vk = WF == kFmtBf16 ? s : s * rsc_a[k];  // a quantised A row's scale leaves the sum
            if (q == 0) a.v[(int64_t)(ma.i0 + e / r) * a.ldv + k] = vk;
            vs[k * 4 + e / r] = WF == kFmtBf16 ? vk : vk * rsc_b[k];  // [rank row][token]; B^T row's scale
        }
    }
    cp_async_wait<0>();
    __syncthreads();  // vs, and the B^T and y slices, are visible to every thread

    // ---- expand over this CTA's d_out slice: 4 columns a thread, every rank row
    if (!mb.ok) return;
    const float sc = a.scale * mb.sc;  // the call's scale times the adapter's
    const size_t brow = (size_t)a.ko / 8 * VB;  // bytes of a B^T row slice
    for (int c4 = tid; c4 < (a.ko >> 2); c4 += TPB) {
        float acc[MAXG][4];
#pragma unroll
        for (int j = 0; j < MAXG; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
#pragma unroll 4
        for (int k = 0; k < r; ++k) {
            float b4[4];
            load_w4<WF>(Bs + (size_t)k * brow, 4 * c4, b4);
            const float4 w = *reinterpret_cast<const float4*>(vs + k * 4);
            const float wj[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int j = 0; j < MAXG; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[j][e] = fmaf(wj[j], b4[e], acc[j][e]);
        }
        const int jcol = cb0 + 4 * c4;
#pragma unroll
        for (int j = 0; j < MAXG; ++j) {
            const int t = mb.tok[j];
            if (j >= n || t < 0) continue;
            if (a.y_dtype == 0) {
                const uint2 yv = *reinterpret_cast<const uint2*>(ys + ((size_t)j * a.ko + 4 * c4) * 2);
                *reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.y) + (int64_t)t * a.ldy + jcol) =
                    make_uint2(pack_bf16x2(fmaf(sc, acc[j][0], bf16lo(yv.x)), fmaf(sc, acc[j][1], bf16hi(yv.x))),
                               pack_bf16x2(fmaf(sc, acc[j][2], bf16lo(yv.y)), fmaf(sc, acc[j][3], bf16hi(yv.y))));
            } else {
                float4 o = *reinterpret_cast<const float4*>(ys + ((size_t)j * a.ko + 4 * c4) * 4);
                o.x = fmaf(sc, acc[j][0], o.x); o.y = fmaf(sc, acc[j][1], o.y);
                o.z = fmaf(sc, acc[j][2], o.z); o.w = fmaf(sc, acc[j][3], o.w);
                *reinterpret_cast<float4*>(static_cast<float*>(a.y) + (int64_t)t * a.ldy + jcol) = o;
            }
        }
    }
}

// ------------------------------------------------------------------ one-shot shrink (bf16)
// The shrink of a single x over bf16 pools when the streaming ring would be latency-bound
// (items whose rank rows take many stages: a rank-64 item streams eight 8-row stages one after
// another).  A cluster of C CTAs per item, CTA q owning d_in columns [q kc, (q+1) kc), with C
// chosen so that the whole slice of A (r x kc) and of x fits in shared memory: after one round
// of page-id loads every copy of the CTA is issued at once (one DRAM round trip), the slab is
// contracted by mma_shrink_slab, and the partial tiles are summed on rank 0 as in the streaming
// shrink (pushed into its shared memory, fixed order).  Launched like the streaming shrink: its
// dependent expand may start as soon as the CTAs have started.
struct SlabShrinkArgs {
    const uint16_t* x;
    int64_t ldx;
    float* v;
    int64_t ldv;
    BatchView b;
    PoolView pool;
    int32_t d_in, kc, proj, cluster, max_rank;
    int32_t off_part, off_wp, off_pid, off_a, off_x;
};
constexpr int kSlabThreads = 2 * kThreads;
constexpr int kSlabMaxRank = 64;            // four 16-row mma tiles
constexpr size_t kSlabBytes = 64 * 1024;    // A slice of one CTA, at most

template <int MAXG, int NI>
__global__ void __launch_bounds__(kSlabThreads, 2)
    shrink_slab_kernel(const __grid_constant__ SlabShrinkArgs a, const __grid_constant__ InlineTable<NI> inl) {
    extern __shared__ __align__(128) uint8_t smem_s[];
    constexpr int kWarps = kSlabThreads / 32;
    pdl_launch_dependents();  // the expand may start staging its B^T pages now
    const int C = a.cluster;
    if (C > 1) cluster_arrive_relaxed();  // (waited on before the partial tiles are pushed)
    const int tid = threadIdx.x;
    const int item_idx = (int)blockIdx.x / C;
    const uint32_t q = cluster_ctarank();
    float* part = reinterpret_cast<float*>(smem_s + a.off_part);       // [C][4 x max_rank]; slot 0 this CTA's own
    float* wpart = reinterpret_cast<float*>(smem_s + a.off_wp);        // [warps][MAXG][max_rank]
    int32_t* pid = reinterpret_cast<int32_t*>(smem_s + a.off_pid);     // [r][kc / P]
    uint16_t* As = reinterpret_cast<uint16_t*>(smem_s + a.off_a);      // [r][kc]
    uint16_t* xs = reinterpret_cast<uint16_t*>(smem_s + a.off_x);      // [MAXG][kc]
    const int slot = kSimtMaxItemRows * a.max_rank;

    const ItemInfo m = NI > 1 ? load_item(a.b, inl, item_idx, MAXG, a.max_rank, 0)
                              : load_item(a.b, a.proj, item_idx, MAXG, a.max_rank, 0);
    if (!m.ok && tid == 0) atomicOr(&g_err_simt, kErrRows);
    const int r = m.r, n = m.n;
    const int P_log2 = a.pool.page_log2, P = 1 << P_log2;
    const int ppr = a.d_in >> P_log2, cpa = a.kc >> P_log2;
    const int c0 = (int)q * a.kc;
    const int gx = a.kc / 8;  // 16-byte granules of a row slice
    if (m.ok) {
        // x slices need no page ids: issued first; granule c of row j at c ^ (j % 8)
#pragma unroll
        for (int j = 0; j < MAXG; ++j) {
            const int t = m.tok[j];
            for (int cg = tid; cg < gx; cg += kSlabThreads)
                cp_async16(xs + (size_t)j * a.kc + (cg ^ (j & 7)) * 8,
                           t >= 0 ? a.x + (int64_t)t * a.ldx + c0 + cg * 8 : a.x, t >= 0);
        }
        for (int i = tid; i < r * cpa; i += kSlabThreads) {
            const int k = i / cpa, pc = i - k * cpa;
            const int64_t e = m.pt + (int64_t)k * ppr + (c0 >> P_log2) + pc;
            int32_t page = (e >= 0 && e < a.pool.pt_capacity) ? a.pool.page_table[e] : -1;
            if (page < 0 || page >= a.pool.num_pages) {
                atomicOr(&g_err_simt, kErrPage);
                page = 0;
            }
            pid[i] = page;
        }
    }
    __syncthreads();
    if (m.ok)
        for (GridWalk w(gx, tid, kSlabThreads); w.k < r; w.next()) {
            const int cl = w.c * 8;
            cp_async16(As + (size_t)w.k * a.kc + (w.c ^ (w.k & 7)) * 8,
                       a.pool.pages + ((int64_t)pid[w.k * cpa + (cl >> P_log2)] << P_log2) + (cl & (P - 1)), true);
        }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    float* mine = part;  // slot 0
    mma_shrink_slab<MAXG, kWarps, kSlabMaxRank / 16>(smem_u32(As), smem_u32(xs), a.kc, r, n, m.ok, wpart,
                                                     a.max_rank, mine);
    __syncthreads();

    // partial tiles into rank 0's slots 1..C-1 (the other CTAs then exit); rank 0 sums 0..C-1
    const int E = n * r;
    if (C > 1) {
        cluster_wait_acquire();
        if (q != 0) {
            if (m.ok) {
                const uint32_t dst = map_cluster(smem_u32(part + (size_t)q * slot), 0u);
                for (int e = tid; e < E; e += kSlabThreads) st_cluster_f32(dst + 4u * (uint32_t)e, mine[e]);
            }
            cluster_arrive_release();
            return;
        }
        cluster_arrive_release();
        cluster_wait_acquire();
    }
    if (m.ok)
        for (int e = tid; e < E; e += kSlabThreads) {
            float sum = 0.f;
            for (int qq = 0; qq < C; ++qq) sum += part[(size_t)qq * slot + e];
            const int jrow = e / r, k = e - jrow * r;
            a.v[(int64_t)(m.i0 + jrow) * a.ldv + k] = sum;
        }
}

int num_sms() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            n = 148;
    }
    return n;
}

}  // namespace

// Raise a kernel's dynamic shared-memory limit when a launch needs more than
// any earlier launch of that kernel did (never lowers it).
cudaError_t raise_smem(const void* kern, size_t bytes) {
    static std::mutex mu;
    static std::map<std::pair<int, const void*>, size_t> done;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mu);
    size_t& cur = done[{dev, kern}];
    if (bytes <= cur) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) cur = bytes;
    return e;
}
template <typename K>
cudaError_t set_smem(K kern, size_t bytes) {
    return raise_smem(reinterpret_cast<const void*>(kern), bytes);
}

// CTAs of 128 threads with `smem` bytes of dynamic shared memory that one SM
// holds at once (cached per device, kernel and size).
int resident_ctas(const void* kern, size_t smem) {
    static std::mutex mu;
    static std::map<std::tuple<int, const void*, size_t>, int> done;
    int dev = 0;
    cudaGetDevice(&dev);
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = done.find({dev, kern, smem});
        if (it != done.end()) return it->second;
    }
    int n = 0;
    if (raise_smem(kern, smem) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kThreads, smem) != cudaSuccess || n < 1) {
        cudaGetLastError();
        n = 1;
    }
    std::lock_guard<std::mutex> lock(mu);
    done[{dev, kern, smem}] = n;
    return n;
}

// Modelled time, in stages, of a launch over `items` SIMT items with `cpi` CTAs
// each (`slots` CTAs resident at a time), every CTA doing npass passes of its
// item's row groups (work.sum_ng row groups over all items, work.max_ng for the
// largest) plus a fixed prologue (page ids, pipeline fill) of about two stages.
// Equal items run in waves; unequal ones (emitted largest first) pack into the
// slots, bounded below by the largest CTA.  `work_passes`: passes over which
// one row group of an item is spread in total.
double split_time(const SimtWork& work, int64_t items, int64_t cpi, int npass, double work_passes, int64_t slots) {
    constexpr double kPrologue = 2.0;
    const int64_t n = items * cpi;
    const double biggest = (double)std::max(work.max_ng, 1) * npass + kPrologue;
    if (slots < 1) slots = 1;
    if (work.sum_ng == items * (int64_t)work.max_ng) return (double)((n + slots - 1) / slots) * biggest;
    const double total = (double)work.sum_ng * work_passes + (double)n * kPrologue;
    return std::max(biggest, total / (double)slots);
}

template <typename K1, typename K2, typename K4>
auto pick(int max_item_rows, K1 k1, K2 k2, K4 k4) {
    return max_item_rows <= 1 ? k1 : max_item_rows <= 2 ? k2 : k4;
}

// Modelled time of a grouped launch: entries j with cpi[j] CTAs per item, each
// doing npass[j] passes of its item's row groups; wp[j] = passes one row group
// of an item is spread over in total.  One entry: split_time.  Several: the
// entries' CTAs (largest first) pack into the slots, bounded by the largest.
double group_time(const SimtWork& work, int64_t items, const int* cpi, const int* npass, const double* wp, int n,
                  int64_t slots) {
    if (n == 1) return split_time(work, items, cpi[0], npass[0], wp[0], slots);
    constexpr double kPrologue = 2.0;
    int max_np = 1;
    double total = 0.0;
    for (int j = 0; j < n; ++j) {
        max_np = std::max(max_np, npass[j]);
        total += (double)work.sum_ng * wp[j] + (double)items * cpi[j] * kPrologue;
    }
    const double biggest = (double)std::max(work.max_ng, 1) * max_np + kPrologue;
    return std::max(biggest, total / (double)std::max<int64_t>(slots, 1));
}

// The one-shot slab shrink, when it applies: bf16 pool, one x with one projection, ranks up to
// 64, a cluster size C <= 8 dividing the page count with an A slice r x (d_in / C) of at most
// kSlabBytes, and at most two waves of clusters.  Then *used = true and the kernel is launched
// (unless `dry`); otherwise nothing happens.  Measured against the streaming shrink (per step,
// L2 flushed): 200 decode tokens on 8192 -> 8192, rank 16: 29.6 against 35.8 us; 64 tokens of
// ranks 8-64 on 4096 -> 14336: 27.7 against 29.7 us; beyond two waves it loses (256 tokens of
// ranks 8-64: 42.0 against 39.9 us; the 70B layer's down projection: 70.6 against 68.6 us),
// the streaming ring overlapping each CTA's loads with its arithmetic.
cudaError_t slab_shrink_launch(const ShrinkJob& j, const BatchView& b, int32_t num_items, int32_t max_item_rows,
                               int32_t max_rank, const PoolView& pool, const InlineTable<kInlineItems>* inl,
                               cudaStream_t stream, bool* used, bool dry) {
    *used = false;
    if (pool.wfmt != kFmtBf16 || j.nsub != 1 || max_rank > kSlabMaxRank || j.d_in <= 0) return cudaSuccess;
    const int mr = std::max(8, max_rank);
    const int maxg = max_item_rows <= 1 ? 1 : max_item_rows <= 2 ? 2 : 4;
    const int pa = j.d_in >> pool.page_log2;
    int C = 0;
    for (int c = 1; c <= 8 && !C; ++c)
        if (pa % c == 0 && (size_t)mr * (j.d_in / c) * 2 <= kSlabBytes) C = c;
    if (!C) return cudaSuccess;
    const int kc = j.d_in / C;
    auto al = [](size_t v) { return (v + 127) & ~(size_t)127; };
    SlabShrinkArgs a;
    std::memset(&a, 0, sizeof(a));
    size_t o = 0;
    a.off_part = (int32_t)(o = al(o));
    o += (size_t)C * kSimtMaxItemRows * mr * 4;
    a.off_wp = (int32_t)(o = al(o));
    o += (size_t)(kSlabThreads / 32) * maxg * mr * 4;
    a.off_pid = (int32_t)(o = al(o));
    o += (size_t)mr * (kc >> pool.page_log2) * 4;
    a.off_a = (int32_t)(o = al(o));
    o += (size_t)mr * kc * 2;
    a.off_x = (int32_t)(o = al(o));
    o += (size_t)maxg * kc * 2;
    const size_t smem = al(o);
    a.x = j.x;
    a.ldx = j.ldx;
    a.v = j.v[0];
    a.ldv = j.ldv[0];
    a.b = b;
    a.pool = pool;
    a.d_in = j.d_in;
    a.kc = kc;
    a.proj = j.proj[0];
    a.cluster = C;
    a.max_rank = mr;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(num_items * C), 1, 1);
    cfg.blockDim = dim3(kSlabThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const void* kern =
        inl ? reinterpret_cast<const void*>(pick(max_item_rows, shrink_slab_kernel<1, kInlineItems>,
                                                 shrink_slab_kernel<2, kInlineItems>, shrink_slab_kernel<4, kInlineItems>))
            : reinterpret_cast<const void*>(pick(max_item_rows, shrink_slab_kernel<1, 1>, shrink_slab_kernel<2, 1>,
                                                 shrink_slab_kernel<4, 1>));
    cudaError_t e = raise_smem(kern, smem);
    if (e != cudaSuccess) return e;
    int clusters = 0;  // clusters resident at once
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return cudaSuccess;
    }
    if (clusters <= 0 || num_items > 2 * clusters) return cudaSuccess;
    *used = true;
    if (dry) return cudaSuccess;
    if (inl) {
        void* args[] = {&a, const_cast<InlineTable<kInlineItems>*>(inl)};
        return cudaLaunchKernelExC(&cfg, kern, args);
    }
    InlineTable<1> none{};
    void* args[] = {&a, &none};
    return cudaLaunchKernelExC(&cfg, kern, args);
}

template <int NE, int WF>
cudaError_t shrink_launch(const ShrinkJob* jobs, int n_jobs, const BatchView& b, int32_t num_items,
                          int32_t max_item_rows, int32_t max_rank, const SimtWork& work, const PoolView& pool,
                          const InlineTable<kInlineItems>* inl, cudaStream_t stream) {
    // entries with the most columns first: their CTAs are scheduled first
    int order[kMaxGroup];
    for (int j = 0; j < n_jobs; ++j) order[j] = j;
    std::stable_sort(order, order + n_jobs, [&](int u, int w) { return jobs[u].d_in > jobs[w].d_in; });
    auto kern_inl = pick(max_item_rows, shrink_simt_kernel<1, kInlineItems, NE, WF>,
                         shrink_simt_kernel<2, kInlineItems, NE, WF>, shrink_simt_kernel<4, kInlineItems, NE, WF>);
    auto kern_tab = pick(max_item_rows, shrink_simt_kernel<1, 1, NE, WF>, shrink_simt_kernel<2, 1, NE, WF>,
                         shrink_simt_kernel<4, 1, NE, WF>);
    const void* kp = inl ? reinterpret_cast<const void*>(kern_inl) : reinterpret_cast<const void*>(kern_tab);
    const int mr = std::max(8, max_rank);
    int max_pages = 0, nsub_max = 1;
    for (int j = 0; j < n_jobs; ++j) {
        max_pages = std::max(max_pages, jobs[j].d_in >> pool.page_log2);
        nsub_max = std::max(nsub_max, jobs[j].nsub);
    }
    const int maxg = max_item_rows <= 1 ? 1 : max_item_rows <= 2 ? 2 : 4;
    const int stages = maxg == 1 ? shrink_stages<1>() : shrink_stages<4>();
    // A rows + x slices
    const size_t ring_bytes = (size_t)stages * ((size_t)stage_bytes<WF>() + (size_t)maxg * kPass * 2);
    auto smem_for = [&](int c) {  // partial tiles, reduction scratch, row scales, page ids, ring
        const size_t part_bytes = (size_t)c * kSimtMaxItemRows * mr * nsub_max * 4;
        // page ids: each stacked projection's rows start on a row group (multiple of 8 rows)
        const size_t pidb = (size_t)nsub_max * ((mr + kRowGroup - 1) / kRowGroup * kRowGroup) *
                            ((max_pages + c - 1) / c) * 4;
        const size_t rsc_bytes = WF == kFmtBf16 ? 0 : (size_t)nsub_max * kMaxRank * 4;
        return (((part_bytes + 1024 + rsc_bytes + pidb + 127) & ~(size_t)127)) + ring_bytes;
    };
    // Cluster size C (chunks of >= 1024 columns, C <= 8, dividing every entry's page
    // count): the smallest C that still gives at least two CTAs for every CTA slot, else
    // the largest valid one.  A CTA pays its prologue (page ids, then its first stage: two
    // dependent DRAM round trips) once, so fewer and longer CTAs stream better as long as
    // there are enough of them to keep every SM busy and balanced; measured on the
    // workloads (the 70B layer: 263 us with C = 1 against 284-286 us with C = 2 or 4; the
    // decode and mixed-rank batches, with fewer items than slots, take the largest C).
    int C = 0, C_max = 1;
    for (int c = 1; c <= 8; ++c) {
        bool valid = true;
        for (int j = 0; j < n_jobs; ++j) {
            const int d = jobs[j].d_in;
            if (((d >> pool.page_log2) % c) || (c > 1 && d / c < kPass)) valid = false;
        }
        if (!valid) continue;
        C_max = c;
        const int64_t ctas = (int64_t)n_jobs * num_items * c;
        if (C == 0 && ctas >= 2 * (int64_t)resident_ctas(kp, smem_for(c)) * num_sms()) C = c;
    }
    if (C == 0) C = C_max;
    (void)work;
    ShrinkArgs<NE> a;
    std::memset(&a, 0, sizeof(a));
    for (int i = 0; i < n_jobs; ++i) {
        const ShrinkJob& j = jobs[order[i]];
        ShrinkEntry& en = a.ent[i];
        en.x = j.x;
        en.ldx = j.ldx;
        en.d_in = j.d_in;
        en.kc = j.d_in / C;
        en.nsub = j.nsub;
        for (int k = 0; k < kMaxShare; ++k) {
            const int src = k < j.nsub ? k : 0;  // unused slots repeat the first projection
            en.proj[k] = j.proj[src];
            en.v[k] = j.v[src];
            en.ldv[k] = j.ldv[src];
        }
    }
    a.n_entries = n_jobs;
    a.items = num_items;
    a.b = b;
    a.pool = pool;
    a.cluster = C;
    a.max_rank = mr;
    a.nsub_max = nsub_max;
    a.stages = stages;
    const size_t smem = smem_for(C);
    a.ring_offset = (int)(smem - ring_bytes);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(n_jobs * C * num_items), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (inl) {
        cudaError_t e = set_smem(kern_inl, smem);
        if (e != cudaSuccess) return e;
        return cudaLaunchKernelEx(&cfg, kern_inl, a, *inl);
    }
    cudaError_t e = set_smem(kern_tab, smem);
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, kern_tab, a, InlineTable<1>{});
}

template <int NE, int WF>
cudaError_t expand_launch(const ExpandJob* jobs, int n_jobs, const BatchView& b, int32_t num_items,
                          int32_t max_item_rows, int32_t max_rank, const SimtWork& work, const PoolView& pool,
                          float scale, int32_t y_dtype, const InlineTable<kInlineItems>* inl, bool y_early,
                          cudaStream_t stream) {
    // entries with the most column passes first
    int order[kMaxGroup];
    for (int j = 0; j < n_jobs; ++j) order[j] = j;
    std::stable_sort(order, order + n_jobs, [&](int u, int w) { return jobs[u].d_out > jobs[w].d_out; });
    auto kern_inl = y_dtype == 0 ? pick(max_item_rows, expand_simt_kernel<1, kInlineItems, NE, WF, 0>,
                                        expand_simt_kernel<2, kInlineItems, NE, WF, 0>,
                                        expand_simt_kernel<4, kInlineItems, NE, WF, 0>)
                                 : pick(max_item_rows, expand_simt_kernel<1, kInlineItems, NE, WF, 1>,
                                        expand_simt_kernel<2, kInlineItems, NE, WF, 1>,
                                        expand_simt_kernel<4, kInlineItems, NE, WF, 1>);
    auto kern_tab = y_dtype == 0 ? pick(max_item_rows, expand_simt_kernel<1, 1, NE, WF, 0>,
                                        expand_simt_kernel<2, 1, NE, WF, 0>, expand_simt_kernel<4, 1, NE, WF, 0>)
                                 : pick(max_item_rows, expand_simt_kernel<1, 1, NE, WF, 1>,
                                        expand_simt_kernel<2, 1, NE, WF, 1>, expand_simt_kernel<4, 1, NE, WF, 1>);
    const void* kp = inl ? reinterpret_cast<const void*>(kern_inl) : reinterpret_cast<const void*>(kern_tab);
    const int mr = std::max(8, max_rank);
    auto smem_for = [&](int npass) {  // v of the item, row scales, page ids, ring
        const size_t pid_bytes = (size_t)mr * ((npass * kPass) >> pool.page_log2) * 4;
        const size_t rsc_bytes = WF == kFmtBf16 ? 0 : kMaxRank * 4;
        return (((size_t)kSimtMaxItemRows * mr * 4 + rsc_bytes + pid_bytes + 127) & ~(size_t)127) +
               (size_t)kExpandStages * stage_bytes<WF>();
    };
    int tiles[kMaxGroup], max_tiles = 1;
    for (int j = 0; j < n_jobs; ++j) {
        tiles[j] = (jobs[order[j]].d_out + kPass - 1) / kPass;
        max_tiles = std::max(max_tiles, tiles[j]);
    }
    // passes per CTA P (each entry takes min(P, its tiles)): the shortest modelled time
    int best_p = max_tiles;
    double best = 1e300;
    for (int P = 1; P <= max_tiles; ++P) {
        int cpi[kMaxGroup], np[kMaxGroup], max_np = 1;
        double wp[kMaxGroup];
        for (int j = 0; j < n_jobs; ++j) {
            np[j] = std::min(P, tiles[j]);
            cpi[j] = (tiles[j] + np[j] - 1) / np[j];
            wp[j] = (double)tiles[j];
            max_np = std::max(max_np, np[j]);
        }
        const double t = group_time(work, num_items, cpi, np, wp, n_jobs,
                                    (int64_t)resident_ctas(kp, smem_for(max_np)) * num_sms());
        if (t < best) {
            best = t;
            best_p = P;
        }
    }
    ExpandArgs<NE> a;
    std::memset(&a, 0, sizeof(a));
    int ctas = 0, max_np = 1;
    for (int i = 0; i < n_jobs; ++i) {
        const ExpandJob& j = jobs[order[i]];
        const int np = std::min(best_p, tiles[i]), cpi = (tiles[i] + np - 1) / np;
        a.ent[i] = ExpandEntry{j.v, j.ldv, j.y, j.ldy, j.d_out, np, cpi, ctas, j.proj, {0, 0, 0}};
        ctas += cpi * num_items;
        max_np = std::max(max_np, np);
    }
    a.n_entries = n_jobs;
    a.items = num_items;
    a.b = b;
    a.pool = pool;
    a.scale = scale;
    a.y_dtype = y_dtype;
    a.y_early = y_early ? 1 : 0;
    a.max_rank = mr;
    a.stages = kExpandStages;
    const size_t smem = smem_for(max_np);
    a.ring_offset = (int)(smem - (size_t)kExpandStages * stage_bytes<WF>());
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ctas, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (inl) {
        cudaError_t e = set_smem(kern_inl, smem);
        if (e != cudaSuccess) return e;
        return cudaLaunchKernelEx(&cfg, kern_inl, a, *inl);
    }
    cudaError_t e = set_smem(kern_tab, smem);
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, kern_tab, a, InlineTable<1>{});
}

// The one-shot fused kernel for a single projection, when every item's cluster fits in
// one wave and a CTA's slices fit in shared memory (*used = true); otherwise nothing is
// launched.  With `dry`, the choice is made and reported but nothing is launched.  The
// largest cluster size (up to 8) that fits is taken: the most CTAs loading at once, and the
// least dependent work per thread.  (Clusters of 16, a non-portable size, were measured
// slower on decode: 18.5 against 16.5 us per step.)
template <int WF>
cudaError_t fused_launch(const ShrinkJob& sj, const ExpandJob& ej, const BatchView& b, int32_t num_items,
                         int32_t max_item_rows, int32_t max_rank, const PoolView& pool, float scale, int32_t y_dtype,
                         const InlineTable<kInlineItems>* inl, cudaStream_t stream, bool* used, bool dry) {
    *used = false;
    if (num_items <= 0 || sj.nsub != 1 || sj.d_in <= 0 || ej.d_out <= 0) return cudaSuccess;
    if (max_rank > kFusedMaxRank) return cudaSuccess;
    const int maxg = max_item_rows <= 1 ? 1 : max_item_rows <= 2 ? 2 : 4;
    const int mr = std::max(8, max_rank);
    const int esz = y_dtype == 0 ? 2 : 4;
    const int pa = sj.d_in >> pool.page_log2, pb = ej.d_out >> pool.page_log2;
    auto al = [](size_t v) { return (v + 127) & ~(size_t)127; };
    auto kern_for = [&](bool use_inl) -> const void* {
        if (use_inl)
            return reinterpret_cast<const void*>(pick(max_item_rows, fused_simt_kernel<1, kInlineItems, WF>,
                                                      fused_simt_kernel<2, kInlineItems, WF>,
                                                      fused_simt_kernel<4, kInlineItems, WF>));
        return reinterpret_cast<const void*>(pick(max_item_rows, fused_simt_kernel<1, 1, WF>,
                                                  fused_simt_kernel<2, 1, WF>, fused_simt_kernel<4, 1, WF>));
    };
    const void* kern = kern_for(inl != nullptr);
    for (int C = 8; C >= 1; --C) {
        if ((pa % C) || (pb % C)) continue;
        const int kc = sj.d_in / C, ko = ej.d_out / C;
        FusedArgs a;
        std::memset(&a, 0, sizeof(a));
        size_t o = 0;
        a.off_part = (int32_t)(o = al(o));
        o += (size_t)C * kSimtMaxItemRows * mr * 4;
        a.off_vs = (int32_t)(o = al(o));
        o += (size_t)kSimtMaxItemRows * mr * 4;
        a.off_rsc = (int32_t)(o = al(o));
        o += WF == kFmtBf16 ? 0 : 2 * kMaxRank * 4;
        a.off_pid_a = (int32_t)(o = al(o));
        o += (size_t)mr * (pa / C) * 4;
        a.off_pid_b = (int32_t)(o = al(o));
        o += (size_t)mr * (pb / C) * 4;
        a.off_a = (int32_t)(o = al(o));  // the bf16 slab of A
        o += (size_t)mr * kc * 2;
        a.off_ac = (int32_t)(o = al(o));  // a quantised pool's codes of A
        o += WF == kFmtBf16 ? 0 : (size_t)mr * kc / 8 * bytes_per_8<WF>();
        a.off_x = (int32_t)(o = al(o));
        o += (size_t)maxg * kc * 2;
        a.off_b = (int32_t)(o = al(o));
        o += (size_t)mr * ko / 8 * bytes_per_8<WF>();
        a.off_y = (int32_t)(o = al(o));
        o += (size_t)maxg * ko * esz;
        a.off_wp = (int32_t)(o = al(o));
        o += (size_t)(kFusedThreads / 32) * maxg * mr * 4;
        const size_t smem = al(o);
        if (smem > 227 * 1024) continue;
        cudaError_t e = raise_smem(kern, smem);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(num_items * C), 1, 1);
        cfg.blockDim = dim3(kFusedThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)C;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;  // every item's cluster resident at once: one wave
        if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess) {
            cudaGetLastError();
            continue;
        }
        if (clusters < num_items) continue;
        if (dry) {
            *used = true;
            return cudaSuccess;
        }
        a.x = sj.x;
        a.ldx = sj.ldx;
        a.v = sj.v[0];
        a.ldv = sj.ldv[0];
        a.y = ej.y;
        a.ldy = ej.ldy;
        a.b = b;
        a.pool = pool;
        a.d_in = sj.d_in;
        a.d_out = ej.d_out;
        a.kc = kc;
        a.ko = ko;
        a.proj = sj.proj[0];
        a.cluster = C;
        a.max_rank = mr;
        a.y_dtype = y_dtype;
        a.scale = scale;
        *used = true;
        if (inl) {
            void* args[] = {&a, const_cast<InlineTable<kInlineItems>*>(inl)};
            return cudaLaunchKernelExC(&cfg, kern, args);
        }
        InlineTable<1> none{};
        void* args[] = {&a, &none};
        return cudaLaunchKernelExC(&cfg, kern, args);
    }
    return cudaSuccess;
}

cudaError_t launch_fused_simt(const ShrinkJob& sj, const ExpandJob& ej, const BatchView& b, int32_t num_items,
                              int32_t max_item_rows, int32_t max_rank, const PoolView& pool, float scale,
                              int32_t y_dtype, const InlineTable<kInlineItems>* inl, cudaStream_t stream,
                              bool* used, bool dry) {
    *used = false;
    switch (pool.wfmt) {
        case kFmtBf16:
            return fused_launch<kFmtBf16>(sj, ej, b, num_items, max_item_rows, max_rank, pool, scale, y_dtype, inl,
                                          stream, used, dry);
        case kFmtFp8:
            return fused_launch<kFmtFp8>(sj, ej, b, num_items, max_item_rows, max_rank, pool, scale, y_dtype, inl,
                                         stream, used, dry);
        case kFmtInt4:
            return fused_launch<kFmtInt4>(sj, ej, b, num_items, max_item_rows, max_rank, pool, scale, y_dtype, inl,
                                          stream, used, dry);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_shrink_simt(const ShrinkJob* jobs, int n_jobs, const BatchView& b, int32_t num_items,
                               int32_t max_item_rows, int32_t max_rank, const SimtWork& work, const PoolView& pool,
                               const InlineTable<kInlineItems>* inl, cudaStream_t stream) {
    if (num_items <= 0 || n_jobs <= 0) return cudaSuccess;
    if (n_jobs > kMaxGroup || (inl && (n_jobs > 1 || jobs[0].nsub != 1))) return cudaErrorInvalidValue;
    for (int j = 0; j < n_jobs; ++j)
        if (jobs[j].nsub < 1 || jobs[j].nsub > kMaxShare) return cudaErrorInvalidValue;
    if (n_jobs == 1) {
        bool used = false;
        cudaError_t e = slab_shrink_launch(jobs[0], b, num_items, max_item_rows, max_rank, pool, inl, stream, &used,
                                           false);
        if (e != cudaSuccess || used) return e;
    }
    // one x: a one-entry table (small launch arguments, no per-CTA lookup)
    auto go = [&](auto wf) {
        constexpr int WF = decltype(wf)::value;
        if (n_jobs == 1)
            return shrink_launch<1, WF>(jobs, n_jobs, b, num_items, max_item_rows, max_rank, work, pool, inl, stream);
        return shrink_launch<kMaxGroup, WF>(jobs, n_jobs, b, num_items, max_item_rows, max_rank, work, pool, inl,
                                            stream);
    };
    switch (pool.wfmt) {
        case kFmtBf16: return go(std::integral_constant<int, kFmtBf16>{});
        case kFmtFp8: return go(std::integral_constant<int, kFmtFp8>{});
        case kFmtInt4: return go(std::integral_constant<int, kFmtInt4>{});
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_expand_simt(const ExpandJob* jobs, int n_jobs, const BatchView& b, int32_t num_items,
                               int32_t max_item_rows, int32_t max_rank, const SimtWork& work, const PoolView& pool,
                               float scale, int32_t y_dtype, const InlineTable<kInlineItems>* inl, bool y_early,
                               cudaStream_t stream) {
    if (num_items <= 0 || n_jobs <= 0) return cudaSuccess;
    if (n_jobs > kMaxGroup || (inl && n_jobs > 1)) return cudaErrorInvalidValue;
    auto go = [&](auto wf) {
        constexpr int WF = decltype(wf)::value;
        if (n_jobs == 1)
            return expand_launch<1, WF>(jobs, n_jobs, b, num_items, max_item_rows, max_rank, work, pool, scale,
                                        y_dtype, inl, y_early, stream);
        return expand_launch<kMaxGroup, WF>(jobs, n_jobs, b, num_items, max_item_rows, max_rank, work, pool, scale,
                                            y_dtype, inl, y_early, stream);
    };
    switch (pool.wfmt) {
        case kFmtBf16: return go(std::integral_constant<int, kFmtBf16>{});
        case kFmtFp8: return go(std::integral_constant<int, kFmtFp8>{});
        case kFmtInt4: return go(std::integral_constant<int, kFmtInt4>{});
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t read_clear_errors_simt(uint32_t* bits, cudaStream_t stream) {
    unsigned int h = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&h, g_err_simt, sizeof(h), 0, cudaMemcpyDeviceToHost, stream);
    if (e != cudaSuccess) return e;
    e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbolAsync(g_err_simt, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return e;
    e = cudaStreamSynchronize(stream);
    *bits |= h;
    return e;
}

}  // namespace sgmv
