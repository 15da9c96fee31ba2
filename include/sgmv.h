/*
 * sgmv.h -- C ABI of libsgmv_b200.so: the multi-LoRA delta on one B200 (sm_100a).
 *
 * The library computes, for every token t of a batch whose tokens carry
 * different LoRA adapters a(t),
 *
 *     y_t  <-  y_t + scale * s_{a(t)} * B_{a(t)} ( A_{a(t)} x_t )
 *
 * where y already holds the base output W x_t, scale is the call's and s_a
 * the adapter's own multiplier (1.0 unless set).  Pages cited by title:
 *
 *   [SGMV post] "Multi-LoRA serving: the single translator with a thousand
 *               glossaries -- shared base, thousands of concurrent adapters
 *               and the SGMV kernel" (blog.lo0.es)
 *   [Glossary]  "Multi-LoRA Serving" (skillsintelligence.tools glossary)
 *   [ClusterBid] "Multi-LoRA Inference Serving: Serving Thousands of
 *               Fine-Tuned Models on One GPU" (clusterbid.com)
 *
 * Orientation ([SGMV post], "The bare mechanism", equations W' = W + BA and
 * y = Wx + B(Ax)): A is r x d_in, B is d_out x r.  The per-token form and its
 * two phases, shrink (d_in -> r) and expand (r -> d_out), are those of
 * [SGMV post], "SGMV: the kernel that holds it all up".
 *
 * Conventions shared by every call
 *   - All matrices are row-major.  bf16 data is passed as raw 16-bit words.
 *   - "device" pointers are CUDA global-memory addresses on the pool's
 *     device; "host" pointers are ordinary process memory.
 *   - Calls that take a stream enqueue work on it and return without
 *     waiting, except where stated.  NULL is the legacy default stream.
 *   - A call that returns anything but SGMV_OK has launched nothing and
 *     changed no caller memory; sgmv_last_error() describes the failure.
 *   - Kernels never trap.  Device-side checks (a page id outside the pool,
 *     a token row outside the batch, a wait that gave up) set a device error
 *     word and skip the access; sgmv_check_errors() reports and clears it.
 *   - The caller owns x, y, v and the plan table; the pool owns its pages
 *     and its page table.  Nothing here is thread-safe on the same pool.
 */
#ifndef SGMV_B200_H
#define SGMV_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SGMV_API __attribute__((visibility("default")))
#else
#define SGMV_API
#endif

typedef struct CUstream_st* sgmv_stream_t; /* same type as cudaStream_t */

typedef enum {
    SGMV_OK = 0,
    SGMV_ERR_INVALID = 1,      /* malformed argument (null pointer, bad size, misaligned row) */
    SGMV_ERR_UNSUPPORTED = 2,  /* well-formed but outside what the library handles          */
    SGMV_ERR_NOT_RESIDENT = 3, /* an adapter id of the batch is not loaded in the pool        */
    SGMV_ERR_OUT_OF_PAGES = 4, /* the pool has too few free pages for an adapter              */
    SGMV_ERR_CUDA = 5,         /* a CUDA runtime call failed                                  */
    SGMV_ERR_BOUNDS = 6,       /* a device-side bounds check failed (from sgmv_check_errors)  */
    SGMV_ERR_TIMEOUT = 7,      /* a device-side wait gave up (from sgmv_check_errors)         */
    SGMV_ERR_CAPACITY = 8      /* a caller-provided buffer is too small                       */
} sgmv_status;

/* Text of a status code (static storage). */
SGMV_API const char* sgmv_status_string(sgmv_status s);
/* Detail of the last failure on the calling thread (thread-local storage). */
SGMV_API const char* sgmv_last_error(void);

/* ------------------------------------------------------------------------ */
/* Paged adapter pool                                                         */
/* ------------------------------------------------------------------------ */
/*
 * Adapter weights live in one device buffer of equal-size pages, in the
 * spirit of the unified paging that [SGMV post] describes (TL;DR, and
 * "Operational pitfalls": memory fragmentation -- weights kept in a pool of
 * interchangeable blocks) and of the fixed-size adapter pool with slots of
 * [ClusterBid] (paragraph on vLLM's GPU memory pool).
 *
 * Layout.  A page holds page_elems values (bf16 by default; codes in a
 * quantised pool, see below).  For each adapter and each
 * projection p the pool stores
 *     A   as r rows of d_in[p]  values (the logical r x d_in matrix), and
 *     B^T as r rows of d_out[p] values (the transpose of the d_out x r B),
 * each row cut into d/page_elems pages.  The page table (int32 page ids) maps
 * (adapter, projection, matrix, rank row k, chunk c) to a page; entries of one
 * (adapter, projection, matrix) are contiguous:
 *     entry = base + k * (d / page_elems) + c.
 * Pages are taken from a free list in any order, so consecutive chunks of a
 * row are in general not adjacent in memory.
 *
 * The payload of a rank-r adapter in a bf16 pool is exactly
 * sum_p (d_in[p]*r + r*d_out[p])*2 bytes -- the bytes-per-matrix formula of
 * [SGMV post], "The maths that matters" -- because page_elems must divide
 * every d_in[p] and d_out[p] (a half or a quarter of that in a quantised pool).
 */
typedef struct sgmv_pool sgmv_pool;

/*
 * Weight formats of a pool.  bf16 is the default and what the pool stores
 * unless it is created with sgmv_pool_create_ex.  The two quantised formats
 * follow [ClusterBid] (paragraph on the GPU memory budget: FP8 adapters halve
 * the memory; paragraph on adapter weight quantization: INT4 adapters, with a
 * dequantisation cost at inference).  [SGMV post] ("Combined pattern with
 * quantisation and disaggregated serving") keeps adapters in BF16 in its
 * canonical stack, which is why bf16 stays the default.
 *
 * Quantised layout.  A page still holds page_elems values of one rank row,
 * now as codes: 1 byte each (FP8_E4M3) or 4 bits each (INT4, two's
 * complement in [-7, 7], value 2i in the low nibble of byte i).  Each rank row
 * k of A and of B^T has one fp32 scale s_k, kept beside the page table (entry
 * of the row's first chunk), and its values are code(q) * s_k:
 *     s_k  = max_c |w_kc| / Q    (Q = 448 for E4M3, 7 for INT4; fp32 division)
 *     q_kc = RN(w_kc / s_k)      (fp32 division; E4M3: round to nearest even,
 *                                 saturating; INT4: round half to even,
 *                                 clamped to [-7, 7]); a row of zeros has s_k = 0.
 * The load call quantises bf16 weights on the device by this rule.  Because
 * the scale belongs to a whole rank row, it leaves both contractions
 * exactly: v_k = s^A_k * sum_c q^A_kc x_c, and the expand multiplies v_k by
 * s^B_k before using the codes of B^T.  The kernels therefore only convert
 * codes (every E4M3 and INT4 value is exact in bf16 and fp32) and the delta
 * equals the bf16 computation on the dequantised weights up to rounding.
 */
typedef enum {
    SGMV_WEIGHTS_BF16 = 0,
    SGMV_WEIGHTS_FP8_E4M3 = 1,
    SGMV_WEIGHTS_INT4 = 2
} sgmv_weight_format;

typedef struct {
    int64_t num_pages;         /* pages in the pool                                 */
    int64_t free_pages;        /* pages not holding adapter data                    */
    int64_t page_bytes;        /* bytes of one page: page_elems * 2, 1 or 1/2       */
    int64_t payload_bytes;     /* (num_pages - free_pages) * page_bytes             */
    int32_t resident_adapters; /* adapters currently loaded                         */
    int32_t page_elems;
    int32_t weight_format;     /* sgmv_weight_format                                */
    int32_t reserved;
} sgmv_pool_stats;

/*
 * Create a bf16 pool on `device` (CUDA ordinal) with `num_pages` pages of
 * `page_elems` bf16 values (a power of two in [64, 65536]), for adapters over
 * `n_proj` projections with shapes d_in[p] -> d_out[p] (host arrays of n_proj
 * entries, each a multiple of page_elems) and ranks up to max_rank (<= 128).
 * device = -1 creates a host-only pool that keeps the bookkeeping (page
 * allocation, page table) without device memory; its loads copy nothing and
 * accept NULL matrix pointers.  A device pool allocates
 * num_pages * page_elems * 2 bytes of pages and 2 * num_pages + 1024 int32
 * page-table entries on `device`, which must be the current device of every
 * later call that uses the pool.  On success *out owns that memory until
 * sgmv_pool_destroy.
 */
SGMV_API sgmv_status sgmv_pool_create(int device, int64_t num_pages, int32_t page_elems, int32_t n_proj,
                             const int32_t* d_in, const int32_t* d_out, int32_t max_rank,
                             sgmv_pool** out);
/*
 * sgmv_pool_create with a weight format (sgmv_weight_format).  A quantised
 * pool allocates num_pages pages of page_elems codes (page_elems or
 * page_elems / 2 bytes each) plus one fp32 scale per page-table entry, and
 * needs page_elems >= 64 as before.  SGMV_ERR_INVALID for an unknown format.
 */
SGMV_API sgmv_status sgmv_pool_create_ex(int device, int64_t num_pages, int32_t page_elems, int32_t n_proj,
                                const int32_t* d_in, const int32_t* d_out, int32_t max_rank,
                                int32_t weight_format, sgmv_pool** out);
SGMV_API sgmv_status sgmv_pool_destroy(sgmv_pool* pool);

/*
 * Load (or replace) adapter `adapter_id` (>= 0) of rank `rank` (0..max_rank).
 * A[p] points to the r x d_in[p] matrix of projection p, B[p] to its
 * d_out[p] x r matrix (bf16, row-major, logical orientation); A and B are host
 * arrays of n_proj pointers.  The pointed-to data is device memory when
 * src_on_device != 0, host memory otherwise.  The copies are enqueued on
 * `stream` and the call waits for them before returning, so the sources may be
 * freed afterwards.  SGMV_ERR_OUT_OF_PAGES leaves the pool unchanged (a
 * resident adapter being replaced stays resident).  SGMV_ERR_CUDA (a copy
 * failed) leaves the adapter not resident -- a replaced one included -- with
 * every page back on the free list.  A quantised pool quantises the bf16 rows
 * on the device as it stores them.
 * Replacing a resident adapter frees its pages and may hand the same pages
 * straight back to the new weights, which are written on `stream`: as for
 * sgmv_pool_evict, no kernel enqueued on another stream may still read the old
 * adapter when the call is made.
 */
SGMV_API sgmv_status sgmv_pool_load(sgmv_pool* pool, int32_t adapter_id, int32_t rank,
                           const void* const* A, const void* const* B, int src_on_device,
                           sgmv_stream_t stream);
/* Remove an adapter and return its pages to the free list.  The caller must
 * not evict an adapter that an enqueued kernel may still read. */
SGMV_API sgmv_status sgmv_pool_evict(sgmv_pool* pool, int32_t adapter_id);
/*
 * Multiplier of adapter `adapter_id`'s delta (LoRA's alpha / r for that
 * adapter): a token on that adapter gets y_t + (scale * s_a) B_a A_a x_t,
 * where `scale` is the expand call's argument.  The pages give no LoRA
 * scaling ("Multi-LoRA serving: the single translator ...", section "The bare
 * mechanism", W' = W + BA); one factor per adapter on its own delta is the
 * reading taken.  The factor belongs to the id, resident or not: it is kept
 * across evictions and reloads until changed, and is 1.0 for an id never set.
 * The segment builder copies it into the plan (seg_scale), so a change takes
 * effect for plans built afterwards.  SGMV_ERR_INVALID for a non-finite scale.
 */
SGMV_API sgmv_status sgmv_pool_set_adapter_scale(sgmv_pool* pool, int32_t adapter_id, float scale);
SGMV_API sgmv_status sgmv_pool_get_adapter_scale(const sgmv_pool* pool, int32_t adapter_id, float* scale);
SGMV_API sgmv_status sgmv_pool_get_stats(const sgmv_pool* pool, sgmv_pool_stats* out);
/* Rank of a resident adapter; SGMV_ERR_NOT_RESIDENT otherwise. */
SGMV_API sgmv_status sgmv_pool_adapter_rank(const sgmv_pool* pool, int32_t adapter_id, int32_t* rank);
/*
 * Copy the page ids of (adapter, projection, matrix) into page_ids (host,
 * capacity `cap`), in page-table order; matrix 0 = A, 1 = B^T.  *n receives
 * the count (r * d / page_elems).  For inspection and tests.
 */
SGMV_API sgmv_status sgmv_pool_adapter_pages(const sgmv_pool* pool, int32_t adapter_id, int32_t proj,
                                    int32_t matrix, int32_t* page_ids, int64_t cap, int64_t* n);
/*
 * Copy the stored form of (adapter, projection, matrix) to the host: `codes`
 * receives its r rank rows (matrix 0 = A: rows of d_in; 1 = B^T: rows of d_out)
 * in row order, as bf16 values (2 bytes each), E4M3 codes (1 byte each) or
 * packed INT4 codes (d / 2 bytes a row); `scales` (may be NULL) receives the r
 * row scales (1.0 for a bf16 pool).  Capacities are checked against cap_codes
 * bytes and cap_scales floats.  Waits for the copies.  For export and tests.
 */
SGMV_API sgmv_status sgmv_pool_read(const sgmv_pool* pool, int32_t adapter_id, int32_t proj, int32_t matrix,
                           void* codes, int64_t cap_codes, float* scales, int64_t cap_scales,
                           sgmv_stream_t stream);
/*
 * Reorder the free-page list pseudo-randomly (seeded), so that later loads
 * place consecutive chunks of a row on scattered pages.  Changes no resident
 * adapter.  For exercising the page-table indirection.
 */
SGMV_API sgmv_status sgmv_pool_shuffle_free_pages(sgmv_pool* pool, uint64_t seed);
/* Device address of the page buffer ([num_pages][page_bytes]); NULL for a
 * host-only pool.  For inspection and tests. */
SGMV_API const void* sgmv_pool_pages_device(const sgmv_pool* pool);

/* ------------------------------------------------------------------------ */
/* Segment builder and dispatch plan                                          */
/* ------------------------------------------------------------------------ */
/*
 * SGMV "groups the batch's tokens by adapter" and picks, per segment, tensor
 * cores for large segments and a batched gather path for small ones
 * ([SGMV post], "SGMV: the kernel that holds it all up", and the figure in
 * that section; heterogeneous ranks in one batch: TL;DR and the S-LoRA
 * MBGMM/MBGMV paragraph).
 *
 * The builder runs on the host.  It writes one table (host memory, 16-byte
 * aligned arrays at the byte offsets below) that the caller copies to the
 * device as is, and fills the plan header, which stays on the host.
 *
 *   token_idx   int32 [num_rows]         sorted row -> token (row of x and y)
 *   seg_offsets int32 [num_segments+1]   rows of segment s: [off[s], off[s+1])
 *   seg_adapter int32 [num_segments]
 *   seg_rank    int32 [num_segments]
 *   seg_scale   float [num_segments]     the segment's adapter multiplier
 *                                        (sgmv_pool_set_adapter_scale) at build time
 *   seg_a_pt    int64 [num_segments*n_proj]  first page-table entry of A, per projection
 *   seg_b_pt    int64 [num_segments*n_proj]  first page-table entry of B^T
 *   simt_items  record [num_simt_items][n_proj]
 *   tc_tiles    record [num_tc_tiles][n_proj]   (<= 128 rows each)
 *               record = {int32 segment, row_begin, row_end, rank;
 *                         int64 first page-table entry of A, of B^T (for that projection)}
 *
 * Segments are in ascending adapter id; rows of a segment keep batch order
 * (stable).  Tokens with adapter id -1 are in no segment and their y rows
 * are never touched.  Segments of rank 0 produce no work item.  A segment
 * with at least `long_threshold` rows goes to the tensor-core path as
 * 128-row tiles; shorter segments go to the SIMT path as items of at most
 * 4 rows (long_threshold <= 0 selects the built-in default, 16; a huge value
 * keeps every segment on the SIMT path; 1 sends every segment to tensor cores).
 * With the default, the tensor-core path is taken only when the long segments
 * hold at least 128 rows in total (one full tile); below that every segment
 * goes to the SIMT path and the plan's long_threshold reads INT32_MAX.
 */
typedef struct {
    int32_t T;              /* tokens in the batch                                   */
    int32_t num_segments;   /* S                                                     */
    int32_t num_rows;       /* tokens in some segment (= off[S]); rows of v           */
    int32_t max_rank;       /* R = max segment rank; v needs ldv >= R                */
    int32_t n_proj;
    int32_t num_simt_items;
    int32_t num_tc_tiles;
    int32_t long_threshold; /* the threshold actually used                           */
    int32_t max_item_rows;  /* largest SIMT item                                     */
    int32_t needs_device_table; /* 0: the kernels take everything from `host_table` as
                               launch arguments (no tensor-core tiles and <= 256 SIMT
                               items, or <= 64 for a pool of several projections, whose
                               grouped calls need the table); the device table may then
                               be NULL and need not be copied */
    int64_t table_bytes;    /* bytes of the table to copy to the device              */
    int64_t off_token_idx, off_seg_offsets, off_seg_adapter, off_seg_rank;
    int64_t off_seg_a_pt, off_seg_b_pt, off_simt_items, off_tc_tiles;
    const void* host_table; /* the host table the builder wrote; it must still hold that
                               table when sgmv_shrink / sgmv_expand are called          */
    int64_t off_seg_scale;
} sgmv_plan;

/* ------------------------------------------------------------------------
 * Residency manager: adapters kept in host memory and made resident in the
 * pool on demand, batch by batch.  "Multi-LoRA serving: the single translator
 * ...", the figure of section "SGMV: the kernel that holds it all up" (an HBM
 * pool of hot adapters over a host-RAM cache: LRU eviction, asynchronous
 * host-to-device copies on use) and "Operational pitfalls" (eviction: LRU by
 * default); "Multi-LoRA Inference Serving ..." (clusterbid.com), the vLLM
 * memory-pool paragraph (an adapter not resident is loaded from host memory
 * into the pool, evicting a least-recently-used one).
 *
 * Use from one host thread with the pool (no other pool_load / pool_evict
 * while a manager call runs).  Adapters loaded directly with sgmv_pool_load
 * take part in the LRU order as the oldest.
 */
typedef struct sgmv_residency sgmv_residency;

typedef struct {
    int64_t hits;          /* batch adapters already resident                      */
    int64_t misses;        /* batch adapters loaded from their host copies         */
    int64_t evictions;     /* adapters evicted to make room                        */
    int64_t bytes_loaded;  /* host -> device bytes of adapter matrices             */
} sgmv_residency_stats;

/* A manager over `pool` (not owned).  A device pool gets a device staging buffer
 * of one largest adapter matrix and two events. */
SGMV_API sgmv_status sgmv_residency_create(sgmv_pool* pool, sgmv_residency** out);
/* Synchronises the pool's device, frees the manager (not the pool). */
SGMV_API sgmv_status sgmv_residency_destroy(sgmv_residency* r);

/* Host copies of an adapter: A[p] bf16 [rank][d_in_p], B[p] bf16 [d_out_p][rank]
 * per projection (the layouts of sgmv_pool_load), owned by the caller and valid
 * until unregistered.  Pinned (page-locked) memory lets the copies run
 * asynchronously.  Re-registering replaces the pointers. */
SGMV_API sgmv_status sgmv_residency_register(sgmv_residency* r, int32_t adapter_id, int32_t rank,
                                             const void* const* A_host, const void* const* B_host);
SGMV_API sgmv_status sgmv_residency_unregister(sgmv_residency* r, int32_t adapter_id);

/*
 * Make every adapter of a batch (adapter_ids: host int32[T], -1 = none)
 * resident before the batch's kernels run:
 *   - adapters already resident count as hits and become the most recently used;
 *   - missing ones are loaded from their host copies: their page-table entries
 *     and pages are written by copies and scatter kernels on `copy_stream`;
 *   - when the free pages do not suffice, resident adapters that the batch does
 *     not use are evicted, least recently used first (ties: lowest id);
 *   - the copies that overwrite pages wait for the work already queued on
 *     `compute_stream` (an event), and `compute_stream` waits for the copies
 *     (another event): kernels enqueued on it afterwards see the adapters.
 * Build the batch's plan after this call (the page-table bases may change).
 * *loaded (optional) = adapters loaded.  Errors, with nothing changed:
 * SGMV_ERR_NOT_RESIDENT (an adapter neither resident nor registered),
 * SGMV_ERR_OUT_OF_PAGES (the batch's adapters do not fit even with every other
 * adapter evicted).
 */
SGMV_API sgmv_status sgmv_residency_prepare(sgmv_residency* r, const int32_t* adapter_ids, int32_t T,
                                            sgmv_stream_t copy_stream, sgmv_stream_t compute_stream,
                                            int32_t* loaded);
SGMV_API sgmv_status sgmv_residency_get_stats(const sgmv_residency* r, sgmv_residency_stats* out);

/* Bytes a table may need for a batch of T tokens over n_proj projections. */
SGMV_API int64_t sgmv_plan_table_capacity(int32_t T, int32_t n_proj);

/*
 * adapter_ids: host int32[T], -1 = no adapter.  Every other id must be
 * resident in `pool` (else SGMV_ERR_NOT_RESIDENT).  `table` is host memory of
 * `table_capacity` bytes (see sgmv_plan_table_capacity), 16-byte aligned.
 * Host only; touches no device memory.
 */
SGMV_API sgmv_status sgmv_build_plan(const int32_t* adapter_ids, int32_t T, const sgmv_pool* pool,
                            int32_t long_threshold, void* table, int64_t table_capacity,
                            sgmv_plan* plan);

/* ------------------------------------------------------------------------ */
/* SGMV-shrink and SGMV-expand                                               */
/* ------------------------------------------------------------------------ */
/*
 * SGMV-shrink ([SGMV post], "SGMV: the kernel that holds it all up", phase 1:
 * projection d_in -> r with A_{a(t)}):
 *
 *   v[i][k] = sum_c A_s[k][c] * x[token_idx[i]][c]     for rows i of segment s, k < r_s
 *
 * x       device bf16 [T][ldx], ldx >= d_in, row starts 16-byte aligned
 * v       device fp32 [plan->num_rows][ldv], ldv >= plan->max_rank; written
 *         for k < r_s (other entries are left as they were); fp32 accumulation
 * proj    projection index, d_in must equal the pool's d_in[proj]
 * table   device copy of the table that built `plan` (may be NULL when
 *         plan->needs_device_table is 0: the work items then travel as launch
 *         arguments, read from plan->host_table at the call)
 * One launch covers every SIMT item (all short segments, any mix of ranks)
 * and one more covers every tensor-core tile, in stream order.  The SIMT
 * path needs the pool's page_elems <= 1024 (else SGMV_ERR_UNSUPPORTED).
 */
SGMV_API sgmv_status sgmv_shrink(const void* x, int64_t ldx, int32_t T, int32_t d_in, int32_t proj,
                        const sgmv_plan* plan, const void* table, const sgmv_pool* pool,
                        float* v, int64_t ldv, sgmv_stream_t stream);

/*
 * SGMV-expand ([SGMV post], "SGMV: the kernel that holds it all up", phase 2:
 * projection r -> d_out with B_{a(t)}, accumulated into Y as in the TL;DR's
 * "Y +=" form):
 *
 *   y[t][j] <- round( y[t][j] + (scale * s_s) * sum_{k < r_s} B_s[j][k] * v[i][k] ),  t = token_idx[i]
 *
 * computed in fp32 with one rounding to the output type; s_s is the multiplier
 * of segment s's adapter (seg_scale of the plan, 1.0 unless set with
 * sgmv_pool_set_adapter_scale).
 * y        device [T][ldy] updated in place, ldy >= d_out, rows 16-byte aligned;
 *          y_dtype 0 = bf16 (round to nearest even), 1 = fp32.
 * Rows of tokens in no segment are not read or written.
 * The SIMT launch is a programmatic dependent of the kernel before it in the
 * stream: it stages adapter pages while that kernel runs and reads v and y
 * only after that kernel has completed.
 */
SGMV_API sgmv_status sgmv_expand(const float* v, int64_t ldv, int32_t T, int32_t d_out, int32_t proj,
                        const sgmv_plan* plan, const void* table, const sgmv_pool* pool,
                        float scale, void* y, int64_t ldy, int32_t y_dtype,
                        sgmv_stream_t stream);

/*
 * Both phases in one call ([SGMV post], "SGMV: the kernel that holds it all
 * up": one pass computes the delta of every token):
 *
 *   y[t][j] <- round( y[t][j] + (scale * s_s) * sum_k B_s[j][k] * sum_c A_s[k][c] * x[t][c] )
 *
 * (s_s: the adapter's multiplier, as for sgmv_expand)
 * = sgmv_shrink into v, then sgmv_expand from v, on `stream`; the expand's
 * SIMT launch overlaps the shrink (programmatic dependent launch), and so does
 * its tensor-core launch when the plan has no SIMT items (it follows the
 * tensor-core shrink directly and reads v only after that shrink completes), so
 * the second launch costs little ([Glossary], "Limits and open questions", names
 * the extra launch per adapted layer as a cost of unmerged adapters).
 * x, y, y_dtype, d_in, d_out, proj as for sgmv_shrink / sgmv_expand.
 * v        device fp32 [plan->num_rows][ldv], ldv >= plan->max_rank: workspace
 *          for the intermediate A x (required whenever the plan has work);
 *          on return it holds v as sgmv_shrink writes it.
 */
SGMV_API sgmv_status sgmv_lora_delta(const void* x, int64_t ldx, int32_t T, int32_t d_in, int32_t d_out,
                                     int32_t proj, const sgmv_plan* plan, const void* table,
                                     const sgmv_pool* pool, float scale, void* y, int64_t ldy,
                                     int32_t y_dtype, float* v, int64_t ldv, sgmv_stream_t stream);

/*
 * Several projections of one layer over the same batch in one call: for each
 * entry, what sgmv_lora_delta does for it, but with one SIMT shrink launch and
 * one SIMT expand launch covering all entries (the tensor-core tiles still take
 * a shrink and an expand launch per entry).  A layer's projections share the
 * batch's adapter assignment ("Multi-LoRA serving: the single translator ...",
 * section "The maths that matters", memory table: q, k, v, o, gate, up and down
 * of Llama-3-70B under one adapter), so one plan serves all of them; the launch
 * boundaries between projections (each a tail and a ramp) go away.
 *
 * entries  host array of n_entries (1 .. 8); entry i: projection `proj` of the
 *          pool with its d_in / d_out, x (bf16 [T][ldx]), y ([T][ldy] of
 *          y_dtype, updated in place) and workspace v (fp32 [num_rows][ldv],
 *          ldv >= plan->max_rank), as for sgmv_lora_delta.  Workspaces must not
 *          overlap (SGMV_ERR_INVALID when two are the same pointer); a y must not
 *          be another entry's x.  The same projection may appear twice (with
 *          different x, y, v).
 * table    the plan's device table.  NULL is accepted for a plan that needs no
 *          device table: the entries then run one after another.
 * Errors as for sgmv_lora_delta; all entries are checked before any launch.
 */
typedef struct {
    int32_t proj;
    int32_t d_in;
    int32_t d_out;
    int32_t reserved;       /* 0 */
    const void* x;
    int64_t ldx;
    void* y;
    int64_t ldy;
    float* v;
    int64_t ldv;
} sgmv_delta_entry;

SGMV_API sgmv_status sgmv_lora_delta_grouped(const sgmv_delta_entry* entries, int32_t n_entries, int32_t T,
                                             const sgmv_plan* plan, const void* table, const sgmv_pool* pool,
                                             float scale, int32_t y_dtype, sgmv_stream_t stream);

/*
 * Copy the plan's table (plan->table_bytes from plan->host_table) to its device
 * copy `device_table` (16-byte aligned, at least table_bytes), in stream order.
 * When the host table is pinned (cudaHostAlloc / cudaMallocHost, device-visible
 * through unified addressing) a small kernel reads it across the bus with
 * coalesced 16-byte loads, which costs a few microseconds where a copy-engine
 * transfer of a table this small takes about ten; pageable memory takes a
 * cudaMemcpyAsync.  The host table must keep its contents until the copy has run
 * (stream order).  Errors: SGMV_ERR_INVALID (null or misaligned tables, a
 * table_bytes that is not a multiple of 16), SGMV_ERR_CUDA.
 */
SGMV_API sgmv_status sgmv_upload_table(const sgmv_plan* plan, void* device_table, sgmv_stream_t stream);

/*
 * Which kernels sgmv_lora_delta (n_entries = 1) or sgmv_lora_delta_grouped (the
 * entries' projections `projs`, with the same `table`, NULL or not) launch for
 * this plan and pool, without launching anything.  The calls' own choices are
 * made, including the test of the one-shot fused kernel (every SIMT item's
 * cluster resident in one wave: an occupancy query on the pool's device, which
 * becomes the calling thread's current device).
 *
 * kinds     out: a mask of SGMV_KERNELS_FUSED (the one-shot fused SIMT kernel),
 *           SGMV_KERNELS_SIMT (a SIMT shrink and expand pair), SGMV_KERNELS_SLAB
 *           (set with SGMV_KERNELS_SIMT: the pair's shrink is the one-shot slab
 *           kernel, each CTA's whole slice of A staged at once, instead of the
 *           streaming one) and SGMV_KERNELS_TC (the tensor-core shrink and expand
 *           of long segments); 0 when the plan has no work.
 * launches  out: kernel launches the call makes.
 * Errors: SGMV_ERR_INVALID (null pointers, a pool without device memory,
 * n_entries outside 1..8, a projection outside the pool, y_dtype not 0 or 1, a
 * plan built for another pool), SGMV_ERR_CUDA.
 */
enum {
    SGMV_KERNELS_FUSED = 1,
    SGMV_KERNELS_SIMT = 2,
    SGMV_KERNELS_TC = 4,
    SGMV_KERNELS_SLAB = 8,
};
SGMV_API sgmv_status sgmv_lora_delta_kernels(const sgmv_plan* plan, const sgmv_pool* pool, const int32_t* projs,
                                             int32_t n_entries, const void* table, int32_t y_dtype,
                                             int32_t* kinds, int32_t* launches);

/*
 * The whole step from host buffers: the segment builder, the host-to-device
 * copies of the step's inputs, the grouped delta and the device-to-host copy
 * of the results, enqueued on `stream` by the library (no Python or other
 * caller work between them).  For serving loops whose activations live in
 * host memory, and for measuring the path end to end.
 *
 * adapter_ids   host int32[T] (-1 = no adapter), as for sgmv_build_plan
 * entries       host array of n_entries (1 .. 8): projection `proj` with its
 *               d_in / d_out, x_host (bf16 [T][d_in], rows contiguous) and
 *               y_host ([T][d_out] of y_dtype, rows contiguous, updated in place).
 *               Entries that name the same x_host (and d_in) share one copy
 *               of it and one stacked shrink pass (as in sgmv_lora_delta_grouped).
 * host_table    host memory of host_table_bytes >= sgmv_plan_table_capacity(T,
 *               pool's n_proj), 16-byte aligned; the plan is built into it and
 *               *plan_out (may be NULL) receives its header.
 * workspace     device memory of workspace_bytes >= sgmv_host_workspace_bytes(...),
 *               256-byte aligned: the device copies of the table, of every
 *               distinct x and of every y, and the intermediates v.
 * Host buffers should be pinned (page-locked) for the copies to run
 * asynchronously.  The call returns once everything is enqueued: y_host holds
 * the results, and host_table, x_host and y_host may be reused, only after the
 * stream has completed.  *h2d_bytes / *d2h_bytes (may be NULL) receive the bytes
 * the copies move.  Errors as for sgmv_build_plan and sgmv_lora_delta_grouped
 * (nothing is enqueued), SGMV_ERR_CAPACITY for a workspace or table too small.
 */
typedef struct {
    int32_t proj;
    int32_t d_in;
    int32_t d_out;
    int32_t reserved;       /* 0 */
    const void* x_host;
    void* y_host;
} sgmv_host_entry;

/* Device workspace bytes sgmv_lora_delta_host needs for a batch of T tokens
 * (an upper bound over every batch of T tokens on this pool); -1 on a bad argument. */
SGMV_API int64_t sgmv_host_workspace_bytes(int32_t T, const sgmv_pool* pool, const sgmv_host_entry* entries,
                                           int32_t n_entries, int32_t y_dtype);

SGMV_API sgmv_status sgmv_lora_delta_host(const int32_t* adapter_ids, int32_t T, const sgmv_pool* pool,
                                          const sgmv_host_entry* entries, int32_t n_entries, float scale,
                                          int32_t y_dtype, void* host_table, int64_t host_table_bytes,
                                          void* workspace, int64_t workspace_bytes, sgmv_plan* plan_out,
                                          int64_t* h2d_bytes, int64_t* d2h_bytes, sgmv_stream_t stream);

/*
 * sgmv_lora_delta for callers that cannot give the library device memory.
 * No counterpart on the pages: this is a deployment convenience.
 *
 * Some callers cannot allocate (their device memory belongs to another
 * runtime's fixed arena, or the library must not grow the process's device
 * footprint or trigger cudaMalloc's synchronisation).  This call takes the
 * same arguments as sgmv_lora_delta without v: the intermediate lives in a
 * fixed array of 2^19 fp32 (2 MiB) compiled into the library, which every GPU
 * that loads the library holds until the process exits.  It allocates nothing
 * and calls no allocating routine.
 *   - The batch must fit: plan->num_rows * max(4, round_up(plan->max_rank, 4))
 *     <= 2^19, else SGMV_ERR_CAPACITY (nothing launched).
 *   - The first call on a device looks up the array's device address, with
 *     that device current; make that first call before any stream capture.
 *     The address is kept for the life of the process: after cudaDeviceReset
 *     (which ends the context the address belongs to) do not call this entry
 *     point on that device again.
 *   - All calls on a device share the array, which keeps the last call's
 *     contents (nothing in it needs to start at zero).  Calls whose kernels
 *     overlap on the same device race on it: serialise them (one stream).
 */
SGMV_API sgmv_status sgmv_lora_delta_noalloc(const void* x, int64_t ldx, int32_t T, int32_t d_in,
                                             int32_t d_out, int32_t proj, const sgmv_plan* plan,
                                             const void* table, const sgmv_pool* pool, float scale,
                                             void* y, int64_t ldy, int32_t y_dtype,
                                             sgmv_stream_t stream);

/*
 * Wait for `stream`, then return and clear the device error word:
 * SGMV_OK, SGMV_ERR_BOUNDS or SGMV_ERR_TIMEOUT.  *flags (may be NULL) receives
 * the raw bits (1 = page id out of range, 2 = token row out of range,
 * 4 = wait timed out, 8 = segment rows out of range).
 */
SGMV_API sgmv_status sgmv_check_errors(sgmv_stream_t stream, uint32_t* flags);

#ifdef __cplusplus
}
#endif
#endif /* SGMV_B200_H */
