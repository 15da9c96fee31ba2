// Tensor-core (tcgen05) path of SGMV-shrink and SGMV-expand for long
// segments (prefill): "for large segments (several requests with the same
// adapter) it goes through tensor cores" -- "Multi-LoRA serving: the single
// translator with a thousand glossaries ..." (blog.lo0.es), section "SGMV: the
// kernel that holds it all up".  A long segment is a real dense contraction:
//
//   shrink  V[128 rows, r]     = X[128 rows, d_in] * A^T          (M=128, N=r padded to 16)
//   expand  Y[128 rows, 128 j] += scale * V[128 rows, r] * B^T    (M=128, N=128, K=r padded to 16)
//
// Operands are staged in shared memory in the 128-byte swizzle by producer
// warps -- X tiles and y blocks of consecutive tokens by 2-D TMA, gathered rows
// (through the segment's token list) and A / B^T chunks (through the page
// table) by 16-byte cp.async -- and multiplied by one thread issuing
// tcgen05.mma (bf16 inputs, fp32 accumulator in tensor memory); mbarriers link
// the producer, MMA and epilogue roles, and the epilogue reads the accumulator
// with tcgen05.ld.
//
// shrink: a cluster of KS CTAs splits d_in; each accumulates its K range in
// tensor memory, and the KS partial tiles are summed in a fixed order through
// distributed shared memory into v.
// expand: persistent CTAs over (tile, column block) units with a
// double-buffered accumulator; v (fp32) is split into bf16 hi + lo parts so
// that the delta keeps ~16 bits of v: D = V_hi B + V_lo B, both products
// exact, fp32 accumulation.
// Quantised pools (template parameter WF): the producers move E4M3 / INT4
// codes by cp.async into a small ring of code slots and convert them to bf16
// (exact) in the swizzled operand tile; the row scales of A multiply v in the
// shrink's epilogue, those of B^T multiply v before the hi / lo split.
#include <cuda.h>  // CUtensorMap (the encoder is reached through the runtime's driver entry point)
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "internal.h"
#include "ptx.cuh"

namespace sgmv {
namespace {

__device__ unsigned int g_err_tc;

constexpr int kKTile = 64;          // K columns per pipeline stage (shrink)
constexpr int kShrinkStages = 4;
constexpr int kShrinkThreads = 160;  // 4 producer / epilogue warps + 1 MMA warp
constexpr int kShrinkCodeSlots = 2;  // quantised pools: k-tiles of A codes in flight

struct ShrinkTcArgs {
    const uint16_t* x;
    int64_t ldx;
    int32_t d_in;
    BatchView b;
    PoolView pool;
    float* v;
    int64_t ldv;
    int32_t ks;          // CTAs per cluster (split of d_in)
    int32_t kcols;       // d_in columns per CTA (multiple of kKTile)
    int32_t npad_max;    // largest padded rank of the launch (multiple of 16)
    int32_t tmem_cols;   // tensor-memory columns allocated per CTA
    int32_t pid_offset;  // byte offset of the page-id table in shared memory
    int32_t raw_offset;  // quantised pools: byte offset of the ring of A codes in shared memory
    int32_t use_tma;     // tmap_x is valid: tiles whose rows are consecutive tokens load X by TMA
};

struct ExpandTcArgs {
    const float* v;
    int64_t ldv;
    int32_t d_out;
    BatchView b;
    PoolView pool;
    float scale;
    void* y;
    int64_t ldy;
    int32_t y_dtype;
    int32_t n_blocks;       // y column blocks per tile (d_out / columns per unit)
    int32_t num_units;      // tiles x n_blocks
    int32_t units_per_cta;  // contiguous run of units per CTA
    int32_t kpad_max;
    int32_t use_tma;        // tmap_y is valid: tiles of consecutive tokens move y by TMA
    int32_t raw_slots;      // quantised pools: slots of B^T codes (2: converted one unit later; 1: at once)
};

__device__ __forceinline__ int32_t safe_page(const PoolView& pool, int64_t entry) {
    int32_t page = (entry >= 0 && entry < pool.pt_capacity) ? pool.page_table[entry] : -1;
    if (page < 0 || page >= pool.num_pages) {
        atomicOr(&g_err_tc, kErrPage);
        page = 0;
    }
    return page;
}

// Codes of a quantised pool: 8 values (8 bytes E4M3 / 4 bytes INT4) of a page,
// read through the non-coherent path, and their exact bf16 form (16 bytes).
template <int WF>
struct Codes8 {
    using T = typename std::conditional<WF == kFmtFp8, uint2, uint32_t>::type;
};
template <int WF>
__device__ __forceinline__ typename Codes8<WF>::T load_codes8(const uint8_t* p) {
    return __ldg(reinterpret_cast<const typename Codes8<WF>::T*>(p));
}
template <int WF>
__device__ __forceinline__ uint4 codes8_to_bf16(const typename Codes8<WF>::T& c) {
    float f[8];
    if constexpr (WF == kFmtFp8) fp8x8_to_f32(c, f);
    else int4x8_to_f32(c, f);
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)  // exact: every code value has at most 4 significant bits
        w[e] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f[2 * e])) |
               ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f[2 * e + 1])) << 16);
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// ------------------------------------------------------------------ shrink
__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    const uint32_t s = smem_u32(p);
    return p + ((1024u - (s & 1023u)) & 1023u);
}

// Warp roles: warps 0-3 (128 threads) fill the stage ring with cp.async and
// then read the accumulator out; warp 4 owns the tensor memory and one of its
// lanes issues the MMAs.  Stage s is "full" once all 128 producers' copies
// into it have landed (cp.async.mbarrier.arrive.noinc, count 128) and "empty"
// once the MMAs that read it have completed (tcgen05.commit).  Every wait is
// bounded; a wait that gives up sets kErrTimeout and the CTA's abort flag, and
// the remaining waits of the CTA are skipped.
template <int WF>
__global__ void __launch_bounds__(kShrinkThreads) shrink_tc_kernel(const ShrinkTcArgs a,
                                                                     const __grid_constant__ CUtensorMap tmap_x) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    __shared__ uint64_t full_bar[kShrinkStages], empty_bar[kShrinkStages], acc_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ volatile int abort_flag;
    __shared__ int32_t tok_s[kTcTileRows];
    __shared__ float rsc_s[kMaxRank];  // row scales of a quantised A

    const int tid = threadIdx.x, warp = tid >> 5;
    // a dependent expand may be scheduled now: its CTAs take SMs as these CTAs leave, and
    // wait for this grid's completion before they read v
    pdl_launch_dependents();
    const int tile_idx = blockIdx.x / a.ks;
    const uint32_t q = cluster_ctarank();
    const ItemRec it = a.b.tc_tiles[(int64_t)tile_idx * a.b.n_proj + a.b.proj];
    int rows = it.row_end - it.row_begin, r = 0;
    int64_t a_base = 0;
    bool ok = !(it.seg < 0 || it.seg >= a.b.num_segments || it.row_begin < 0 || rows <= 0 ||
                rows > kTcTileRows || it.row_end > a.b.num_rows);
    if (ok) {
        r = it.rank;
        a_base = it.a_pt;
        ok = r > 0 && ((r + 15) & ~15) <= a.npad_max;
    }
    if (!ok && tid == 0) atomicOr(&g_err_tc, kErrRows);
    const int npad = ok ? ((r + 15) & ~15) : 16;

    const int x_tile_bytes = kTcTileRows * kKTile * 2;      // 16 KB
    const int a_tile_bytes = a.npad_max * kKTile * 2;
    const int stage_bytes = x_tile_bytes + a_tile_bytes;
    uint8_t* stage0 = smem;

    if (tid == 0) {
        abort_flag = 0;
        // full: the producers' cp.async arrivals, plus (quantised pools) their arrivals
        // after storing the converted A codes
        for (int i = 0; i < kShrinkStages; ++i) {
            mbar_init(&full_bar[i], WF == kFmtBf16 ? kTcTileRows : 2 * kTcTileRows);
            mbar_init(&empty_bar[i], 1);
        }
        mbar_init(&acc_bar, 1);
        fence_mbar_init();
    }
    if (warp == 4) {
        tmem_alloc(&tmem_slot, (uint32_t)a.tmem_cols);
        tmem_relinquish();
    }

    const int P_log2 = a.pool.page_log2;
    const int pages_per_row = a.d_in >> P_log2;
    const int k_begin = (int)q * a.kcols;
    const int nk = a.kcols / kKTile;

    // token of each tile row (-1: none) and the page ids of the A rows over this
    // CTA's K range ([rank row][page]; the range may start and end inside a page),
    // each in one round of independent loads
    if (tid < kTcTileRows) {
        int t = -1;
        if (ok && tid < rows) {
            t = a.b.token_idx[it.row_begin + tid];
            if (t < 0 || t >= a.b.T) {
                atomicOr(&g_err_tc, kErrToken);
                t = -1;
            }
        }
        tok_s[tid] = t;
    }
    const int first_page = k_begin >> P_log2;
    const int span_pages = ((k_begin + a.kcols - 1) >> P_log2) - first_page + 1;
    int32_t* pid_s = reinterpret_cast<int32_t*>(smem + a.pid_offset);
    for (int e = tid; e < r * span_pages; e += kShrinkThreads) {
        const int n = e / span_pages, pc = e - n * span_pages;
        pid_s[e] = safe_page(a.pool, a_base + (int64_t)n * pages_per_row + first_page + pc);
    }
    if (WF != kFmtBf16)
        for (int n = tid; n < r; n += kShrinkThreads) {
            const int64_t e = a_base + (int64_t)n * pages_per_row;
            rsc_s[n] = (e >= 0 && e < a.pool.pt_capacity) ? a.pool.row_scale[e] : 0.f;
        }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    // rows that are consecutive tokens (a prefill segment): X tiles come by one TMA
    // load each, 128 rows of 128 bytes in the same 128-byte swizzle (rows past the
    // tile are other tokens or zero fill; their results are discarded)
    const int t0 = tok_s[0];
    const bool x_tma = __syncthreads_and(tid >= rows || tid >= kTcTileRows || (t0 >= 0 && tok_s[tid] == t0 + tid)) &&
                       a.use_tma && ok;

    if (warp < 4) {
        // ---- producers.  Tiles are K-major with the 128-byte swizzle (8-row atoms of
        // 128-byte rows, 1024-byte aligned).  Granule g (16 bytes): row g >> 3,
        // chunk g & 7, so each 8-lane quarter of a warp copies one row's 128
        // contiguous bytes into one (permuted) 128-byte row of shared memory.
        auto issue_x = [&](int kt, uint8_t* xs) {
            const int c = k_begin + kt * kKTile;
            if (x_tma) {
                if (tid == 0) {
                    mbar_expect_tx(&full_bar[kt % kShrinkStages], (uint32_t)x_tile_bytes);
                    tma_load_2d(xs, &tmap_x, c, t0, &full_bar[kt % kShrinkStages]);
                }
            } else {
#pragma unroll
                for (int i = 0; i < (kTcTileRows * 8) / kTcTileRows; ++i) {
                    const int g = tid + i * kTcTileRows;
                    const int row = g >> 3, kg = g & 7;
                    const int t = tok_s[row];
                    const uint32_t off = (uint32_t)(row >> 3) * 1024 + sw128_off((uint32_t)row, (uint32_t)kg);
                    const uint16_t* src = t >= 0 ? a.x + (int64_t)t * a.ldx + c + kg * 8 : a.x;
                    cp_async16(xs + off, src, t >= 0);
                }
            }
        };
        auto wait_empty = [&](int kt) {
            if (kt >= kShrinkStages && !abort_flag &&
                !mbar_wait(&empty_bar[kt % kShrinkStages], (uint32_t)((kt / kShrinkStages - 1) & 1), &g_err_tc))
                abort_flag = 1;
        };
        if constexpr (WF == kFmtBf16) {
            // A: rank rows n < npad (zero past r); the thread's granules g = tid + 128 i are
            // rank rows (tid >> 3) + 16 i at column chunk tid & 7.  Their page ids stay in
            // registers while the K tiles stay in one page, so a stage issues its copies
            // back to back without a shared-memory load in front of each.
            constexpr int kMaxI = kMaxRank * 8 / kTcTileRows;
            const int n_i = npad / 16, kg = tid & 7;
            int32_t pg[kMaxI];
            int cur_rel = -1;
            for (int kt = 0; kt < nk; ++kt) {
                const int st = kt % kShrinkStages;
                wait_empty(kt);
                uint8_t* xs = stage0 + (size_t)st * stage_bytes;
                uint8_t* as = xs + x_tile_bytes;
                const int c = k_begin + kt * kKTile;
                issue_x(kt, xs);
                // the 64 columns lie in one page
                const int page_rel = (c >> P_log2) - first_page, in_page = c & ((1 << P_log2) - 1);
                if (page_rel != cur_rel) {
                    cur_rel = page_rel;
#pragma unroll
                    for (int i = 0; i < kMaxI; ++i) {
                        const int n = (tid >> 3) + 16 * i;
                        pg[i] = (i < n_i && ok && n < r) ? pid_s[n * span_pages + page_rel] : 0;
                    }
                }
#pragma unroll
                for (int i = 0; i < kMaxI; ++i) {
                    if (i < n_i) {
                        const int n = (tid >> 3) + 16 * i;
                        const uint32_t off = (uint32_t)(n >> 3) * 1024 + sw128_off((uint32_t)n, (uint32_t)kg);
                        const bool valid = ok && n < r;
                        const uint16_t* src =
                            valid ? a.pool.pages + ((int64_t)pg[i] << P_log2) + in_page + kg * 8 : a.pool.pages;
                        cp_async16(as + off, src, valid);
                    }
                }
                cp_async_commit();  // close the group: the copies of every stage form their own
                cp_async_mbar_arrive_noinc(&full_bar[st]);
            }
        } else {
            // Quantised A: the codes of k-tile kt travel by cp.async into raw slot kt % D,
            // D k-tiles ahead of their use; at iteration kt a thread waits for its own
            // copies of tile kt (one commit group per iteration), converts them to bf16
            // into the swizzled A tile, fences them to the async proxy and arrives on the
            // stage's barrier a second time.  Granule g (8 values) of a tile: rank row
            // g >> 3, columns 8 (g & 7); a thread handles g = tid + 128 i.  Two slots keep
            // the shared memory of two CTAs per SM within the limit.
            constexpr int D = kShrinkCodeSlots;
            constexpr int VB = bytes_per_8<WF>();
            const int page_shift = P_log2 + (WF == kFmtFp8 ? 0 : -1);
            const uint8_t* pages8 = reinterpret_cast<const uint8_t*>(a.pool.pages);
            uint8_t* raw0 = smem + a.raw_offset;
            const int raw_slot = a.npad_max * 8 * VB;
            // granules g = tid + 128 i: rank row (tid >> 3) + 16 i, column chunk tid & 7; their
            // page ids stay in registers while the K tiles stay in one page
            constexpr int kMaxI = kMaxRank * 8 / kTcTileRows;
            const int n_i = npad / 16, kg = tid & 7;
            int32_t pg[kMaxI];
            int cur_rel = -1;
            auto issue_codes = [&](int kt) {
                const int c = k_begin + kt * kKTile;
                const int page_rel = (c >> P_log2) - first_page, in_page = c & ((1 << P_log2) - 1);
                uint8_t* raw = raw0 + (size_t)(kt % D) * raw_slot;
                if (page_rel != cur_rel) {
                    cur_rel = page_rel;
#pragma unroll
                    for (int i = 0; i < kMaxI; ++i) {
                        const int n = (tid >> 3) + 16 * i;
                        pg[i] = (i < n_i && ok && n < r) ? pid_s[n * span_pages + page_rel] : 0;
                    }
                }
#pragma unroll
                for (int i = 0; i < kMaxI; ++i) {
                    const int n = (tid >> 3) + 16 * i;
                    if (i < n_i && ok && n < r)
                        cp_async_n<VB>(raw + (tid + kTcTileRows * i) * VB,
                                       pages8 + ((int64_t)pg[i] << page_shift) + (in_page / 8 + kg) * VB);
                }
            };
#pragma unroll 1
            for (int kt = 0; kt < D; ++kt) {
                if (kt < nk) issue_codes(kt);
                cp_async_commit();
            }
            for (int kt = 0; kt < nk; ++kt) {
                const int st = kt % kShrinkStages;
                wait_empty(kt);
                uint8_t* xs = stage0 + (size_t)st * stage_bytes;
                uint8_t* as = xs + x_tile_bytes;
                issue_x(kt, xs);
                cp_async_wait<D - 1>();  // groups up to the one holding tile kt's codes
                const uint8_t* raw = raw0 + (size_t)(kt % D) * raw_slot;
                for (int g = tid; g < npad * 8; g += kTcTileRows) {
                    const int n = g >> 3, kg = g & 7;
                    typename Codes8<WF>::T cv{};
                    if (ok && n < r) cv = *reinterpret_cast<const typename Codes8<WF>::T*>(raw + g * VB);
                    *reinterpret_cast<uint4*>(as + (uint32_t)(n >> 3) * 1024 + sw128_off((uint32_t)n, (uint32_t)kg)) =
                        codes8_to_bf16<WF>(cv);
                }
                fence_proxy_async_smem();
                mbar_arrive(&full_bar[st]);
                cp_async_mbar_arrive_noinc(&full_bar[st]);  // this thread's x copies (and earlier codes)
                if (kt + D < nk) issue_codes(kt + D);        // into the slot just converted
                cp_async_commit();
            }
        }
    } else if (tid == 4 * 32) {
        // ---- MMA issuer
        const uint32_t idesc = idesc_bf16_f32(128, npad, false, false);
        for (int kt = 0; kt < nk; ++kt) {
            const int st = kt % kShrinkStages;
            if (!abort_flag && !mbar_wait(&full_bar[st], (uint32_t)((kt / kShrinkStages) & 1), &g_err_tc))
                abort_flag = 1;
            fence_proxy_async_smem();  // the copies above were made through the generic proxy
            tc_fence_after();
            const uint32_t xs = smem_u32(stage0 + (size_t)st * stage_bytes);
            const uint32_t as = xs + (uint32_t)x_tile_bytes;
#pragma unroll
            for (int ks = 0; ks < kKTile / 16; ++ks) {  // K step of 16 = 32 bytes inside the swizzled rows
                const uint64_t ad = smem_desc_sw128(xs + ks * 32, 16, 1024);
                const uint64_t bd = smem_desc_sw128(as + ks * 32, 16, 1024);
                tc_mma_bf16(tmem, ad, bd, idesc, kt > 0 || ks > 0);
            }
            tc_commit(&empty_bar[st]);
        }
        tc_commit(&acc_bar);  // every MMA of the tile has completed
    }
    __syncwarp();  // warp 4 reconverges before the warp-collective instructions below

    // ---- epilogue: tensor memory -> red[128][RS] (reuses the stages).  RS = npad_max + 4 is
    // 4 or 20 modulo 32 words, so the 16-byte stores of 8 consecutive rows (one store
    // phase) fall into 8 different 4-bank groups, and every 4 columns are one 16-byte word
    // for the cluster reduction below.
    float* red = reinterpret_cast<float*>(smem);
    const int RS = a.npad_max + 4;
    if (warp < 4) {
        if (!abort_flag && !mbar_wait(&acc_bar, 0u, &g_err_tc)) abort_flag = 1;
        tc_fence_after();
        const int m = warp * 32 + (tid & 31);
        for (int c0 = 0; c0 < npad; c0 += 32) {
            uint32_t regs[32];
            tmem_ld_32x32b_x32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, regs);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; e += 4)
                if (c0 + e < a.npad_max)
                    *reinterpret_cast<float4*>(red + m * RS + c0 + e) =
                        make_float4(__uint_as_float(regs[e]), __uint_as_float(regs[e + 1]),
                                    __uint_as_float(regs[e + 2]), __uint_as_float(regs[e + 3]));
        }
    }
    tc_fence_before();
    cluster_sync();

    if (ok && !abort_flag) {
        // CTA q sums rows [m0, m1) of the KS partial tiles, 4 rank columns per 16-byte load
        const int KS = a.ks, G = npad / 4;
        const int m0 = (int)((kTcTileRows * q) / KS), m1 = (int)((kTcTileRows * (q + 1)) / KS);
        const uint32_t red_s = smem_u32(red);
        for (int e = tid; e < (m1 - m0) * G; e += kShrinkThreads) {
            const int mm = m0 + e / G, k4 = (e % G) * 4;
            if (mm >= rows || k4 >= r) continue;
            float4 pv[8];
#pragma unroll
            for (int qq = 0; qq < 8; ++qq)  // all loads in flight before the fixed-order sum
                pv[qq] = qq < KS ? ld_cluster_v4(map_cluster(red_s + 4u * (uint32_t)(mm * RS + k4), (uint32_t)qq))
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
            float sum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int qq = 0; qq < 8; ++qq) {
                sum[0] += pv[qq].x;
                sum[1] += pv[qq].y;
                sum[2] += pv[qq].z;
                sum[3] += pv[qq].w;
            }
            float* vrow = a.v + (int64_t)(it.row_begin + mm) * a.ldv;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                // a quantised row's scale leaves the sum: v_k = s_k * sum_c q_kc x_c
                if (k4 + c < r) vrow[k4 + c] = WF == kFmtBf16 ? sum[c] : sum[c] * rsc_s[k4 + c];
        }
    }
    cluster_sync();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, (uint32_t)a.tmem_cols);
    }
}

// ------------------------------------------------------------------ expand
// Persistent: CTA b takes a contiguous run of units (tile of <= 128 rows, block
// of kYRowBytes of y columns), so consecutive units mostly share the tile and
// its v rows.  Warp roles:
//   warps 8-11 (producers): per unit, fetch the token rows and B^T page ids (one
//     unit ahead); copy the y block (two 2-D TMA boxes that complete on the stage's
//     mbarrier by bytes when the tile's rows are consecutive tokens, else 16-byte
//     cp.async) and the B^T block (16-byte cp.async); then, when the tile changes,
//     write V_hi / V_lo (v split into bf16 hi + lo).  Launched as a programmatic
//     dependent of the shrink, they wait for it (griddepcontrol.wait) only there,
//     before the first read of v.
//   warp 12 (one lane): tcgen05.mma  acc[i & 1] = V_hi B + V_lo B  (N = block);
//     with bf16 y (YM), V carries the scale and the MMAs go on with acc += Y I:
//     the staged y block, already in the K-major 128-byte swizzle of an A
//     operand, times a 128 x 128 identity kept in shared memory (each product
//     y * 1 exact), so the accumulator ends as y + scale V B^T
//   warps 0-7 (epilogue): two groups of four warps take alternate units (the
//     group of unit i reads acc[i & 1]); warp w reads rows 32 (w % 4) .. + 31 of
//     the accumulator (tcgen05.ld) and either rounds it to bf16 into its y rows in
//     shared memory (YM) or adds scale * acc to them; the group then stores the
//     block: one TMA store per half for a full tile of consecutive tokens,
//     coalesced 16-byte stores otherwise.  (Measured on the long-prefill batch
//     without YM: the read-modify-write of y took 2 us of a unit's epilogue.)
// mbarriers: full[s] (producers' copies landed: 128 cp.async arrivals plus the
// TMA bytes), yfree[s] (the unit's epilogue group has stored slot s), accf[b]
// (MMAs done, tcgen05.commit), acce[b] (the group has read acc[b] out),
// vfull / vempty (V of a tile written / its last MMA done).  The accumulator
// is double-buffered in tensor memory, so the MMAs of unit i+1 overlap the
// epilogue of unit i.  Every wait is bounded.
constexpr int kYRowBytes = 256;             // y bytes of one tile row per unit (128 bf16 / 64 fp32)
constexpr int kMaxPagesPerUnit = 2;         // pages of one B^T row a unit spans (page_elems >= 64)
constexpr int kExpandThreads = 416;         // 8 epilogue + 4 producer warps + 1 MMA warp
constexpr int kExpandProducers = 128;
constexpr int kMmaWarp = 12;

// ESZ: bytes of a y element (2: bf16, 4: fp32); WF: weight format; YM: y enters the accumulator
// by an identity MMA (bf16 y only)
template <int S, int ESZ, int WF, bool YM>
__global__ void __launch_bounds__(kExpandThreads, 1) expand_tc_kernel(const ExpandTcArgs a,
                                                                      const __grid_constant__ CUtensorMap tmap_y) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    __shared__ uint64_t full_bar[S], yfree_bar[S], accf_bar[2], acce_bar[2], vfull_bar, vempty_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ volatile int abort_flag;
    __shared__ int32_t pid_s[S][kMaxRank * kMaxPagesPerUnit];  // B^T page ids of a unit [rank row][page]
    __shared__ int32_t tok_s[S][kTcTileRows];                    // producers: token of each row of a unit
    __shared__ int32_t tok_row[2][kTcTileRows];                  // epilogue groups: token of each row, -1 = none
    __shared__ float rsc_s[kMaxRank];                            // producers: row scales of a quantised B^T

    const int tid = threadIdx.x, warp = tid >> 5;
    const int u0 = blockIdx.x * a.units_per_cta, u1 = min(u0 + a.units_per_cta, a.num_units);
    if (u0 >= u1) return;  // uniform, before anything is allocated
    constexpr int esz = ESZ;
    constexpr int NB = kYRowBytes / ESZ;          // output columns per unit
    const int kpm = a.kpad_max;
    // V_hi / V_lo: K-major, 128-byte swizzle, blocks of 64 K columns (128 rows x 128 bytes each)
    const int kpmv = (kpm + 63) & ~63;
    uint8_t* vhi = smem;
    uint8_t* vlo = vhi + (size_t)kTcTileRows * kpmv * 2;
    // B^T block: MN-major, 128-byte swizzle: atoms of 8 K rows x 64 columns; atoms along N
    // 1024 bytes apart (lbo), 8-row K groups sbo_b apart
    constexpr uint32_t sbo_b = (uint32_t)(NB / 64) * 1024;
    uint8_t* bst = vlo + (size_t)kTcTileRows * kpmv * 2;          // [S][kpm x NB]
    const size_t b_bytes = (size_t)kpm * NB * 2;
    // Y block: two halves of 128 rows x 128 bytes, each in the 128-byte swizzle (as a
    // TMA box lands): chunk q of row m of half h at h * 16 KB + m * 128 + (q ^ (m & 7)) * 16
    uint8_t* yst = bst + (size_t)S * b_bytes;                      // [S][2][128 x 128 bytes]
    constexpr int kYHalf = kTcTileRows * (kYRowBytes / 2);
    const size_t y_bytes = 2 * (size_t)kYHalf;

    static_assert(!YM || ESZ == 2, "the identity MMA adds bf16 y only");
    // YM: the identity I[k][n] (k, n < NB = 128) in the layout of a B^T block with 128 K rows
    uint8_t* ident = nullptr;
    if constexpr (YM) {
        constexpr int VBq = bytes_per_8<WF>();
        uint8_t* const after = yst + (size_t)S * y_bytes +
                               (WF == kFmtBf16 ? 0 : (size_t)a.raw_slots * ((size_t)kpm * (NB / 8) * VBq));
        ident = align1024(after);
        for (int i = tid; i < NB * NB * 2 / 16; i += kExpandThreads)
            reinterpret_cast<uint4*>(ident)[i] = make_uint4(0u, 0u, 0u, 0u);
        __syncthreads();
        if (tid < NB) {
            const int k = tid;  // element (k, k): granule k / 8 of row k, value k % 8 inside it
            *reinterpret_cast<uint16_t*>(ident + (uint32_t)(k >> 3) * sbo_b + (uint32_t)(k >> 6) * 1024 +
                                         sw128_off((uint32_t)k, (uint32_t)(k >> 3)) + (k & 7) * 2) = 0x3F80;  // 1.0
        }
        fence_proxy_async_smem();  // the identity, to the async proxy (the barrier below orders it)
    }
    if (tid == 0) {
        abort_flag = 0;
        // full: the producers' cp.async arrivals, plus (quantised pools) their arrivals
        // after storing the converted B^T codes
        for (int i = 0; i < S; ++i) {
            mbar_init(&full_bar[i], WF == kFmtBf16 ? kExpandProducers : 2 * kExpandProducers);
            mbar_init(&yfree_bar[i], kTcTileRows);  // one epilogue group per unit
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&accf_bar[i], 1);
            mbar_init(&acce_bar[i], kTcTileRows);
        }
        mbar_init(&vfull_bar, 1);
        mbar_init(&vempty_bar, 1);
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&tmem_slot, (uint32_t)(2 * NB));
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    const int P_log2 = a.pool.page_log2;
    const int pages_per_row = a.d_out >> P_log2;
    uint8_t* const ybase = static_cast<uint8_t*>(a.y);

    struct Unit {
        int tile, row_begin, rows, r, j0;
        int64_t b_base;
        float sc;  // multiplier of the tile's adapter
        bool ok;
    };
    // unit u: its tile record; ok depends on the tile only, so it is the same for
    // every unit of a tile and for every thread
    auto unit = [&](int u) {
        Unit w;
        w.tile = u / a.n_blocks;
        w.j0 = (u - w.tile * a.n_blocks) * NB;
        const ItemRec it = a.b.tc_tiles[(int64_t)w.tile * a.b.n_proj + a.b.proj];
        w.row_begin = it.row_begin;
        w.rows = it.row_end - it.row_begin;
        w.r = it.rank;
        w.b_base = it.b_pt;
        w.ok = !(it.seg < 0 || it.seg >= a.b.num_segments || it.row_begin < 0 || w.rows <= 0 ||
                 w.rows > kTcTileRows || it.row_end > a.b.num_rows || w.r <= 0 || ((w.r + 15) & ~15) > kpm);
        w.sc = w.ok ? a.b.seg_scale[it.seg] : 1.f;
        return w;
    };
    auto wait = [&](uint64_t* bar, uint32_t parity) {
        if (!abort_flag && !mbar_wait(bar, parity, &g_err_tc)) abort_flag = 1;
    };

    if (warp >= 8 && warp < kMmaWarp) {
        // ------------------------------------------------------------ producers
        const int pt = tid - 256;  // 0 .. 127: also the tile row this thread handles
        const int npc = NB > (1 << P_log2) ? (NB >> P_log2) : 1;
        // indices of a unit (token row of this thread's tile row, <= 2 B^T page ids),
        // loaded one unit ahead so that their latency overlaps the current copies
        auto fetch = [&](const Unit& w, int& t, int& t0, int32_t (&pg)[2]) {
            t = t0 = -1;
            pg[0] = pg[1] = 0;
            if (!w.ok) return;
            t0 = a.b.token_idx[w.row_begin];  // (checked by the thread of row 0)
            if (pt < w.rows) {
                t = a.b.token_idx[w.row_begin + pt];
                if (t < 0 || t >= a.b.T) {
                    atomicOr(&g_err_tc, kErrToken);
                    t = -1;
                }
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int e = pt + h * kExpandProducers;
                if (e < w.r * npc) {
                    const int k = e / npc, pc = e - k * npc;
                    pg[h] = safe_page(a.pool, w.b_base + (int64_t)k * pages_per_row + (w.j0 >> P_log2) + pc);
                }
            }
        };
        int t_next, t0_next;
        int32_t pg_next[2];
        fetch(unit(u0), t_next, t0_next, pg_next);
        int ts = -1, cur_tile = -1;
        // V = v split into bf16 hi + lo for the unit's tile, when the tile changes
        auto v_split = [&](const Unit& w) {
            if (!(w.ok && w.tile != cur_tile)) return;
            pdl_wait();  // v is final once the preceding kernel (the shrink) has completed
            if (ts >= 0) wait(&vempty_bar, (uint32_t)(ts & 1));  // the MMAs of the previous tile are done
            if (WF != kFmtBf16) {  // v_k takes the scale of B^T row k
                if (pt < w.r) {
                    const int64_t e = w.b_base + (int64_t)pt * pages_per_row;
                    rsc_s[pt] = (e >= 0 && e < a.pool.pt_capacity) ? a.pool.row_scale[e] : 0.f;
                }
                named_bar_sync(1, kExpandProducers);
            }
            const int m = pt, kpad = (w.r + 15) & ~15;
            const bool row_ok = m < w.rows;
            const float vsc = a.scale * w.sc;
            const float* vrow = a.v + (int64_t)(w.row_begin + (row_ok ? m : 0)) * a.ldv;
            // v row in chunks of 64 floats, each chunk's 16-byte loads all in flight
            // (a load starts below r and below ldv, a multiple of 4: it stays in the row)
            float4 vq[16];
#pragma unroll
            for (int kg = 0; kg < kMaxRank / 8; ++kg) {
                if (kg >= kpad / 8) break;
                if ((kg & 7) == 0) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int k4 = kg * 8 + 4 * e;
                        vq[e] = (row_ok && k4 < w.r && k4 < a.ldv) ? *reinterpret_cast<const float4*>(vrow + k4)
                                                                   : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                }
                float f[8];
                const float4 q0 = vq[2 * (kg & 7)], q1 = vq[2 * (kg & 7) + 1];
                f[0] = q0.x; f[1] = q0.y; f[2] = q0.z; f[3] = q0.w;
                f[4] = q1.x; f[5] = q1.y; f[6] = q1.z; f[7] = q1.w;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    if (kg * 8 + e >= w.r) f[e] = 0.f;
                    else if (WF != kFmtBf16) f[e] *= rsc_s[kg * 8 + e];
                    if (YM) f[e] *= vsc;  // the call's scale times the adapter's
                }
                uint32_t hw[4], lw[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __nv_bfloat16 h0 = __float2bfloat16_rn(f[2 * e]);
                    const __nv_bfloat16 h1 = __float2bfloat16_rn(f[2 * e + 1]);
                    const __nv_bfloat16 l0 = __float2bfloat16_rn(f[2 * e] - __bfloat162float(h0));
                    const __nv_bfloat16 l1 = __float2bfloat16_rn(f[2 * e + 1] - __bfloat162float(h1));
                    hw[e] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
                    lw[e] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
                }
                const uint32_t off = (uint32_t)(kg >> 3) * (kTcTileRows * 128) + (uint32_t)(m >> 3) * 1024 +
                                     sw128_off((uint32_t)m, (uint32_t)kg);
                *reinterpret_cast<uint4*>(vhi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4*>(vlo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
            fence_proxy_async_smem();  // the tensor core reads V through the async proxy
            named_bar_sync(1, kExpandProducers);
            if (pt == 0) mbar_arrive(&vfull_bar);
            ++ts;
            cur_tile = w.tile;
        };
        constexpr int kGr = kMaxRank * (kYRowBytes / 16) / kExpandProducers;  // <= 16 B^T granules a thread
        // quantised pools: the unit's B^T codes go by cp.async into raw slot i % raw_slots
        // (granule g = this thread's g-th B^T granule, VB bytes) and are converted to bf16
        // into stage slot st once this thread's copies have landed: one unit later with two
        // raw slots (their latency overlaps the next unit's copies), at once with one
        constexpr int VB = bytes_per_8<WF>();
        uint8_t* const rawst = yst + (size_t)S * y_bytes;
        const size_t raw_b = (size_t)kpm * (NB / 8) * VB;
        const int lag = a.raw_slots > 1 ? 1 : 0;
        auto convert_codes = [&](const Unit& w, int i_unit) {
            const int slot = i_unit % S;
            if (w.ok) {
                const int kpad = (w.r + 15) & ~15;
                const uint8_t* raw = rawst + (size_t)(i_unit % a.raw_slots) * raw_b;
                uint8_t* bs = bst + (size_t)slot * b_bytes;
#pragma unroll
                for (int gi = 0; gi < kGr; ++gi) {
                    const int g = pt + gi * kExpandProducers;
                    if (g >= kpad * (NB / 8)) break;
                    const int jg = g % (NB / 8), k = g / (NB / 8);
                    typename Codes8<WF>::T cv{};
                    if (k < w.r) cv = *reinterpret_cast<const typename Codes8<WF>::T*>(raw + (size_t)g * VB);
                    *reinterpret_cast<uint4*>(bs + (uint32_t)(k >> 3) * sbo_b + (uint32_t)(jg >> 3) * 1024 +
                                              sw128_off((uint32_t)k, (uint32_t)jg)) = codes8_to_bf16<WF>(cv);
                }
            }
            fence_proxy_async_smem();  // the converted codes, to the async proxy; then the second arrival
            mbar_arrive(&full_bar[slot]);
        };
        for (int u = u0; u < u1; ++u) {
            const int i = u - u0, st = i % S;
            const Unit w = unit(u);
            const int t = t_next, t0 = t0_next;
            const int32_t pg0 = pg_next[0], pg1 = pg_next[1];
            if (u + 1 < u1) fetch(unit(u + 1), t_next, t0_next, pg_next);
            if (i >= S) wait(&yfree_bar[st], (uint32_t)((i / S - 1) & 1));
            if (w.ok) {
                if (pt < w.r * npc) pid_s[st][pt] = pg0;
                if (pt + kExpandProducers < w.r * npc) pid_s[st][pt + kExpandProducers] = pg1;
                tok_s[st][pt] = t;
                // page ids and token rows in shared memory; are the rows consecutive tokens?
                const bool contig = named_bar_and(1, kExpandProducers, pt >= w.rows || (t == t0 + pt && t0 >= 0));
                uint8_t* ys = yst + (size_t)st * y_bytes;
                if (contig && a.use_tma) {
                    if (pt == 0) {  // two boxes of 128 rows (rows past the tile: other tokens or zero fill)
                        mbar_expect_tx(&full_bar[st], (uint32_t)y_bytes);
                        tma_load_2d(ys, &tmap_y, w.j0, t0, &full_bar[st]);
                        tma_load_2d(ys + kYHalf, &tmap_y, w.j0 + NB / 2, t0, &full_bar[st]);
                    }
                } else {
                    // 16 threads per row; each 8-lane quarter copies 128 contiguous bytes
#pragma unroll
                    for (int k16 = 0; k16 < kTcTileRows * (kYRowBytes / 16) / kExpandProducers; ++k16) {
                        const int g = pt + k16 * kExpandProducers;
                        const int m = g >> 4, q16 = g & 15;
                        const int tm = tok_s[st][m];
                        if (tm >= 0)
                            cp_async16(ys + (q16 >> 3) * kYHalf + m * 128 +
                                           (((uint32_t)(q16 & 7) ^ (uint32_t)(m & 7)) << 4),
                                       ybase + ((int64_t)tm * a.ldy + w.j0) * esz + q16 * 16, true);
                    }
                }
                // B^T block: granule (k, jg) = B^T[k][j0 + 8 jg .. +8], zero past r
                const int kpad = (w.r + 15) & ~15;
                if constexpr (WF == kFmtBf16) {
                    uint8_t* bs = bst + (size_t)st * b_bytes;
#pragma unroll
                    for (int gi = 0; gi < kGr; ++gi) {
                        const int g = pt + gi * kExpandProducers;
                        if (g >= kpad * (NB / 8)) break;
                        const int jg = g % (NB / 8), k = g / (NB / 8);
                        const int j = w.j0 + jg * 8;
                        const uint32_t off = (uint32_t)(k >> 3) * sbo_b + (uint32_t)(jg >> 3) * 1024 +
                                             sw128_off((uint32_t)k, (uint32_t)jg);
                        const bool valid = k < w.r;
                        const uint16_t* src = a.pool.pages;
                        if (valid)
                            src = a.pool.pages + ((int64_t)pid_s[st][k * npc + ((j - w.j0) >> P_log2)] << P_log2) +
                                  (j & ((1 << P_log2) - 1));
                        cp_async16(bs + off, src, valid);
                    }
                } else {
                    const int page_shift = P_log2 + (WF == kFmtFp8 ? 0 : -1);
                    const uint8_t* pages8 = reinterpret_cast<const uint8_t*>(a.pool.pages);
                    uint8_t* raw = rawst + (size_t)(i % a.raw_slots) * raw_b;
#pragma unroll
                    for (int gi = 0; gi < kGr; ++gi) {
                        const int g = pt + gi * kExpandProducers;
                        if (g >= kpad * (NB / 8)) break;
                        const int jg = g % (NB / 8), k = g / (NB / 8);
                        const int j = w.j0 + jg * 8;
                        if (k < w.r)
                            cp_async_n<VB>(raw + (size_t)g * VB,
                                           pages8 + ((int64_t)pid_s[st][k * npc + ((j - w.j0) >> P_log2)] << page_shift) +
                                               ((j & ((1 << P_log2) - 1)) / 8) * VB);
                    }
                }
            } else if (pt == 0) {
                atomicOr(&g_err_tc, kErrRows);
            }
            cp_async_commit();
            cp_async_mbar_arrive_noinc(&full_bar[st]);
            // V after the unit's copies: with a programmatic launch, the first unit's y and
            // B^T copies go out before the wait for the shrink
            if constexpr (WF == kFmtBf16) v_split(w);
            if constexpr (WF != kFmtBf16) {
                // the codes of unit i - lag (its commit group) have landed: convert them; then
                // the V split, which may wait for the MMAs of that unit
                if (lag) {
                    if (i >= 1) {
                        cp_async_wait<1>();
                        convert_codes(unit(u - 1), i - 1);
                    }
                } else {
                    cp_async_wait<0>();
                    convert_codes(w, i);
                }
                v_split(w);
            }
        }
        if constexpr (WF != kFmtBf16) {
            if (lag && u1 > u0) {
                cp_async_wait<0>();
                convert_codes(unit(u1 - 1), u1 - 1 - u0);
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if ((tid & 31) == 0) {
            const uint32_t idesc = idesc_bf16_f32(128, NB, false, true);
            const uint32_t ah = smem_u32(vhi), al = smem_u32(vlo);
            int ts = -1, cur_tile = -1;
            for (int u = u0; u < u1; ++u) {
                const int i = u - u0, st = i % S, bsel = i & 1;
                const Unit w = unit(u);
                if (w.ok && w.tile != cur_tile) {
                    ++ts;
                    cur_tile = w.tile;
                    wait(&vfull_bar, (uint32_t)(ts & 1));
                }
                if (i >= 2) wait(&acce_bar[bsel], (uint32_t)((i / 2 - 1) & 1));
                wait(&full_bar[st], (uint32_t)((i / S) & 1));
                fence_proxy_async_smem();  // the B^T copies were made through the generic proxy
                tc_fence_after();
                if (w.ok) {
                    const int kpad = (w.r + 15) & ~15;
                    const uint32_t acc = tmem + (uint32_t)(bsel * NB);
                    const uint32_t bb = smem_u32(bst + (size_t)st * b_bytes);
                    // K step ks: V at block ks / 4, 32 bytes per step inside its rows; B^T two K groups on
                    for (int ks = 0; ks < kpad / 16; ++ks)
                        tc_mma_bf16(acc, smem_desc_sw128(ah + (ks >> 2) * (kTcTileRows * 128) + (ks & 3) * 32, 16, 1024),
                                    smem_desc_sw128(bb + ks * 2 * sbo_b, 1024, sbo_b), idesc, ks > 0);
                    for (int ks = 0; ks < kpad / 16; ++ks)
                        tc_mma_bf16(acc, smem_desc_sw128(al + (ks >> 2) * (kTcTileRows * 128) + (ks & 3) * 32, 16, 1024),
                                    smem_desc_sw128(bb + ks * 2 * sbo_b, 1024, sbo_b), idesc, true);
                    if constexpr (YM) {  // acc += Y I: the y block (two 64-column halves) as the A operand
                        const uint32_t yb = smem_u32(yst + (size_t)st * y_bytes), ib = smem_u32(ident);
                        for (int ks = 0; ks < NB / 16; ++ks)
                            tc_mma_bf16(acc, smem_desc_sw128(yb + (ks >> 2) * kYHalf + (ks & 3) * 32, 16, 1024),
                                        smem_desc_sw128(ib + ks * 2 * sbo_b, 1024, sbo_b), idesc, true);
                    }
                }
                tc_commit(&accf_bar[bsel]);
                if (w.ok && (u + 1 == u1 || (u + 1) / a.n_blocks != w.tile))
                    tc_commit(&vempty_bar);  // last MMA of the tile: V may be rewritten once it completes
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        // Two warp groups take turns: group g (warps 4g .. 4g+3) handles the units
        // i with i % 2 == g, whose accumulator is acc[g], over whole rows.
        const int grp = warp >> 2;
        const int m = (warp & 3) * 32 + (tid & 31);  // tile row (tensor-memory lane)
        const int gt = tid & 127;                     // thread within the group
        for (int u = u0 + grp; u < u1; u += 2) {
            const int i = u - u0, st = i % S, bsel = i & 1;
            const Unit w = unit(u);
            // the row's token and the tile's first token are loaded before the waits, so their
            // latency is spent waiting for the accumulator rather than after it
            int t = -1;  // (the producer flags a bad token and leaves the row alone)
            if (w.ok && m < w.rows) {
                t = a.b.token_idx[w.row_begin + m];
                if (t >= a.b.T) t = -1;
            }
            const int t0 = w.ok ? a.b.token_idx[w.row_begin] : -1;
            wait(&accf_bar[bsel], (uint32_t)((i / 2) & 1));
            wait(&full_bar[st], (uint32_t)((i / S) & 1));  // (completed: makes the staged y visible here)
            tc_fence_after();
            uint8_t* ys = yst + (size_t)st * y_bytes;
            const bool row_ok = t >= 0 && !abort_flag;
            const float sc = a.scale * w.sc;  // the call's scale times the adapter's
            for (int c00 = 0; c00 < NB; c00 += 64) {
                uint32_t rr[2][32];  // two loads in flight per wait
                const uint32_t ta = tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(bsel * NB + c00);
                tmem_ld_32x32b_x32(ta, rr[0]);
                tmem_ld_32x32b_x32(ta + 32, rr[1]);
                tmem_ld_wait();
                if (!row_ok) continue;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int c0 = c00 + 32 * h;                 // column within the block
                    const int hf = c0 / (NB / 2), cc = c0 % (NB / 2);  // half, column within it
                    uint8_t* yrow = ys + (size_t)hf * kYHalf + (size_t)m * 128;  // swizzled row
                    const uint32_t (&regs)[32] = rr[h];
                    if (YM) {  // the accumulator already holds y + scale V B^T
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            uint32_t wv[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                wv[e] = pack_bf16x2(__uint_as_float(regs[q4 * 8 + 2 * e]),
                                                    __uint_as_float(regs[q4 * 8 + 2 * e + 1]));
                            *reinterpret_cast<uint4*>(yrow + ((((cc >> 3) + q4) ^ (m & 7)) << 4)) =
                                make_uint4(wv[0], wv[1], wv[2], wv[3]);
                        }
                    } else if (ESZ == 2) {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            uint4* yp = reinterpret_cast<uint4*>(yrow + ((((cc >> 3) + q4) ^ (m & 7)) << 4));
                            float yf[8];
                            unpack8(*yp, yf);
                            uint32_t wv[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float lo = fmaf(sc, __uint_as_float(regs[q4 * 8 + 2 * e]), yf[2 * e]);
                                const float hi = fmaf(sc, __uint_as_float(regs[q4 * 8 + 2 * e + 1]), yf[2 * e + 1]);
                                wv[e] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
                                        ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
                            }
                            *yp = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                        }
                    } else {
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4) {
                            float4* yp = reinterpret_cast<float4*>(yrow + ((((cc >> 2) + q4) ^ (m & 7)) << 4));
                            float4 yv = *yp;
                            yv.x = fmaf(sc, __uint_as_float(regs[q4 * 4 + 0]), yv.x);
                            yv.y = fmaf(sc, __uint_as_float(regs[q4 * 4 + 1]), yv.y);
                            yv.z = fmaf(sc, __uint_as_float(regs[q4 * 4 + 2]), yv.z);
                            yv.w = fmaf(sc, __uint_as_float(regs[q4 * 4 + 3]), yv.w);
                            *yp = yv;
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&acce_bar[bsel]);  // acc[bsel] has been read out
            tok_row[grp][m] = t;
            // a full tile of consecutive tokens goes back by TMA (a partial one must not
            // touch the rows past it)
            const bool full = named_bar_and(2 + grp, kTcTileRows, w.ok && w.rows == kTcTileRows && t0 >= 0 &&
                                                                      t == t0 + m && !abort_flag);
            if (full && a.use_tma) {
                fence_proxy_async_smem();  // this thread's row, to the async proxy
                named_bar_sync(2 + grp, kTcTileRows);
                if (gt == 0) {
                    tma_store_2d(&tmap_y, w.j0, t0, ys);
                    tma_store_2d(&tmap_y, w.j0 + NB / 2, t0, ys + kYHalf);
                    bulk_commit();
                    bulk_wait_read_all();  // the block has been read: slot st may be refilled
                }
            } else if (w.ok && !abort_flag) {
                // coalesced 16-byte stores: 16 threads per row, two rows per warp instruction
#pragma unroll
                for (int k16 = 0; k16 < kTcTileRows * (kYRowBytes / 16) / kTcTileRows; ++k16) {
                    const int mm = (gt >> 4) + k16 * (kTcTileRows / 16), q16 = gt & 15;
                    const int tt = tok_row[grp][mm];
                    if (tt >= 0)
                        *reinterpret_cast<uint4*>(ybase + ((int64_t)tt * a.ldy + w.j0) * esz + q16 * 16) =
                            *reinterpret_cast<const uint4*>(ys + (q16 >> 3) * kYHalf + mm * 128 +
                                                             (((uint32_t)(q16 & 7) ^ (uint32_t)(mm & 7)) << 4));
                }
            }
            named_bar_sync(2 + grp, kTcTileRows);  // tok_row may be rewritten
            mbar_arrive(&yfree_bar[st]);  // slot st may be refilled
        }
        if (gt == 0) bulk_wait_all();  // the TMA stores have reached global memory
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, (uint32_t)(2 * NB));
    }
}

// 2-D tensor map over a row-major matrix (rows x cols elements, row stride in
// bytes), box of box_rows x box_cols with the 128-byte swizzle.  False if the
// encoder is unavailable or rejects the layout (the kernels then gather).
bool encode_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t cols, uint64_t rows,
               uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows) {
    static std::mutex mu;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static bool tried = false;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!tried) {
            tried = true;
            cudaDriverEntryPointQueryResult q;
            void* f = nullptr;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
                q == cudaDriverEntryPointSuccess)
                fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
            cudaGetLastError();
        }
    }
    if (!fn || rows == 0 || (reinterpret_cast<uintptr_t>(base) & 15) || (row_stride_bytes & 15)) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t es[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int pow2_at_least(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

}  // namespace

cudaError_t launch_shrink_tc(const uint16_t* x, int64_t ldx, int32_t d_in, const BatchView& b, int32_t num_tiles,
                             int32_t max_rank, const PoolView& pool, float* v, int64_t ldv, cudaStream_t stream) {
    if (num_tiles <= 0) return cudaSuccess;
    ShrinkTcArgs a;
    a.x = x;
    a.ldx = ldx;
    a.d_in = d_in;
    a.b = b;
    a.pool = pool;
    a.v = v;
    a.ldv = ldv;
    a.npad_max = std::max(16, (max_rank + 15) & ~15);
    a.tmem_cols = std::max(32, pow2_at_least(a.npad_max));
    // split d_in so that the launch has about two CTAs per SM
    const int ktiles = d_in / kKTile;
    int ks = 1;
    for (int c = 8; c >= 1; --c)
        if (ktiles % c == 0 && (int64_t)num_tiles * c <= 2 * 148) {
            ks = c;
            break;
        }
    a.ks = ks;
    a.kcols = d_in / ks;
    const size_t stage_bytes = (size_t)kTcTileRows * kKTile * 2 + (size_t)a.npad_max * kKTile * 2;
    const size_t main_bytes = std::max(stage_bytes * kShrinkStages, (size_t)kTcTileRows * (a.npad_max + 4) * 4);
    const size_t span_pages = ((size_t)a.kcols >> pool.page_log2) + 2;  // pages one K range can touch
    // quantised pools: a ring of kShrinkCodeSlots slots of A codes (npad_max rows x 64 values)
    const size_t raw_bytes = pool.wfmt == kFmtBf16 ? 0  // 1 byte (E4M3) or half a byte (INT4) a value
                             : (size_t)kShrinkCodeSlots * a.npad_max * kKTile / (pool.wfmt == kFmtFp8 ? 1 : 2);
    a.raw_offset = (int)main_bytes;
    a.pid_offset = (int)(main_bytes + raw_bytes);
    const size_t pid_bytes = ((size_t)a.npad_max * span_pages * 4 + 15) & ~(size_t)15;
    // >= 80 KB: at most two CTAs per SM, so tensor memory is never oversubscribed
    const size_t smem = std::max(main_bytes + raw_bytes + pid_bytes, (size_t)80 << 10) + 1024;
    if (smem > (227u << 10)) return cudaErrorInvalidValue;
    auto kern = pool.wfmt == kFmtFp8 ? shrink_tc_kernel<kFmtFp8>
                : pool.wfmt == kFmtInt4 ? shrink_tc_kernel<kFmtInt4> : shrink_tc_kernel<kFmtBf16>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(ks * num_tiles), 1, 1);
    cfg.blockDim = dim3(kShrinkThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)ks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    CUtensorMap tmap_x;
    std::memset(&tmap_x, 0, sizeof(tmap_x));
    a.use_tma = encode_2d(&tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)d_in, (uint64_t)b.T,
                          (uint64_t)ldx * 2, kKTile, kTcTileRows) ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, a, tmap_x);
}

cudaError_t launch_expand_tc(const float* v, int64_t ldv, int32_t d_out, const BatchView& b, int32_t num_tiles,
                             int32_t max_rank, const PoolView& pool, float scale, void* y, int64_t ldy,
                             int32_t y_dtype, bool after_shrink, cudaStream_t stream) {
    if (num_tiles <= 0) return cudaSuccess;
    ExpandTcArgs a;
    a.v = v;
    a.ldv = ldv;
    a.d_out = d_out;
    a.b = b;
    a.pool = pool;
    a.scale = scale;
    a.y = y;
    a.ldy = ldy;
    a.y_dtype = y_dtype;
    a.kpad_max = std::max(16, (max_rank + 15) & ~15);
    const int NB = kYRowBytes / (y_dtype == 0 ? 2 : 4);
    if (d_out % NB) return cudaErrorInvalidValue;  // d_out is a multiple of the page size (>= 512)
    a.n_blocks = d_out / NB;
    a.num_units = a.n_blocks * num_tiles;
    // shared memory: V hi + lo, S stages of (B^T block, Y block); three stages when they fit
    const size_t v_bytes = (size_t)2 * kTcTileRows * ((a.kpad_max + 63) & ~63) * 2;
    // a stage: B^T block (bf16) and y block; a quantised pool adds 1 or 2 slots of B^T codes
    // (1 or 1/2 byte a value)
    const size_t raw_slot = pool.wfmt == kFmtBf16 ? 0 : (size_t)a.kpad_max * NB / (pool.wfmt == kFmtFp8 ? 1 : 2);
    const size_t stage = (size_t)a.kpad_max * NB * 2 + (size_t)kTcTileRows * kYRowBytes;
    // the opt-in limit covers dynamic (+1 KB alignment) and static shared memory (index tables,
    // barriers, row scales: 6.1 KB with three stages, rounded up)
    const size_t limit = (227u << 10) - 1024 - 6656;
    // stages S and code slots R (quantised pools): three stages when they fit, two code slots
    // when they fit (one otherwise)
    // bf16 y: the identity of the Y I products (32 KB, 1 KB aligned) when it fits, with three
    // stages before two
    const size_t ident_bytes = (size_t)NB * NB * 2 + 1024;
    int S = 2, R = raw_slot ? 1 : 0;
    bool ym = false;
    const int cand[6][3] = {{3, 2, 1}, {2, 2, 1}, {2, 1, 1}, {3, 2, 0}, {2, 2, 0}, {2, 1, 0}};
    for (const auto& c : cand) {
        const int r = raw_slot ? c[1] : 0;
        const bool with_ident = c[2] != 0;
        if (with_ident && y_dtype != 0) continue;
        if (v_bytes + c[0] * stage + r * raw_slot + (with_ident ? ident_bytes : 0) <= limit) {
            S = c[0];
            R = r;
            ym = with_ident;
            break;
        }
    }
    a.raw_slots = std::max(R, 1);
    // at least 116 KB: one CTA per SM, so tensor memory (2 x NB <= 256 columns) is never oversubscribed
    const size_t smem =
        std::max(v_bytes + S * stage + R * raw_slot + (ym ? ident_bytes : 0), (size_t)116 << 10) + 1024;
    if (smem > (227u << 10)) return cudaErrorInvalidValue;
    // one CTA per SM, each a contiguous run of units
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    const int grid = std::min(a.num_units, sms);
    a.units_per_cta = (a.num_units + grid - 1) / grid;
    const int blocks = (a.num_units + a.units_per_cta - 1) / a.units_per_cta;
    CUtensorMap tmap_y;
    std::memset(&tmap_y, 0, sizeof(tmap_y));
    const int esz = y_dtype == 0 ? 2 : 4;
    a.use_tma = encode_2d(&tmap_y, y_dtype == 0 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, y,
                          (uint64_t)d_out, (uint64_t)b.T, (uint64_t)ldy * esz, (uint32_t)(NB / 2), kTcTileRows) ? 1 : 0;
    auto pick = [&](auto wf) {
        constexpr int WF = decltype(wf)::value;
        if (ym) return S == 3 ? expand_tc_kernel<3, 2, WF, true> : expand_tc_kernel<2, 2, WF, true>;
        return S == 3 ? (esz == 2 ? expand_tc_kernel<3, 2, WF, false> : expand_tc_kernel<3, 4, WF, false>)
                      : (esz == 2 ? expand_tc_kernel<2, 2, WF, false> : expand_tc_kernel<2, 4, WF, false>);
    };
    auto kern = pool.wfmt == kFmtFp8    ? pick(std::integral_constant<int, kFmtFp8>{})
                : pool.wfmt == kFmtInt4 ? pick(std::integral_constant<int, kFmtInt4>{})
                                        : pick(std::integral_constant<int, kFmtBf16>{});
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks, 1, 1);
    cfg.blockDim = dim3(kExpandThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after_shrink ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, a, tmap_y);
}

cudaError_t read_clear_errors_tc(uint32_t* bits, cudaStream_t stream) {
    unsigned int h = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&h, g_err_tc, sizeof(h), 0, cudaMemcpyDeviceToHost, stream);
    if (e != cudaSuccess) return e;
    e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbolAsync(g_err_tc, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return e;
    e = cudaStreamSynchronize(stream);
    *bits |= h;
    return e;
}

}  // namespace sgmv
