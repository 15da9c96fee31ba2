// Tensor-core (tcgen05) path of SGMV-shrink and SGMV-expand for long
// segments (prefill): "for large segments (several requests with the same
// adapter) it goes through tensor cores" -- "Multi-LoRA serving: the single
// translator with a thousand glossaries ..." (blog.lo0.es), section "SGMV: the
// kernel that holds it all up".  A long segment is a real dense contraction:
//
//   shrink  V[128 rows, r]     = X[128 rows, d_in] * A^T          (M=128, N=r padded to 16)
//   expand  Y[128 rows, 128 j] += scale * V[128 rows, r] * B^T    (M=128, N=128, K=r padded to 16)
//
// Operands are staged in shared memory in the canonical no-swizzle layout
// (8 rows x 16 bytes core matrices) with 16-byte cp.async copies -- x rows are
// gathered through the segment's token list and A / B^T chunks through the
// page table -- and multiplied by one thread issuing tcgen05.mma (bf16 inputs,
// fp32 accumulator in tensor memory).  The epilogue reads the accumulator with
// tcgen05.ld.
//
// shrink: a cluster of KS CTAs splits d_in; each accumulates its K range in
// tensor memory, and the KS partial tiles are summed in a fixed order through
// distributed shared memory into v.
// expand: v (fp32) is split into bf16 hi + lo parts so that the delta keeps
// ~16 bits of v: D = V_hi B + V_lo B, both products exact, fp32 accumulation.
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace sgmv {
namespace {

__device__ unsigned int g_err_tc;

constexpr int kThreads = 128;
constexpr int kKTile = 64;          // K columns per pipeline stage (shrink)
constexpr int kShrinkStages = 4;

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
};

__device__ __forceinline__ int32_t safe_page(const PoolView& pool, int64_t entry) {
    int32_t page = (entry >= 0 && entry < pool.pt_capacity) ? pool.page_table[entry] : -1;
    if (page < 0 || page >= pool.num_pages) {
        atomicOr(&g_err_tc, kErrPage);
        page = 0;
    }
    return page;
}

// ------------------------------------------------------------------ shrink
__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    const uint32_t s = smem_u32(p);
    return p + ((1024u - (s & 1023u)) & 1023u);
}

__global__ void __launch_bounds__(kThreads) shrink_tc_kernel(const ShrinkTcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    __shared__ uint64_t mma_bar[kShrinkStages];
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;
    __shared__ int32_t tok_s[kTcTileRows];

    const int tid = threadIdx.x, warp = tid >> 5;
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
        for (int i = 0; i < kShrinkStages; ++i) mbar_init(&mma_bar[i], 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_slot, (uint32_t)a.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    const int P_log2 = a.pool.page_log2;
    const int pages_per_row = a.d_in >> P_log2;
    const int k_begin = (int)q * a.kcols;
    const int nk = a.kcols / kKTile;

    // token of each tile row (-1: none), read once
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
    __syncthreads();

    // page ids of the A rows over this CTA's K range, [rank row][page], one round
    // (the range may start and end inside a page)
    const int first_page = k_begin >> P_log2;
    const int span_pages = ((k_begin + a.kcols - 1) >> P_log2) - first_page + 1;
    int32_t* pid_s = reinterpret_cast<int32_t*>(smem + a.pid_offset);
    for (int e = tid; e < r * span_pages; e += kThreads) {
        const int n = e / span_pages, pc = e - n * span_pages;
        pid_s[e] = safe_page(a.pool, a_base + (int64_t)n * pages_per_row + first_page + pc);
    }
    __syncthreads();

    // Granule g of a tile (16 bytes): row (g & 7) + 8 (g >> 6), K granule (g >> 3) & 7.
    // A warp reads 8 rows x 64 contiguous bytes; each 8-lane phase writes one
    // contiguous 128-byte line of a core-matrix column (no bank conflicts).
    auto load_tile = [&](int kt, int slot) {
        uint8_t* xs = stage0 + (size_t)slot * stage_bytes;
        uint8_t* as = xs + x_tile_bytes;
        const int c = k_begin + kt * kKTile;
#pragma unroll
        for (int i = 0; i < (kTcTileRows * 8) / kThreads; ++i) {
            const int g = tid + i * kThreads;
            const int row = (g & 7) + 8 * (g >> 6), kg = (g >> 3) & 7;
            const int t = tok_s[row];
            const uint32_t off = (uint32_t)(row >> 3) * 1024 + kg * 128 + (row & 7) * 16;
            const uint16_t* src = t >= 0 ? a.x + (int64_t)t * a.ldx + c + kg * 8 : a.x;
            cp_async16(xs + off, src, t >= 0);
        }
        // A: rank rows n < npad, zero past r; the 64 columns lie in one page
        const int page_rel = (c >> P_log2) - first_page, in_page = c & ((1 << P_log2) - 1);
        for (int g = tid; g < npad * 8; g += kThreads) {
            const int n = (g & 7) + 8 * (g >> 6), kg = (g >> 3) & 7;
            const uint32_t off = (uint32_t)(n >> 3) * 1024 + kg * 128 + (n & 7) * 16;
            const bool valid = ok && n < r;
            const uint16_t* src = a.pool.pages;
            if (valid) src = a.pool.pages + ((int64_t)pid_s[n * span_pages + page_rel] << P_log2) + in_page + kg * 8;
            cp_async16(as + off, src, valid);
        }
    };

    const uint32_t idesc = idesc_bf16_f32(128, npad, false, false);
#pragma unroll 1
    for (int s = 0; s < kShrinkStages - 1; ++s) {
        if (s < nk) load_tile(s, s);
        cp_async_commit();
    }
#pragma unroll 1
    for (int kt = 0; kt < nk; ++kt) {
        const int nxt = kt + kShrinkStages - 1;
        if (nxt < nk) {
            if (kt >= 1) {  // the slot of tile kt-1 is free once its MMAs completed
                const int ps = (kt - 1) % kShrinkStages;
                if (!mbar_wait(&mma_bar[ps], (uint32_t)(((kt - 1) / kShrinkStages) & 1), &g_err_tc))
                    abort_flag = 1;
            }
            load_tile(nxt, nxt % kShrinkStages);
        }
        cp_async_commit();
        cp_async_wait<kShrinkStages - 1>();
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const int slot = kt % kShrinkStages;
            const uint32_t xs = smem_u32(stage0 + (size_t)slot * stage_bytes);
            const uint32_t as = xs + (uint32_t)x_tile_bytes;
#pragma unroll
            for (int ks = 0; ks < kKTile / 16; ++ks) {
                const uint64_t ad = smem_desc_noswizzle(xs + ks * 256, 128, 1024);
                const uint64_t bd = smem_desc_noswizzle(as + ks * 256, 128, 1024);
                tc_mma_bf16(tmem, ad, bd, idesc, kt > 0 || ks > 0);
            }
            tc_commit(&mma_bar[slot]);
        }
    }
    // accumulator complete once the last commit arrives
    if (nk > 0) {
        const int ls = (nk - 1) % kShrinkStages;
        if (!mbar_wait(&mma_bar[ls], (uint32_t)(((nk - 1) / kShrinkStages) & 1), &g_err_tc)) abort_flag = 1;
    }
    tc_fence_after();
    cp_async_wait<0>();
    __syncthreads();

    // tensor memory -> shared memory partial tile red[128][npad_max] (reuses the stages)
    float* red = reinterpret_cast<float*>(smem);
    const int RS = a.npad_max;
    const int m = warp * 32 + (tid & 31);
    for (int c0 = 0; c0 < npad; c0 += 32) {
        uint32_t regs[32];
        tmem_ld_32x32b_x32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, regs);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e)
            if (c0 + e < RS) red[m * RS + c0 + e] = __uint_as_float(nk > 0 ? regs[e] : 0u);
    }
    tc_fence_before();
    cluster_sync();

    if (ok && !abort_flag) {
        const int KS = a.ks;
        const int m0 = (int)((kTcTileRows * q) / KS), m1 = (int)((kTcTileRows * (q + 1)) / KS);
        const uint32_t red_s = smem_u32(red);
        for (int e = tid; e < (m1 - m0) * r; e += kThreads) {
            const int mm = m0 + e / r, k = e % r;
            if (mm >= rows) continue;
            float pv[8];
#pragma unroll
            for (int qq = 0; qq < 8; ++qq)  // all loads in flight before the fixed-order sum
                pv[qq] = qq < KS ? ld_cluster_f32(map_cluster(red_s + 4u * (uint32_t)(mm * RS + k), (uint32_t)qq)) : 0.f;
            float s = 0.f;
#pragma unroll
            for (int qq = 0; qq < 8; ++qq) s += pv[qq];
            a.v[(int64_t)(it.row_begin + mm) * a.ldv + k] = s;
        }
    }
    cluster_sync();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, (uint32_t)a.tmem_cols);
    }
}

// ------------------------------------------------------------------ expand
// Persistent: CTA b takes a contiguous run of units (tile of <= 128 rows, block
// of kYRowBytes of y columns), so consecutive units mostly share the tile and
// its v rows.  The y rows and the B^T block of the next S-1 units are in flight
// (cp.async) while the current unit is multiplied and written back:
//   V_hi/V_lo [128 x kpad] (K-major)  <- v rows of the tile, split once per tile
//   B^T block [kpad x NB]  (MN-major) <- page table
//   Y block   [128 x NB]   (row stride kYStride: 16-byte accesses conflict-free)
//   TMEM acc  [128 lanes x NB fp32]   <- V_hi B + V_lo B (tcgen05.mma, one thread)
// The epilogue adds scale * acc to the Y block in shared memory (one row per
// thread) and the block is stored with coalesced 16-byte stores.
constexpr int kYRowBytes = 256;             // y bytes of one tile row per unit (128 bf16 / 64 fp32)
constexpr int kMaxPagesPerUnit = 2;         // pages of one B^T row a unit spans (page_elems >= 64)
constexpr int kYStride = kYRowBytes + 16;   // padded shared-memory row stride

template <int S>
__global__ void __launch_bounds__(kThreads, 1) expand_tc_kernel(const ExpandTcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    __shared__ uint64_t mma_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ int32_t tok_s[S][kTcTileRows];
    __shared__ int32_t pid_s[S][kMaxRank * kMaxPagesPerUnit];  // B^T page ids of a unit [rank row][page]

    const int tid = threadIdx.x, warp = tid >> 5;
    const int u0 = blockIdx.x * a.units_per_cta, u1 = min(u0 + a.units_per_cta, a.num_units);
    if (u0 >= u1) return;  // uniform, before anything is allocated
    const int esz = a.y_dtype == 0 ? 2 : 4;
    const int NB = kYRowBytes / esz;              // output columns per unit
    const int kpm = a.kpad_max;
    const uint32_t sbo = (uint32_t)(kpm / 8) * 128;  // 8-row (A) / 8-column (B) group stride
    uint8_t* vhi = smem;
    uint8_t* vlo = vhi + (size_t)kTcTileRows * kpm * 2;
    uint8_t* bst = vlo + (size_t)kTcTileRows * kpm * 2;          // [S][kpm x NB]
    const size_t b_bytes = (size_t)kpm * NB * 2;
    uint8_t* yst = bst + (size_t)S * b_bytes;                      // [S][128 x kYStride]
    const size_t y_bytes = (size_t)kTcTileRows * kYStride;

    if (tid == 0) {
        mbar_init(&mma_bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_slot, (uint32_t)NB);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    const int P_log2 = a.pool.page_log2;
    const int pages_per_row = a.d_out >> P_log2;
    uint8_t* const ybase = static_cast<uint8_t*>(a.y);

    // tile record of unit u; ok is uniform across the CTA
    struct Unit {
        int row_begin, rows, r, j0;
        int64_t b_base;
        bool ok;
    };
    auto unit = [&](int u) {
        Unit w;
        const int tile = u / a.n_blocks;
        w.j0 = (u - tile * a.n_blocks) * NB;
        const ItemRec it = a.b.tc_tiles[(int64_t)tile * a.b.n_proj + a.b.proj];
        w.row_begin = it.row_begin;
        w.rows = it.row_end - it.row_begin;
        w.r = it.rank;
        w.b_base = it.b_pt;
        w.ok = !(it.seg < 0 || it.seg >= a.b.num_segments || it.row_begin < 0 || w.rows <= 0 ||
                 w.rows > kTcTileRows || it.row_end > a.b.num_rows || w.r <= 0 || ((w.r + 15) & ~15) > kpm);
        return w;
    };

    // Issue the copies of unit u into stage slot `slot` (one commit group).
    // All threads call it.  First every index the copies need (token rows, B^T
    // page ids) is fetched into shared memory in one round of independent loads,
    // then the copies are issued from there.
    auto issue = [&](int u, int slot) {
        const Unit w = unit(u);
        const int kpad = (w.r + 15) & ~15;
        const int npc = NB > (1 << P_log2) ? (NB >> P_log2) : 1;  // pages a B^T row spans in one unit
        if (w.ok) {
            if (tid < kTcTileRows) {
                int t = -1;
                if (tid < w.rows) {
                    t = a.b.token_idx[w.row_begin + tid];
                    if (t < 0 || t >= a.b.T) {
                        atomicOr(&g_err_tc, kErrToken);
                        t = -1;
                    }
                }
                tok_s[slot][tid] = t;
            }
            for (int e = tid; e < w.r * npc; e += kThreads) {
                const int k = e / npc, pc = e - k * npc;
                pid_s[slot][e] = safe_page(a.pool, w.b_base + (int64_t)k * pages_per_row + (w.j0 >> P_log2) + pc);
            }
        } else if (tid == 0) {
            atomicOr(&g_err_tc, kErrRows);
        }
        __syncthreads();
        if (w.ok) {
            uint8_t* ys = yst + (size_t)slot * y_bytes;
            // y rows: 16 threads per row, 16 bytes each
#pragma unroll 4
            for (int i = 0; i < kTcTileRows * (kYRowBytes / 16) / kThreads; ++i) {
                const int g = tid + i * kThreads;
                const int m = g >> 4, q16 = g & 15;
                const int t = tok_s[slot][m];
                if (t >= 0)
                    cp_async16(ys + m * kYStride + q16 * 16,
                               ybase + ((int64_t)t * a.ldy + w.j0) * esz + q16 * 16, true);
            }
            // B^T block: granule (k, jg) = B^T[k][j0 + 8 jg .. +8], zero past r
            uint8_t* bs = bst + (size_t)slot * b_bytes;
            for (int g = tid; g < kpad * (NB / 8); g += kThreads) {
                const int jg = g % (NB / 8), k = g / (NB / 8);
                const int j = w.j0 + jg * 8;
                const uint32_t off = (uint32_t)jg * sbo + (uint32_t)(k >> 3) * 128 + (uint32_t)(k & 7) * 16;
                const bool valid = k < w.r;
                const uint16_t* src = a.pool.pages;
                if (valid) {
                    const int32_t page = pid_s[slot][k * npc + ((j - w.j0) >> P_log2)];
                    src = a.pool.pages + ((int64_t)page << P_log2) + (j & ((1 << P_log2) - 1));
                }
                cp_async16(bs + off, src, valid);
            }
        }
        cp_async_commit();
    };

#pragma unroll 1
    for (int i = 0; i < S - 1; ++i) {
        if (u0 + i < u1) issue(u0 + i, i);
        else cp_async_commit();
    }

    int cur_tile = -1;
    uint32_t phase = 0;
    bool alive = true;
#pragma unroll 1
    for (int u = u0; u < u1; ++u) {
        const int i = u - u0, slot = i % S;
        __syncthreads();  // slot (i + S - 1) % S was fully read by the stores of unit i - 1
        if (u + S - 1 < u1) issue(u + S - 1, (i + S - 1) % S);
        else cp_async_commit();
        const Unit w = unit(u);
        const int tile = u / a.n_blocks;
        if (w.ok && tile != cur_tile) {
            // v rows of the tile -> bf16 hi + lo, row m = tid (the previous MMA has completed)
            const int m = tid, kpad = (w.r + 15) & ~15;
            const bool row_ok = m < w.rows;
            const float* vrow = a.v + (int64_t)(w.row_begin + (row_ok ? m : 0)) * a.ldv;
            for (int kg = 0; kg < kpad / 8; ++kg) {
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int k = kg * 8 + e;
                    f[e] = (row_ok && k < w.r) ? vrow[k] : 0.f;
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
                const uint32_t off = (uint32_t)(m >> 3) * sbo + (uint32_t)kg * 128 + (uint32_t)(m & 7) * 16;
                *reinterpret_cast<uint4*>(vhi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4*>(vlo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
            cur_tile = tile;
        }
        if (S == 3) cp_async_wait<2>();
        else cp_async_wait<1>();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (!w.ok || !alive) continue;  // uniform

        const int kpad = (w.r + 15) & ~15;
        if (tid == 0) {
            const uint32_t idesc = idesc_bf16_f32(128, NB, false, true);
            const uint32_t ah = smem_u32(vhi), al = smem_u32(vlo);
            const uint32_t bb = smem_u32(bst + (size_t)slot * b_bytes);
            for (int ks = 0; ks < kpad / 16; ++ks)
                tc_mma_bf16(tmem, smem_desc_noswizzle(ah + ks * 256, 128, sbo),
                            smem_desc_noswizzle(bb + ks * 256, 128, sbo), idesc, ks > 0);
            for (int ks = 0; ks < kpad / 16; ++ks)
                tc_mma_bf16(tmem, smem_desc_noswizzle(al + ks * 256, 128, sbo),
                            smem_desc_noswizzle(bb + ks * 256, 128, sbo), idesc, true);
            tc_commit(&mma_bar);
        }
        const bool done = mbar_wait(&mma_bar, phase, &g_err_tc);
        phase ^= 1u;
        tc_fence_after();

        // epilogue: row m = tid of the Y block += scale * acc, 32 columns per tcgen05.ld
        {
            const int m = tid;
            uint8_t* yrow = yst + (size_t)slot * y_bytes + (size_t)m * kYStride;
            const bool row_ok = m < w.rows && done;
            for (int c0 = 0; c0 < NB; c0 += 32) {
                uint32_t regs[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, regs);
                tmem_ld_wait();
                if (!row_ok) continue;
                if (a.y_dtype == 0) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint4* yp = reinterpret_cast<uint4*>(yrow + (c0 + q4 * 8) * 2);
                        float yf[8];
                        unpack8(*yp, yf);
                        uint32_t wv[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float lo = fmaf(a.scale, __uint_as_float(regs[q4 * 8 + 2 * e]), yf[2 * e]);
                            const float hi = fmaf(a.scale, __uint_as_float(regs[q4 * 8 + 2 * e + 1]), yf[2 * e + 1]);
                            wv[e] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
                                    ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
                        }
                        *yp = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                    }
                } else {
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4) {
                        float4* yp = reinterpret_cast<float4*>(yrow + (c0 + q4 * 4) * 4);
                        float4 yv = *yp;
                        yv.x = fmaf(a.scale, __uint_as_float(regs[q4 * 4 + 0]), yv.x);
                        yv.y = fmaf(a.scale, __uint_as_float(regs[q4 * 4 + 1]), yv.y);
                        yv.z = fmaf(a.scale, __uint_as_float(regs[q4 * 4 + 2]), yv.z);
                        yv.w = fmaf(a.scale, __uint_as_float(regs[q4 * 4 + 3]), yv.w);
                        *yp = yv;
                    }
                }
            }
        }
        tc_fence_before();
        alive = __syncthreads_and(done) != 0;  // uniform: a wait that gave up stops the CTA's work
        if (!alive) continue;
        // coalesced store of the Y block: 16 threads per row
        {
            const uint8_t* ys = yst + (size_t)slot * y_bytes;
            for (int g = tid; g < kTcTileRows * (kYRowBytes / 16); g += kThreads) {
                const int m = g >> 4, q16 = g & 15;
                const int t = tok_s[slot][m];
                if (m < w.rows && t >= 0)
                    *reinterpret_cast<uint4*>(ybase + ((int64_t)t * a.ldy + w.j0) * esz + q16 * 16) =
                        *reinterpret_cast<const uint4*>(ys + m * kYStride + q16 * 16);
            }
        }
    }
    cp_async_wait<0>();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, (uint32_t)NB);
    }
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
    const size_t main_bytes = std::max(stage_bytes * kShrinkStages, (size_t)kTcTileRows * a.npad_max * 4);
    const size_t span_pages = ((size_t)a.kcols >> pool.page_log2) + 2;  // pages one K range can touch
    a.pid_offset = (int)main_bytes;
    const size_t pid_bytes = ((size_t)a.npad_max * span_pages * 4 + 15) & ~(size_t)15;
    // >= 80 KB: at most two CTAs per SM, so tensor memory is never oversubscribed
    const size_t smem = std::max(main_bytes + pid_bytes, (size_t)80 << 10) + 1024;
    if (smem > (227u << 10)) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(shrink_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(ks * num_tiles), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)ks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, shrink_tc_kernel, a);
}

cudaError_t launch_expand_tc(const float* v, int64_t ldv, int32_t d_out, const BatchView& b, int32_t num_tiles,
                             int32_t max_rank, const PoolView& pool, float scale, void* y, int64_t ldy,
                             int32_t y_dtype, cudaStream_t stream) {
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
    const size_t v_bytes = (size_t)2 * kTcTileRows * a.kpad_max * 2;
    const size_t stage = (size_t)a.kpad_max * NB * 2 + (size_t)kTcTileRows * kYStride;
    // the opt-in limit covers dynamic (+1 KB alignment) and static (index tables) shared memory
    const size_t limit = (227u << 10) - 1024 - 3 * kTcTileRows * 4 - 3 * kMaxRank * kMaxPagesPerUnit * 4;
    const int S = (v_bytes + 3 * stage <= limit) ? 3 : 2;
    // at least 116 KB: one CTA per SM, so tensor memory (NB <= 128 columns) is never oversubscribed
    const size_t smem = std::max(v_bytes + S * stage, (size_t)116 << 10) + 1024;
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
    if (S == 3) {
        cudaError_t e = cudaFuncSetAttribute(expand_tc_kernel<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        expand_tc_kernel<3><<<(unsigned)blocks, kThreads, smem, stream>>>(a);
    } else {
        cudaError_t e = cudaFuncSetAttribute(expand_tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        expand_tc_kernel<2><<<(unsigned)blocks, kThreads, smem, stream>>>(a);
    }
    return cudaGetLastError();
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
