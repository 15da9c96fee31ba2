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
constexpr int kExpandN = 128;       // output columns per expand CTA
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
    int32_t n_tiles;     // column tiles of d_out
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

    // this thread's x row (token) for the whole loop
    const uint16_t* xrow = nullptr;
    if (ok && tid < rows) {
        const int t = a.b.token_idx[it.row_begin + tid];
        if (t >= 0 && t < a.b.T) xrow = a.x + (int64_t)t * a.ldx;
        else atomicOr(&g_err_tc, kErrToken);
    }

    auto load_tile = [&](int kt, int slot) {
        uint8_t* xs = stage0 + (size_t)slot * stage_bytes;
        uint8_t* as = xs + x_tile_bytes;
        const int c = k_begin + kt * kKTile;
        // X: row = tid, eight 16-byte granules along K
#pragma unroll
        for (int kg = 0; kg < 8; ++kg) {
            const int off = (tid >> 3) * 1024 + kg * 128 + (tid & 7) * 16;
            const uint16_t* src = xrow ? xrow + c + kg * 8 : a.x;
            cp_async16(xs + off, src, xrow != nullptr);
        }
        // A: rank rows n < npad, zero past r; the 64 columns lie in one page
        const int page_col = c >> P_log2, in_page = c & ((1 << P_log2) - 1);
        for (int g = tid; g < npad * 8; g += kThreads) {
            const int n = g % npad, kg = g / npad;
            const int off = (n >> 3) * 1024 + kg * 128 + (n & 7) * 16;
            const bool valid = ok && n < r;
            const uint16_t* src = a.pool.pages;
            if (valid) {
                const int32_t page = safe_page(a.pool, a_base + (int64_t)n * pages_per_row + page_col);
                src = a.pool.pages + ((int64_t)page << P_log2) + in_page + kg * 8;
            }
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
            float s = 0.f;
            for (int qq = 0; qq < KS; ++qq)
                s += ld_cluster_f32(map_cluster(red_s + 4u * (uint32_t)(mm * RS + k), (uint32_t)qq));
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
__global__ void __launch_bounds__(kThreads) expand_tc_kernel(const ExpandTcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    __shared__ uint64_t mma_bar;
    __shared__ uint32_t tmem_slot;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ntile = blockIdx.x % a.n_tiles, tile_idx = blockIdx.x / a.n_tiles;
    const ItemRec it = a.b.tc_tiles[(int64_t)tile_idx * a.b.n_proj + a.b.proj];
    int rows = it.row_end - it.row_begin, r = 0;
    int64_t b_base = 0;
    bool ok = !(it.seg < 0 || it.seg >= a.b.num_segments || it.row_begin < 0 || rows <= 0 ||
                rows > kTcTileRows || it.row_end > a.b.num_rows);
    if (ok) {
        r = it.rank;
        b_base = it.b_pt;
        ok = r > 0 && ((r + 15) & ~15) <= a.kpad_max;
    }
    if (!ok) {  // uniform across the CTA: nothing is allocated yet
        if (tid == 0) atomicOr(&g_err_tc, kErrRows);
        return;
    }
    const int kpad = (r + 15) & ~15;
    const int j0 = ntile * kExpandN;

    // shared memory: A_hi [128 x kpad] | A_lo [128 x kpad] | B [kExpandN x kpad] (MN-major)
    const int a_bytes = kTcTileRows * kpad * 2;
    uint8_t* ahi = smem;
    uint8_t* alo = smem + a_bytes;
    uint8_t* bs = smem + 2 * a_bytes;
    const uint32_t sbo_a = (uint32_t)(kpad / 8) * 128;   // K-major: 8-row groups
    const uint32_t sbo_b = (uint32_t)(kpad / 8) * 128;   // MN-major: 8-column groups

    if (tid == 0) {
        mbar_init(&mma_bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_slot, kExpandN);
        tmem_relinquish();
    }

    // B^T tile: granule (k, jg) = B^T[k][j0 + 8 jg .. +8], zero past r or d_out
    const int P_log2 = a.pool.page_log2;
    const int pages_per_row = a.d_out >> P_log2;
    for (int g = tid; g < kpad * (kExpandN / 8); g += kThreads) {
        const int k = g % kpad, jg = g / kpad;
        const int j = j0 + jg * 8;
        const uint32_t off = (uint32_t)jg * sbo_b + (uint32_t)(k >> 3) * 128 + (uint32_t)(k & 7) * 16;
        const bool valid = k < r && j < a.d_out;
        const uint16_t* src = a.pool.pages;
        if (valid) {
            const int32_t page = safe_page(a.pool, b_base + (int64_t)k * pages_per_row + (j >> P_log2));
            src = a.pool.pages + ((int64_t)page << P_log2) + (j & ((1 << P_log2) - 1));
        }
        cp_async16(bs + off, src, valid);
    }
    cp_async_commit();

    // A = v split into bf16 hi + lo, row m = tid
    {
        const int m = tid;
        const bool row_ok = m < rows;
        const float* vrow = a.v + (int64_t)(it.row_begin + (row_ok ? m : 0)) * a.ldv;
        for (int kg = 0; kg < kpad / 8; ++kg) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int k = kg * 8 + e;
                f[e] = (row_ok && k < r) ? vrow[k] : 0.f;
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
            const uint32_t off = (uint32_t)(m >> 3) * sbo_a + (uint32_t)kg * 128 + (uint32_t)(m & 7) * 16;
            *reinterpret_cast<uint4*>(ahi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            *reinterpret_cast<uint4*>(alo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
    }
    cp_async_wait<0>();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    if (tid == 0) {
        const uint32_t idesc = idesc_bf16_f32(128, kExpandN, false, true);
        const uint32_t ah = smem_u32(ahi), al = smem_u32(alo), b = smem_u32(bs);
        for (int ks = 0; ks < kpad / 16; ++ks) {
            const uint64_t bd = smem_desc_noswizzle(b + ks * 256, 128, sbo_b);
            tc_mma_bf16(tmem, smem_desc_noswizzle(ah + ks * 256, 128, sbo_a), bd, idesc, ks > 0);
        }
        for (int ks = 0; ks < kpad / 16; ++ks) {
            const uint64_t bd = smem_desc_noswizzle(b + ks * 256, 128, sbo_b);
            tc_mma_bf16(tmem, smem_desc_noswizzle(al + ks * 256, 128, sbo_a), bd, idesc, true);
        }
        tc_commit(&mma_bar);
    }

    // epilogue: row m = tid, 32 columns per tcgen05.ld
    const int m = warp * 32 + lane;
    int t = -1;
    if (m < rows) {
        t = a.b.token_idx[it.row_begin + m];
        if (t < 0 || t >= a.b.T) {
            atomicOr(&g_err_tc, kErrToken);
            t = -1;
        }
    }
    const bool done = mbar_wait(&mma_bar, 0u, &g_err_tc);
    tc_fence_after();
    for (int c0 = 0; c0 < kExpandN; c0 += 32) {
        uint32_t regs[32];
        tmem_ld_32x32b_x32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, regs);
        tmem_ld_wait();
        const int j = j0 + c0;
        if (t < 0 || !done || j >= a.d_out) continue;
        if (a.y_dtype == 0) {
            uint16_t* yp = static_cast<uint16_t*>(a.y) + (int64_t)t * a.ldy + j;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                uint4 yq = reinterpret_cast<const uint4*>(yp)[q4];
                float yf[8];
                unpack8(yq, yf);
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float lo = fmaf(a.scale, __uint_as_float(regs[q4 * 8 + 2 * e]), yf[2 * e]);
                    const float hi = fmaf(a.scale, __uint_as_float(regs[q4 * 8 + 2 * e + 1]), yf[2 * e + 1]);
                    w[e] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
                           ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
                }
                reinterpret_cast<uint4*>(yp)[q4] = make_uint4(w[0], w[1], w[2], w[3]);
            }
        } else {
            float* yp = static_cast<float*>(a.y) + (int64_t)t * a.ldy + j;
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
                float4 yv = reinterpret_cast<const float4*>(yp)[q4];
                yv.x = fmaf(a.scale, __uint_as_float(regs[q4 * 4 + 0]), yv.x);
                yv.y = fmaf(a.scale, __uint_as_float(regs[q4 * 4 + 1]), yv.y);
                yv.z = fmaf(a.scale, __uint_as_float(regs[q4 * 4 + 2]), yv.z);
                yv.w = fmaf(a.scale, __uint_as_float(regs[q4 * 4 + 3]), yv.w);
                reinterpret_cast<float4*>(yp)[q4] = yv;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kExpandN);
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
    size_t smem = std::max(stage_bytes * kShrinkStages, (size_t)kTcTileRows * a.npad_max * 4);
    smem = std::max(smem, (size_t)80 << 10) + 1024;  // <= two CTAs per SM: tensor memory never oversubscribed
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
    a.n_tiles = (d_out + kExpandN - 1) / kExpandN;
    size_t smem = (size_t)2 * kTcTileRows * a.kpad_max * 2 + (size_t)kExpandN * a.kpad_max * 2;
    smem = std::max(smem, (size_t)56 << 10) + 1024;  // <= four CTAs (4 x 128 tensor-memory columns) per SM
    cudaError_t e = cudaFuncSetAttribute(expand_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    expand_tc_kernel<<<(unsigned)(a.n_tiles * num_tiles), kThreads, smem, stream>>>(a);
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
