// SIMT path of SGMV-shrink and SGMV-expand for short segments (decode).
//
// "Multi-LoRA serving: the single translator with a thousand glossaries ..."
// (blog.lo0.es), section "SGMV: the kernel that holds it all up": phase 1
// projects d_in -> r with A_{a(t)}, phase 2 projects r -> d_out with B_{a(t)};
// small segments take a batched gather path.  One launch per phase covers
// every short segment of the batch, whatever its rank, with no padded work.
//
// shrink:  a thread-block cluster of C CTAs per work item (<= 64 rows of one
//          segment) splits d_in into C chunks.  Each CTA streams its chunk of
//          every rank row of A from the page pool into shared memory with bulk
//          asynchronous copies (one per page, completion on an mbarrier), keeps
//          8 columns of up to 4 tokens' x in registers, and reduces the
//          per-thread partial dot products with warp shuffles.  The C partial
//          results are summed in a fixed order through distributed shared
//          memory and written to v: deterministic, no atomics, no scratch.
//
// expand:  one CTA per (work item, tile of d_out columns).  v of the item is
//          staged in shared memory; each thread owns 8 consecutive output
//          columns, streams the B^T rank rows for them with 16-byte loads and
//          updates y in place with a single rounding.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace sgmv {
namespace {

__device__ unsigned int g_err_simt;

constexpr int kMaxStages = 4;

struct ShrinkArgs {
    const uint16_t* x;
    int64_t ldx;
    int32_t d_in;
    BatchView b;
    PoolView pool;
    float* v;
    int64_t ldv;
    int32_t cluster;     // C
    int32_t kc;          // columns of d_in per CTA (multiple of the page size)
    int32_t stages;      // depth of the A ring
    int32_t part_floats; // capacity of the partial buffer
};

struct ExpandArgs {
    const float* v;
    int64_t ldv;
    int32_t d_out;
    BatchView b;
    PoolView pool;
    float scale;
    void* y;
    int64_t ldy;
    int32_t y_dtype;
    int32_t tile_cols;   // output columns per CTA = 8 * blockDim.x
    int32_t num_tiles;
    int32_t span;        // pages of one rank row covered by a tile
};

__device__ __forceinline__ float dot8(const float (&a)[8], const float (&b)[8]) {
    float s = a[0] * b[0];
#pragma unroll
    for (int e = 1; e < 8; ++e) s = fmaf(a[e], b[e], s);
    return s;
}

// Sum N values per thread over the whole CTA.  On return, thread t < N holds
// the CTA-wide sum of value index t.  N is 8, 16 or 32.
template <int N>
__device__ __forceinline__ float block_reduce(float (&vals)[N], float* red, int nwarps) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int LOGN = (N == 8) ? 3 : (N == 16) ? 4 : 5;
    // transpose-reduce: each step halves the values a lane keeps
#pragma unroll
    for (int step = 0; step < LOGN; ++step) {
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
#pragma unroll
    for (int o = (16 >> LOGN); o >= 1; o >>= 1) vals[0] += __shfl_xor_sync(0xFFFFFFFFu, vals[0], o);
    constexpr int SPAN = 32 / N;  // lanes sharing one value index
    if ((lane & (SPAN - 1)) == 0) red[warp * N + (lane >> (5 - LOGN))] = vals[0];
    __syncthreads();
    float s = 0.f;
    if (threadIdx.x < N)
        for (int w = 0; w < nwarps; ++w) s += red[w * N + threadIdx.x];
    __syncthreads();
    return s;
}

// ------------------------------------------------------------------ shrink
template <int G>
__device__ void shrink_item(const ShrinkArgs& a, int i0, int n, int r, int64_t a_base, uint32_t q, uint64_t* bars,
                            uint16_t* ring, float* part, float* red, int* abort_flag) {
    const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, warp = tid >> 5;
    const int P_log2 = a.pool.page_log2, P = 1 << P_log2;
    const int kc = a.kc, c0 = (int)q * kc;
    const int pages_per_row = a.d_in >> P_log2, cpr = kc >> P_log2;
    const int n_groups = (r + 7) >> 3;
    const int NS = a.stages;

    auto issue = [&](int g) {  // warp 0: bulk-copy the chunk of rank rows [8g, 8g+8) into the ring
        const int slot = g % NS;
        const int rows = min(8, r - 8 * g);
        if (lane == 0) mbar_arrive_expect_tx(&bars[slot], (uint32_t)(rows * kc * 2));
        __syncwarp();
        for (int idx = lane; idx < rows * cpr; idx += 32) {
            const int kk = idx / cpr, pq = idx - kk * cpr;
            const int64_t e = a_base + (int64_t)(8 * g + kk) * pages_per_row + (c0 >> P_log2) + pq;
            int32_t page = (e >= 0 && e < a.pool.pt_capacity) ? a.pool.page_table[e] : -1;
            if (page < 0 || page >= a.pool.num_pages) {
                atomicOr(&g_err_simt, kErrPage);
                page = 0;  // keep the transaction count exact; the result is flagged
            }
            bulk_g2s(ring + ((size_t)slot * 8 + kk) * kc + (size_t)pq * P,
                     a.pool.pages + ((int64_t)page << P_log2), (uint32_t)P * 2u, &bars[slot]);
        }
    };
    if (warp == 0)
        for (int g = 0; g < min(NS, n_groups); ++g) issue(g);

    for (int g = 0; g < n_groups; ++g) {
        const int slot = g % NS;
        const uint32_t parity = (uint32_t)((g / NS) & 1);
        if (!mbar_wait(&bars[slot], parity, &g_err_simt)) *abort_flag = 1;
        const uint16_t* As = ring + (size_t)slot * 8 * kc;
        const int rows = min(8, r - 8 * g);
        for (int j0 = 0; j0 < n; j0 += G) {
            float p[8 * G];
#pragma unroll
            for (int i = 0; i < 8 * G; ++i) p[i] = 0.f;
            const uint16_t* xrow[G];
#pragma unroll
            for (int jj = 0; jj < G; ++jj) {
                xrow[jj] = nullptr;
                if (j0 + jj < n) {
                    const int t = a.b.token_idx[i0 + j0 + jj];
                    if (t >= 0 && t < a.b.T) xrow[jj] = a.x + (int64_t)t * a.ldx + c0;
                    else atomicOr(&g_err_simt, kErrToken);
                }
            }
            for (int col = 8 * tid; col < kc; col += 8 * nthr) {
                float xf[G][8];
#pragma unroll
                for (int jj = 0; jj < G; ++jj) {
                    if (xrow[jj]) {
                        const uint4 xq = __ldg(reinterpret_cast<const uint4*>(xrow[jj] + col));
                        unpack8(xq, xf[jj]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) xf[jj][e] = 0.f;
                    }
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint4 aq = *reinterpret_cast<const uint4*>(As + (size_t)kk * kc + col);
                    float af[8];
                    unpack8(aq, af);
#pragma unroll
                    for (int jj = 0; jj < G; ++jj) p[kk * G + jj] += dot8(af, xf[jj]);
                }
            }
            const float s = block_reduce<8 * G>(p, red, nthr >> 5);
            if (tid < 8 * G) {
                const int kk = tid / G, jj = tid - (tid / G) * G;
                if (kk < rows && j0 + jj < n) part[(j0 + jj) * r + 8 * g + kk] = s;
            }
        }
        __syncthreads();  // every thread is done with this slot
        if (warp == 0 && g + NS < n_groups) issue(g + NS);
    }
}

__global__ void __launch_bounds__(256) shrink_simt_kernel(const ShrinkArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int abort_flag;
    const int C = a.cluster;
    const int item_idx = blockIdx.x / C;
    const uint32_t q = cluster_ctarank();
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    uint16_t* ring = reinterpret_cast<uint16_t*>(smem + 128);
    float* part = reinterpret_cast<float*>(smem + 128 + (size_t)a.stages * 8 * a.kc * 2);
    float* red = part + a.part_floats;

    const Item it = a.b.simt_items[item_idx];
    int n = it.row_end - it.row_begin, r = 0;
    int64_t a_base = 0;
    if (it.seg < 0 || it.seg >= a.b.num_segments || it.row_begin < 0 || n < 0 || it.row_end > a.b.num_rows) {
        if (threadIdx.x == 0) atomicOr(&g_err_simt, kErrRows);
        n = 0;
    } else {
        r = a.b.seg_rank[it.seg];
        a_base = a.b.seg_a_pt[(int64_t)it.seg * a.b.n_proj + a.b.proj];
        if (r < 0 || n * r > a.part_floats) {
            if (threadIdx.x == 0) atomicOr(&g_err_simt, kErrRows);
            n = 0;
        }
    }
    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int i = 0; i < a.stages; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }
    __syncthreads();

    if (n > 0 && r > 0) {
        if (n == 1) shrink_item<1>(a, it.row_begin, n, r, a_base, q, bars, ring, part, red, &abort_flag);
        else if (n == 2) shrink_item<2>(a, it.row_begin, n, r, a_base, q, bars, ring, part, red, &abort_flag);
        else shrink_item<4>(a, it.row_begin, n, r, a_base, q, bars, ring, part, red, &abort_flag);
    }

    // Sum the C partial results in a fixed order through distributed shared memory.
    cluster_sync();
    if (n > 0 && r > 0 && !abort_flag) {
        const int E = n * r;
        const int e0 = (int)(((int64_t)E * q) / C), e1 = (int)(((int64_t)E * (q + 1)) / C);
        const uint32_t part_s = smem_u32(part);
        for (int e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
            float s = 0.f;
            for (int qq = 0; qq < C; ++qq) s += ld_cluster_f32(map_cluster(part_s + 4u * (uint32_t)e, (uint32_t)qq));
            const int jrow = e / r, k = e - jrow * r;
            a.v[(int64_t)(it.row_begin + jrow) * a.ldv + k] = s;
        }
    }
    cluster_sync();  // peers keep their shared memory until every read is done
}

// ------------------------------------------------------------------ expand
template <int G>
__device__ void expand_item(const ExpandArgs& a, int i0, int n, int r, const float* vs, const int32_t* pg, int j,
                            int pc) {
    const int P_log2 = a.pool.page_log2;
    const int off = j & ((1 << P_log2) - 1);
    for (int j0 = 0; j0 < n; j0 += G) {
        float acc[G][8];
#pragma unroll
        for (int jj = 0; jj < G; ++jj)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[jj][e] = 0.f;
#pragma unroll 4
        for (int k = 0; k < r; ++k) {
            const int32_t page = pg[k * a.span + pc];
            const uint4 bq = __ldg(reinterpret_cast<const uint4*>(a.pool.pages + ((int64_t)page << P_log2) + off));
            float bf[8];
            unpack8(bq, bf);
#pragma unroll
            for (int jj = 0; jj < G; ++jj) {
                const float w = vs[min(j0 + jj, n - 1) * r + k];
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[jj][e] = fmaf(w, bf[e], acc[jj][e]);
            }
        }
#pragma unroll
        for (int jj = 0; jj < G; ++jj) {
            if (j0 + jj >= n) break;
            const int t = a.b.token_idx[i0 + j0 + jj];
            if (t < 0 || t >= a.b.T) {
                atomicOr(&g_err_simt, kErrToken);
                continue;
            }
            if (a.y_dtype == 0) {
                uint16_t* yp = static_cast<uint16_t*>(a.y) + (int64_t)t * a.ldy + j;
                uint4 yq = *reinterpret_cast<const uint4*>(yp);
                float yf[8];
                unpack8(yq, yf);
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float lo = fmaf(a.scale, acc[jj][2 * e], yf[2 * e]);
                    const float hi = fmaf(a.scale, acc[jj][2 * e + 1], yf[2 * e + 1]);
                    w[e] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
                           ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
                }
                *reinterpret_cast<uint4*>(yp) = make_uint4(w[0], w[1], w[2], w[3]);
            } else {
                float* yp = static_cast<float*>(a.y) + (int64_t)t * a.ldy + j;
                float4 y0 = *reinterpret_cast<const float4*>(yp);
                float4 y1 = *reinterpret_cast<const float4*>(yp + 4);
                y0.x = fmaf(a.scale, acc[jj][0], y0.x); y0.y = fmaf(a.scale, acc[jj][1], y0.y);
                y0.z = fmaf(a.scale, acc[jj][2], y0.z); y0.w = fmaf(a.scale, acc[jj][3], y0.w);
                y1.x = fmaf(a.scale, acc[jj][4], y1.x); y1.y = fmaf(a.scale, acc[jj][5], y1.y);
                y1.z = fmaf(a.scale, acc[jj][6], y1.z); y1.w = fmaf(a.scale, acc[jj][7], y1.w);
                *reinterpret_cast<float4*>(yp) = y0;
                *reinterpret_cast<float4*>(yp + 4) = y1;
            }
        }
    }
}

__global__ void __launch_bounds__(256) expand_simt_kernel(const ExpandArgs a) {
    extern __shared__ __align__(16) uint8_t smem_e[];
    uint8_t* smem = smem_e;
    const int tile = blockIdx.x % a.num_tiles, item_idx = blockIdx.x / a.num_tiles;
    const Item it = a.b.simt_items[item_idx];
    const int n = it.row_end - it.row_begin;
    if (it.seg < 0 || it.seg >= a.b.num_segments || it.row_begin < 0 || n <= 0 || it.row_end > a.b.num_rows) {
        if (threadIdx.x == 0) atomicOr(&g_err_simt, kErrRows);
        return;
    }
    const int r = a.b.seg_rank[it.seg];
    if (r <= 0 || r > kMaxRank || n > kSimtMaxItemRows) {
        if (threadIdx.x == 0 && r != 0) atomicOr(&g_err_simt, kErrRows);
        return;
    }
    const int64_t b_base = a.b.seg_b_pt[(int64_t)it.seg * a.b.n_proj + a.b.proj];
    const int P_log2 = a.pool.page_log2;
    const int j0 = tile * a.tile_cols;
    const int pages_per_row = a.d_out >> P_log2;
    const int first_page = j0 >> P_log2;

    float* vs = reinterpret_cast<float*>(smem);
    int32_t* pg = reinterpret_cast<int32_t*>(vs + kSimtMaxItemRows * kMaxRank);
    for (int e = threadIdx.x; e < n * r; e += blockDim.x) {
        const int jrow = e / r, k = e - jrow * r;
        vs[e] = a.v[(int64_t)(it.row_begin + jrow) * a.ldv + k];
    }
    for (int e = threadIdx.x; e < r * a.span; e += blockDim.x) {
        const int k = e / a.span, pc = e - k * a.span;
        int32_t page = 0;
        if (first_page + pc < pages_per_row) {
            const int64_t ent = b_base + (int64_t)k * pages_per_row + first_page + pc;
            page = (ent >= 0 && ent < a.pool.pt_capacity) ? a.pool.page_table[ent] : -1;
            if (page < 0 || page >= a.pool.num_pages) {
                atomicOr(&g_err_simt, kErrPage);
                page = 0;
            }
        }
        pg[e] = page;
    }
    __syncthreads();
    const int j = j0 + 8 * threadIdx.x;
    if (j >= a.d_out) return;
    const int pc = (j >> P_log2) - first_page;
    if (n == 1) expand_item<1>(a, it.row_begin, n, r, vs, pg, j, pc);
    else if (n == 2) expand_item<2>(a, it.row_begin, n, r, vs, pg, j, pc);
    else expand_item<4>(a, it.row_begin, n, r, vs, pg, j, pc);
}

}  // namespace

cudaError_t launch_shrink_simt(const uint16_t* x, int64_t ldx, int32_t d_in, const BatchView& b, int32_t num_items,
                               int32_t max_item_rows, int32_t max_rank, const PoolView& pool, float* v, int64_t ldv,
                               cudaStream_t stream) {
    if (num_items <= 0) return cudaSuccess;
    const int pages = d_in >> pool.page_log2;
    int C = 1;
    for (int c = 8; c >= 1; --c)
        if (pages % c == 0) {
            C = c;
            break;
        }
    ShrinkArgs a;
    a.x = x;
    a.ldx = ldx;
    a.d_in = d_in;
    a.b = b;
    a.pool = pool;
    a.v = v;
    a.ldv = ldv;
    a.cluster = C;
    a.kc = d_in / C;
    const size_t stage_bytes = (size_t)8 * a.kc * 2;
    a.stages = (int)std::max<size_t>(2, std::min<size_t>(kMaxStages, (96u << 10) / stage_bytes));
    a.part_floats = std::max(1, max_item_rows * max_rank);
    int threads = std::min(256, std::max(32, a.kc / 8));
    threads = (threads + 31) / 32 * 32;
    const size_t smem = 128 + (size_t)a.stages * stage_bytes + (size_t)a.part_floats * 4 + (size_t)(threads / 32) * 32 * 4;
    cudaError_t e = cudaFuncSetAttribute(shrink_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(C * num_items), 1, 1);
    cfg.blockDim = dim3((unsigned)threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, shrink_simt_kernel, a);
}

cudaError_t launch_expand_simt(const float* v, int64_t ldv, int32_t d_out, const BatchView& b, int32_t num_items,
                               int32_t max_item_rows, int32_t max_rank, const PoolView& pool, float scale, void* y,
                               int64_t ldy, int32_t y_dtype, cudaStream_t stream) {
    (void)max_item_rows;
    (void)max_rank;
    if (num_items <= 0) return cudaSuccess;
    ExpandArgs a;
    a.v = v;
    a.ldv = ldv;
    a.d_out = d_out;
    a.b = b;
    a.pool = pool;
    a.scale = scale;
    a.y = y;
    a.ldy = ldy;
    a.y_dtype = y_dtype;
    int threads = 128;
    if ((int64_t)num_items * ((d_out + 1023) / 1024) < 2 * 148) threads = 64;
    a.tile_cols = threads * 8;
    a.num_tiles = (d_out + a.tile_cols - 1) / a.tile_cols;
    const int P = 1 << pool.page_log2;
    a.span = a.tile_cols >= P ? a.tile_cols / P : 1;
    const size_t smem = (size_t)kSimtMaxItemRows * kMaxRank * 4 + (size_t)kMaxRank * a.span * 4;
    cudaError_t e = cudaFuncSetAttribute(expand_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    expand_simt_kernel<<<(unsigned)(a.num_tiles * num_items), threads, smem, stream>>>(a);
    return cudaGetLastError();
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
