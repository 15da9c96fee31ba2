// Paged adapter pool: page allocator, page table and the copy of adapter
// matrices into pages.
//
// The pool is one device buffer of equal-size pages that any adapter may use
// ("Multi-LoRA serving: the single translator with a thousand glossaries ...",
// TL;DR and "Operational pitfalls": weights live in a pool of interchangeable
// blocks, so loading and evicting adapters does not fragment HBM).  For each
// (adapter, projection) the pool keeps A as its r rank rows of d_in values and
// B^T as r rank rows of d_out values; the page table maps every
// (rank row, page-sized chunk) to a page.  A quantised pool (FP8 E4M3 or INT4
// codes with one fp32 scale per rank row: "Multi-LoRA Inference Serving ..."
// (clusterbid.com), paragraphs on the GPU memory budget and on adapter weight
// quantization) quantises rows on the device as it stores them.
#include <cuda_fp8.h>

#include <algorithm>
#include <cmath>
#include <cstring>

#include "internal.h"
#include "ptx.cuh"

namespace sgmv {
namespace {

// Copy a logical [rows][cols] bf16 matrix into pages.  With `transpose`, the
// source is stored as [cols][rows] and is read transposed.  One thread writes
// eight consecutive values (16 bytes) of one logical row.
__global__ void pool_scatter_kernel(const uint16_t* __restrict__ src, int64_t rows, int64_t cols, int transpose,
                                    const int32_t* __restrict__ page_table, int64_t pt_base, int32_t page_log2,
                                    uint16_t* __restrict__ pages, int vec_ok) {
    const int64_t groups_per_row = cols >> 3;
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= rows * groups_per_row) return;
    const int64_t row = g / groups_per_row;
    const int64_t col = (g - row * groups_per_row) << 3;
    const int64_t chunks_per_row = cols >> page_log2;
    const int32_t page = page_table[pt_base + row * chunks_per_row + (col >> page_log2)];
    uint16_t* dst = pages + ((int64_t)page << page_log2) + (col & ((1 << page_log2) - 1));
    uint16_t v[8];
    if (transpose) {
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = src[(col + e) * rows + row];
    } else if (vec_ok) {
        *reinterpret_cast<uint4*>(v) = *reinterpret_cast<const uint4*>(src + row * cols + col);
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = src[row * cols + col + e];
    }
    *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(v);
}

// Quantise a logical [rows][cols] bf16 matrix row by row into a quantised pool
// (one CTA per rank row).  Scale s = max |w| / Q (Q = 448 for E4M3, 7 for
// INT4); code = RN(w / s), E4M3 with saturation, INT4 clamped to [-7, 7]; a
// zero row keeps s = 0 and zero codes.  Both divisions are IEEE (round to
// nearest), so the codes are those of any fp32 implementation of the rule.
// The scale goes to the page-table entry of the row's first chunk.
template <int WF>
__global__ void __launch_bounds__(256) pool_quantize_kernel(const uint16_t* __restrict__ src, int64_t rows,
                                                            int64_t cols, int transpose,
                                                            const int32_t* __restrict__ page_table, int64_t pt_base,
                                                            int32_t page_log2, uint8_t* __restrict__ pages,
                                                            float* __restrict__ row_scale) {
    __shared__ float red[8];
    const int64_t row = blockIdx.x;
    auto val = [&](int64_t c) {
        const uint16_t h = transpose ? src[c * rows + row] : src[row * cols + c];
        return __uint_as_float((uint32_t)h << 16);
    };
    float amax = 0.f;
    for (int64_t c = threadIdx.x; c < cols; c += blockDim.x) amax = fmaxf(amax, fabsf(val(c)));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) amax = fmaxf(amax, red[w]);
    const float s = __fdiv_rn(amax, WF == kFmtFp8 ? 448.f : 7.f);
    const int64_t chunks = cols >> page_log2;
    if (threadIdx.x == 0) row_scale[pt_base + row * chunks] = s;
    for (int64_t c0 = (int64_t)threadIdx.x * 8; c0 < cols; c0 += (int64_t)blockDim.x * 8) {
        const int32_t page = page_table[pt_base + row * chunks + (c0 >> page_log2)];
        const int64_t e = ((int64_t)page << page_log2) + (c0 & ((1 << page_log2) - 1));  // value index
        if (WF == kFmtFp8) {
            uint32_t w[2] = {0u, 0u};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float r = s > 0.f ? __fdiv_rn(val(c0 + i), s) : 0.f;
                w[i >> 2] |= (uint32_t)__nv_cvt_float_to_fp8(r, __NV_SATFINITE, __NV_E4M3) << (8 * (i & 3));
            }
            *reinterpret_cast<uint2*>(pages + e) = make_uint2(w[0], w[1]);
        } else {
            uint32_t w = 0u;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                int q = s > 0.f ? __float2int_rn(__fdiv_rn(val(c0 + i), s)) : 0;
                q = min(7, max(-7, q));
                w |= ((uint32_t)q & 0xFu) << (4 * i);
            }
            *reinterpret_cast<uint32_t*>(pages + (e >> 1)) = w;
        }
    }
}

}  // namespace

cudaError_t write_matrix(sgmv_pool* p, const uint16_t* src, int64_t rows, int64_t cols, bool transpose,
                         int64_t pt_base, cudaStream_t stream) {
    if (rows == 0 || cols == 0) return cudaSuccess;
    if (p->wfmt == kFmtBf16) {
        const int64_t n = rows * (cols >> 3);
        const int threads = 256;
        const int64_t blocks = (n + threads - 1) / threads;
        const int vec_ok = ((reinterpret_cast<uintptr_t>(src) & 15) == 0) ? 1 : 0;
        pool_scatter_kernel<<<(unsigned)blocks, threads, 0, stream>>>(
            src, rows, cols, transpose ? 1 : 0, p->pt_dev, pt_base, p->page_log2,
            static_cast<uint16_t*>(p->pages_dev), vec_ok);
    } else {
        auto kern = p->wfmt == kFmtFp8 ? pool_quantize_kernel<kFmtFp8> : pool_quantize_kernel<kFmtInt4>;
        kern<<<(unsigned)rows, 256, 0, stream>>>(src, rows, cols, transpose ? 1 : 0, p->pt_dev, pt_base,
                                                 p->page_log2, static_cast<uint8_t*>(p->pages_dev), p->scale_dev);
    }
    return cudaGetLastError();
}

namespace {

int64_t adapter_pages(const sgmv_pool* p, int32_t rank) {
    int64_t n = 0;
    for (int i = 0; i < p->n_proj; ++i)
        n += (int64_t)rank * ((p->d_in[i] >> p->page_log2) + (p->d_out[i] >> p->page_log2));
    return n;
}

// First-fit allocation of `n` contiguous page-table entries.
bool pt_alloc(sgmv_pool* p, int64_t n, int64_t* start) {
    if (n == 0) {
        *start = 0;
        return true;
    }
    for (auto it = p->free_pt.begin(); it != p->free_pt.end(); ++it) {
        if (it->second >= n) {
            *start = it->first;
            const int64_t rest = it->second - n, rest_start = it->first + n;
            p->free_pt.erase(it);
            if (rest > 0) p->free_pt[rest_start] = rest;
            return true;
        }
    }
    return false;
}

void pt_free(sgmv_pool* p, int64_t start, int64_t n) {
    if (n == 0) return;
    auto it = p->free_pt.emplace(start, n).first;
    auto next = std::next(it);
    if (next != p->free_pt.end() && it->first + it->second == next->first) {
        it->second += next->second;
        p->free_pt.erase(next);
    }
    if (it != p->free_pt.begin()) {
        auto prev = std::prev(it);
        if (prev->first + prev->second == it->first) {
            prev->second += it->second;
            p->free_pt.erase(it);
        }
    }
}

void release(sgmv_pool* p, int32_t adapter_id) {
    auto it = p->adapters.find(adapter_id);
    if (it == p->adapters.end()) return;
    const AdapterRec& rec = it->second;
    for (int64_t e = rec.pt_begin; e < rec.pt_begin + rec.pt_count; ++e) {
        p->free_pages.push_back(p->pt_host[e]);
        p->pt_host[e] = -1;
    }
    pt_free(p, rec.pt_begin, rec.pt_count);
    p->adapters.erase(it);
}

// Host bookkeeping of a load: find a page-table range for the new placement
// (the adapter's old range, if any, counting as free), then drop the old
// placement and take the range and pages from the free stack.  False, with
// nothing changed (a resident adapter stays resident), when the page table has
// no free range that long.  The caller has checked that the free pages (plus
// the old placement's) suffice.
bool place(sgmv_pool* p, int32_t adapter_id, int32_t rank, AdapterRec* rec) {
    const int64_t need = adapter_pages(p, rank);
    auto old = p->adapters.find(adapter_id);
    int64_t start = 0;
    if (old == p->adapters.end()) {
        if (!pt_alloc(p, need, &start)) return false;
    } else {
        // first fit on a copy of the free ranges with the old range returned: the same
        // search on the real map after the release below gives the same range
        const std::map<int64_t, int64_t> saved = p->free_pt;
        pt_free(p, old->second.pt_begin, old->second.pt_count);
        const bool fits = pt_alloc(p, need, &start);
        p->free_pt = saved;
        if (!fits) return false;
        release(p, adapter_id);
        int64_t again = 0;
        pt_alloc(p, need, &again);
        start = again;
    }
    rec->rank = rank;
    rec->pt_begin = start;
    rec->pt_count = need;
    rec->a_pt.resize(p->n_proj);
    rec->b_pt.resize(p->n_proj);
    int64_t e = start;
    for (int i = 0; i < p->n_proj; ++i) {
        rec->a_pt[i] = e;
        e += (int64_t)rank * (p->d_in[i] >> p->page_log2);
        rec->b_pt[i] = e;
        e += (int64_t)rank * (p->d_out[i] >> p->page_log2);
    }
    for (int64_t k = start; k < start + need; ++k) {
        p->pt_host[k] = (int32_t)p->free_pages.back();
        p->free_pages.pop_back();
    }
    return true;
}

// Undo a placement that no adapter took (its copies failed): its pages and its
// page-table range go back to the free lists.
void unplace(sgmv_pool* p, const AdapterRec& rec) {
    for (int64_t e = rec.pt_begin; e < rec.pt_begin + rec.pt_count; ++e) {
        p->free_pages.push_back(p->pt_host[e]);
        p->pt_host[e] = -1;
    }
    pt_free(p, rec.pt_begin, rec.pt_count);
}

}  // namespace
}  // namespace sgmv

using namespace sgmv;

extern "C" sgmv_status sgmv_pool_create(int device, int64_t num_pages, int32_t page_elems, int32_t n_proj,
                                        const int32_t* d_in, const int32_t* d_out, int32_t max_rank,
                                        sgmv_pool** out) {
    return sgmv_pool_create_ex(device, num_pages, page_elems, n_proj, d_in, d_out, max_rank, SGMV_WEIGHTS_BF16, out);
}

extern "C" sgmv_status sgmv_pool_create_ex(int device, int64_t num_pages, int32_t page_elems, int32_t n_proj,
                                           const int32_t* d_in, const int32_t* d_out, int32_t max_rank,
                                           int32_t weight_format, sgmv_pool** out) {
    if (!out) return fail(SGMV_ERR_INVALID, "pool_create: out is NULL");
    if (weight_format != SGMV_WEIGHTS_BF16 && weight_format != SGMV_WEIGHTS_FP8_E4M3 &&
        weight_format != SGMV_WEIGHTS_INT4)
        return fail(SGMV_ERR_INVALID, "pool_create: unknown weight format");
    *out = nullptr;
    if (num_pages <= 0 || num_pages > (int64_t)INT32_MAX)
        return fail(SGMV_ERR_INVALID, "pool_create: num_pages must be in [1, 2^31-1]");
    if (page_elems < 64 || page_elems > 65536 || (page_elems & (page_elems - 1)))
        return fail(SGMV_ERR_INVALID, "pool_create: page_elems must be a power of two in [64, 65536]");
    if (n_proj <= 0 || !d_in || !d_out) return fail(SGMV_ERR_INVALID, "pool_create: need n_proj > 0 and shapes");
    if (max_rank < 0 || max_rank > kMaxRank) return fail(SGMV_ERR_INVALID, "pool_create: max_rank must be <= 128");
    for (int i = 0; i < n_proj; ++i)
        if (d_in[i] <= 0 || d_out[i] <= 0 || d_in[i] % page_elems || d_out[i] % page_elems)
            return fail(SGMV_ERR_INVALID, "pool_create: every d_in/d_out must be a positive multiple of page_elems");
    auto* p = new sgmv_pool();
    p->device = device;
    p->num_pages = num_pages;
    p->page_elems = page_elems;
    while ((1 << p->page_log2) < page_elems) ++p->page_log2;
    p->n_proj = n_proj;
    p->max_rank = max_rank;
    p->wfmt = weight_format;
    p->page_bytes = weight_format == SGMV_WEIGHTS_BF16 ? 2 * (int64_t)page_elems
                    : weight_format == SGMV_WEIGHTS_FP8_E4M3 ? (int64_t)page_elems : (int64_t)page_elems / 2;
    p->d_in.assign(d_in, d_in + n_proj);
    p->d_out.assign(d_out, d_out + n_proj);
    p->pt_capacity = 2 * num_pages + 1024;
    p->pt_host.assign((size_t)p->pt_capacity, -1);
    p->free_pt[0] = p->pt_capacity;
    p->free_pages.reserve((size_t)num_pages);
    for (int64_t i = num_pages - 1; i >= 0; --i) p->free_pages.push_back(i);  // pop order 0, 1, 2, ...
    if (device >= 0) {
        cudaError_t e = cudaSetDevice(device);
        if (e == cudaSuccess) e = cudaMalloc(&p->pages_dev, (size_t)num_pages * p->page_bytes);
        if (e == cudaSuccess) e = cudaMalloc((void**)&p->pt_dev, (size_t)p->pt_capacity * sizeof(int32_t));
        if (e == cudaSuccess) e = cudaMemset(p->pt_dev, 0xFF, (size_t)p->pt_capacity * sizeof(int32_t));
        if (e == cudaSuccess && weight_format != SGMV_WEIGHTS_BF16) {
            e = cudaMalloc((void**)&p->scale_dev, (size_t)p->pt_capacity * sizeof(float));
            if (e == cudaSuccess) e = cudaMemset(p->scale_dev, 0, (size_t)p->pt_capacity * sizeof(float));
        }
        if (e != cudaSuccess) {
            if (p->pages_dev) cudaFree(p->pages_dev);
            if (p->pt_dev) cudaFree(p->pt_dev);
            if (p->scale_dev) cudaFree(p->scale_dev);
            delete p;
            return cuda_fail(e, "pool_create: device allocation");
        }
    }
    *out = p;
    return SGMV_OK;
}

extern "C" sgmv_status sgmv_pool_destroy(sgmv_pool* p) {
    if (!p) return SGMV_OK;
    if (p->device >= 0) {
        cudaSetDevice(p->device);
        if (p->pages_dev) cudaFree(p->pages_dev);
        if (p->pt_dev) cudaFree(p->pt_dev);
        if (p->scale_dev) cudaFree(p->scale_dev);
        if (p->staging_dev) cudaFree(p->staging_dev);
    }
    delete p;
    return SGMV_OK;
}

extern "C" sgmv_status sgmv_pool_load(sgmv_pool* p, int32_t adapter_id, int32_t rank, const void* const* A,
                                      const void* const* B, int src_on_device, sgmv_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (!p) return fail(SGMV_ERR_INVALID, "pool_load: pool is NULL");
    if (adapter_id < 0) return fail(SGMV_ERR_INVALID, "pool_load: adapter_id must be >= 0");
    if (rank < 0 || rank > p->max_rank) return fail(SGMV_ERR_INVALID, "pool_load: rank outside [0, max_rank]");
    const bool copy = p->device >= 0 && rank > 0;  // a host-only pool keeps bookkeeping only
    if (copy && (!A || !B)) return fail(SGMV_ERR_INVALID, "pool_load: A and B pointer arrays required");
    if (copy)
        for (int i = 0; i < p->n_proj; ++i)
            if (!A[i] || !B[i]) return fail(SGMV_ERR_INVALID, "pool_load: a matrix pointer is NULL");

    // Check room before touching anything (a replaced adapter's own pages count as free).
    const int64_t need = adapter_pages(p, rank);
    int64_t have = (int64_t)p->free_pages.size();
    auto old = p->adapters.find(adapter_id);
    if (old != p->adapters.end()) have += old->second.pt_count;
    if (need > have) return fail(SGMV_ERR_OUT_OF_PAGES, "pool_load: not enough free pages");
    AdapterRec rec;
    if (!place(p, adapter_id, rank, &rec)) return fail(SGMV_ERR_OUT_OF_PAGES, "pool_load: page table is fragmented");
    const int64_t start = rec.pt_begin;

    // the copies; if one fails, the placement goes back to the free lists (the pool stays
    // consistent, and the adapter -- a replaced one included -- is not resident)
    auto copy_in = [&]() -> sgmv_status {
        if (p->device < 0 || need == 0) return SGMV_OK;
        SGMV_CUDA_TRY(cudaSetDevice(p->device));
        SGMV_CUDA_TRY(cudaMemcpyAsync(p->pt_dev + start, p->pt_host.data() + start, (size_t)need * sizeof(int32_t),
                                      cudaMemcpyHostToDevice, stream));
        size_t max_bytes = 0;
        for (int i = 0; i < p->n_proj; ++i)
            max_bytes = std::max(max_bytes, (size_t)rank * std::max(p->d_in[i], p->d_out[i]) * 2);
        if (!src_on_device && p->staging_bytes < max_bytes) {
            if (p->staging_dev) {
                SGMV_CUDA_TRY(cudaStreamSynchronize(stream));
                cudaFree(p->staging_dev);
                p->staging_dev = nullptr;
                p->staging_bytes = 0;
            }
            SGMV_CUDA_TRY(cudaMalloc(&p->staging_dev, max_bytes));
            p->staging_bytes = max_bytes;
        }
        for (int i = 0; i < p->n_proj; ++i) {
            for (int m = 0; m < 2; ++m) {
                const int64_t cols = m == 0 ? p->d_in[i] : p->d_out[i];
                const size_t bytes = (size_t)rank * cols * 2;
                const void* src = m == 0 ? A[i] : B[i];
                if (!src_on_device) {
                    SGMV_CUDA_TRY(cudaMemcpyAsync(p->staging_dev, src, bytes, cudaMemcpyHostToDevice, stream));
                    src = p->staging_dev;
                }
                SGMV_CUDA_TRY(write_matrix(p, static_cast<const uint16_t*>(src), rank, cols, m == 1,
                                           m == 0 ? rec.a_pt[i] : rec.b_pt[i], stream));
                if (!src_on_device) SGMV_CUDA_TRY(cudaStreamSynchronize(stream));  // staging is reused
            }
        }
        SGMV_CUDA_TRY(cudaStreamSynchronize(stream));
        return SGMV_OK;
    };
    const sgmv_status st = copy_in();
    if (st != SGMV_OK) {
        unplace(p, rec);
        return st;
    }
    p->adapters[adapter_id] = std::move(rec);
    return SGMV_OK;
}

extern "C" sgmv_status sgmv_pool_evict(sgmv_pool* p, int32_t adapter_id) {
    if (!p) return fail(SGMV_ERR_INVALID, "pool_evict: pool is NULL");
    if (!p->adapters.count(adapter_id)) return fail(SGMV_ERR_NOT_RESIDENT, "pool_evict: adapter not resident");
    release(p, adapter_id);
    return SGMV_OK;
}

extern "C" sgmv_status sgmv_pool_set_adapter_scale(sgmv_pool* p, int32_t adapter_id, float scale) {
    if (!p) return fail(SGMV_ERR_INVALID, "pool_set_adapter_scale: pool is NULL");
    if (adapter_id < 0) return fail(SGMV_ERR_INVALID, "pool_set_adapter_scale: adapter_id must be >= 0");
    if (!std::isfinite(scale)) return fail(SGMV_ERR_INVALID, "pool_set_adapter_scale: scale must be finite");
    if (scale == 1.0f) p->adapter_scale.erase(adapter_id);
    else p->adapter_scale[adapter_id] = scale;
    return SGMV_OK;
}

extern "C" sgmv_status sgmv_pool_get_adapter_scale(const sgmv_pool* p, int32_t adapter_id, float* scale) {
    if (!p || !scale) return fail(SGMV_ERR_INVALID, "pool_get_adapter_scale: NULL argument");
    if (adapter_id < 0) return fail(SGMV_ERR_INVALID, "pool_get_adapter_scale: adapter_id must be >= 0");
    const auto it = p->adapter_scale.find(adapter_id);
    *scale = it == p->adapter_scale.end() ? 1.0f : it->second;
    return SGMV_OK;
}

extern "C" sgmv_status sgmv_pool_get_stats(const sgmv_pool* p, sgmv_pool_stats* out) {
    if (!p || !out) return fail(SGMV_ERR_INVALID, "pool_get_stats: NULL argument");
    out->num_pages = p->num_pages;
    out->free_pages = (int64_t)p->free_pages.size();
    out->page_bytes = p->page_bytes;
    out->payload_bytes = (p->num_pages - out->free_pages) * out->page_bytes;
    out->resident_adapters = (int32_t)p->adapters.size();
    out->page_elems = p->page_elems;
    out->weight_format = p->wfmt;
    out->reserved = 0;
    return SGMV_OK;
}

extern "C" sgmv_status sgmv_pool_adapter_rank(const sgmv_pool* p, int32_t adapter_id, int32_t* rank) {
    if (!p || !rank) return fail(SGMV_ERR_INVALID, "pool_adapter_rank: NULL argument");
    auto it = p->adapters.find(adapter_id);
    if (it == p->adapters.end()) return fail(SGMV_ERR_NOT_RESIDENT, "pool_adapter_rank: adapter not resident");
    *rank = it->second.rank;
    return SGMV_OK;
}

extern "C" sgmv_status sgmv_pool_adapter_pages(const sgmv_pool* p, int32_t adapter_id, int32_t proj,
                                               int32_t matrix, int32_t* page_ids, int64_t cap, int64_t* n) {
    if (!p || !n) return fail(SGMV_ERR_INVALID, "pool_adapter_pages: NULL argument");
    if (proj < 0 || proj >= p->n_proj || (matrix != 0 && matrix != 1))
        return fail(SGMV_ERR_INVALID, "pool_adapter_pages: bad projection or matrix");
    auto it = p->adapters.find(adapter_id);
    if (it == p->adapters.end()) return fail(SGMV_ERR_NOT_RESIDENT, "pool_adapter_pages: adapter not resident");
    const AdapterRec& rec = it->second;
    const int64_t d = matrix == 0 ? p->d_in[proj] : p->d_out[proj];
    const int64_t count = (int64_t)rec.rank * (d >> p->page_log2);
    *n = count;
    if (count > cap || (count > 0 && !page_ids)) return fail(SGMV_ERR_CAPACITY, "pool_adapter_pages: buffer too small");
    const int64_t base = matrix == 0 ? rec.a_pt[proj] : rec.b_pt[proj];
    for (int64_t i = 0; i < count; ++i) page_ids[i] = p->pt_host[base + i];
    return SGMV_OK;
}

extern "C" sgmv_status sgmv_pool_read(const sgmv_pool* p, int32_t adapter_id, int32_t proj, int32_t matrix,
                                      void* codes, int64_t cap_codes, float* scales, int64_t cap_scales,
                                      sgmv_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (!p) return fail(SGMV_ERR_INVALID, "pool_read: pool is NULL");
    if (p->device < 0 || !p->pages_dev) return fail(SGMV_ERR_INVALID, "pool_read: pool has no device memory");
    if (proj < 0 || proj >= p->n_proj || (matrix != 0 && matrix != 1))
        return fail(SGMV_ERR_INVALID, "pool_read: bad projection or matrix");
    auto it = p->adapters.find(adapter_id);
    if (it == p->adapters.end()) return fail(SGMV_ERR_NOT_RESIDENT, "pool_read: adapter not resident");
    const AdapterRec& rec = it->second;
    const int64_t d = matrix == 0 ? p->d_in[proj] : p->d_out[proj];
    const int64_t cpr = d >> p->page_log2;                  // chunks (pages) per rank row
    const int64_t row_bytes = cpr * p->page_bytes;
    if (codes && cap_codes < rec.rank * row_bytes) return fail(SGMV_ERR_CAPACITY, "pool_read: codes buffer too small");
    if (scales && cap_scales < rec.rank) return fail(SGMV_ERR_CAPACITY, "pool_read: scales buffer too small");
    const int64_t base = matrix == 0 ? rec.a_pt[proj] : rec.b_pt[proj];
    SGMV_CUDA_TRY(cudaSetDevice(p->device));
    const uint8_t* pages = static_cast<const uint8_t*>(p->pages_dev);
    if (codes)
        for (int64_t k = 0; k < rec.rank; ++k)
            for (int64_t c = 0; c < cpr; ++c)
                SGMV_CUDA_TRY(cudaMemcpyAsync(static_cast<uint8_t*>(codes) + k * row_bytes + c * p->page_bytes,
                                              pages + (int64_t)p->pt_host[base + k * cpr + c] * p->page_bytes,
                                              (size_t)p->page_bytes, cudaMemcpyDeviceToHost, stream));
    std::vector<float> sc((size_t)std::max<int64_t>(rec.rank * cpr, 1), 1.0f);
    if (scales && p->scale_dev && rec.rank > 0)
        SGMV_CUDA_TRY(cudaMemcpyAsync(sc.data(), p->scale_dev + base, (size_t)(rec.rank * cpr) * sizeof(float),
                                      cudaMemcpyDeviceToHost, stream));
    SGMV_CUDA_TRY(cudaStreamSynchronize(stream));
    if (scales)
        for (int64_t k = 0; k < rec.rank; ++k) scales[k] = p->scale_dev ? sc[(size_t)(k * cpr)] : 1.0f;
    return SGMV_OK;
}

extern "C" const void* sgmv_pool_pages_device(const sgmv_pool* p) { return p ? p->pages_dev : nullptr; }

extern "C" sgmv_status sgmv_pool_shuffle_free_pages(sgmv_pool* p, uint64_t seed) {
    if (!p) return fail(SGMV_ERR_INVALID, "pool_shuffle_free_pages: pool is NULL");
    uint64_t z = seed ? seed : 0x9E3779B97F4A7C15ull;
    for (size_t i = p->free_pages.size(); i > 1; --i) {  // Fisher-Yates with xorshift64*
        z ^= z >> 12; z ^= z << 25; z ^= z >> 27;
        const size_t j = (size_t)((z * 0x2545F4914F6CDD1Dull) % i);
        std::swap(p->free_pages[i - 1], p->free_pages[j]);
    }
    return SGMV_OK;
}

// ---------------------------------------------------------------------------
// Residency manager: adapters registered with host copies are made resident on
// demand, batch by batch, least-recently-used adapters giving way.

struct sgmv_residency {
    sgmv_pool* pool = nullptr;
    struct Host {
        int32_t rank = 0;
        std::vector<const void*> A, B;
    };
    std::unordered_map<int32_t, Host> host;       // registered host copies
    std::unordered_map<int32_t, uint64_t> used;   // resident adapter -> batch tick of its last use
    uint64_t tick = 0;
    void* staging = nullptr;                      // device staging for host -> device copies
    size_t staging_bytes = 0;
    cudaEvent_t before = nullptr, after = nullptr;
    sgmv_residency_stats stats{};
};

namespace {

// Largest matrix of one adapter of rank `rank` (bytes).
size_t largest_matrix(const sgmv_pool* p, int32_t rank) {
    size_t m = 0;
    for (int i = 0; i < p->n_proj; ++i) m = std::max(m, (size_t)rank * std::max(p->d_in[i], p->d_out[i]) * 2);
    return m;
}

}  // namespace

extern "C" sgmv_status sgmv_residency_create(sgmv_pool* pool, sgmv_residency** out) {
    if (!pool || !out) return fail(SGMV_ERR_INVALID, "residency_create: NULL argument");
    auto* r = new sgmv_residency();
    r->pool = pool;
    if (pool->device >= 0) {
        SGMV_CUDA_TRY(cudaSetDevice(pool->device));
        r->staging_bytes = std::max<size_t>(largest_matrix(pool, pool->max_rank), 16);
        cudaError_t e = cudaMalloc(&r->staging, r->staging_bytes);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&r->before, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&r->after, cudaEventDisableTiming);
        if (e != cudaSuccess) {
            if (r->staging) cudaFree(r->staging);
            if (r->before) cudaEventDestroy(r->before);
            delete r;
            return cuda_fail(e, "residency_create");
        }
    }
    // adapters already resident take part in the LRU order as the oldest
    for (const auto& kv : pool->adapters) r->used[kv.first] = 0;
    *out = r;
    return SGMV_OK;
}

extern "C" sgmv_status sgmv_residency_destroy(sgmv_residency* r) {
    if (!r) return SGMV_OK;
    if (r->pool && r->pool->device >= 0) {
        cudaSetDevice(r->pool->device);
        cudaDeviceSynchronize();  // copies in flight read the staging buffer
        if (r->staging) cudaFree(r->staging);
        if (r->before) cudaEventDestroy(r->before);
        if (r->after) cudaEventDestroy(r->after);
    }
    delete r;
    return SGMV_OK;
}

extern "C" sgmv_status sgmv_residency_register(sgmv_residency* r, int32_t adapter_id, int32_t rank,
                                               const void* const* A_host, const void* const* B_host) {
    if (!r) return fail(SGMV_ERR_INVALID, "residency_register: NULL manager");
    if (adapter_id < 0) return fail(SGMV_ERR_INVALID, "residency_register: adapter_id must be >= 0");
    sgmv_pool* p = r->pool;
    if (rank < 0 || rank > p->max_rank) return fail(SGMV_ERR_INVALID, "residency_register: rank outside [0, max_rank]");
    sgmv_residency::Host h;
    h.rank = rank;
    if (p->device >= 0 && rank > 0) {
        if (!A_host || !B_host) return fail(SGMV_ERR_INVALID, "residency_register: A and B pointer arrays required");
        for (int i = 0; i < p->n_proj; ++i) {
            if (!A_host[i] || !B_host[i]) return fail(SGMV_ERR_INVALID, "residency_register: a matrix pointer is NULL");
            h.A.push_back(A_host[i]);
            h.B.push_back(B_host[i]);
        }
    }
    r->host[adapter_id] = std::move(h);
    return SGMV_OK;
}

extern "C" sgmv_status sgmv_residency_unregister(sgmv_residency* r, int32_t adapter_id) {
    if (!r) return fail(SGMV_ERR_INVALID, "residency_unregister: NULL manager");
    if (!r->host.erase(adapter_id)) return fail(SGMV_ERR_NOT_RESIDENT, "residency_unregister: not registered");
    return SGMV_OK;
}

extern "C" sgmv_status sgmv_residency_prepare(sgmv_residency* r, const int32_t* adapter_ids, int32_t T,
                                              sgmv_stream_t copy_stream_, sgmv_stream_t compute_stream_,
                                              int32_t* loaded) {
    if (!r) return fail(SGMV_ERR_INVALID, "residency_prepare: NULL manager");
    if (T < 0 || (T > 0 && !adapter_ids)) return fail(SGMV_ERR_INVALID, "residency_prepare: bad batch");
    sgmv_pool* p = r->pool;
    cudaStream_t copy_stream = reinterpret_cast<cudaStream_t>(copy_stream_);
    cudaStream_t compute_stream = reinterpret_cast<cudaStream_t>(compute_stream_);
    const uint64_t tick = ++r->tick;
    // the batch's distinct adapters; check all of them before changing anything
    std::vector<int32_t> ids;
    for (int32_t t = 0; t < T; ++t)
        if (adapter_ids[t] >= 0) ids.push_back(adapter_ids[t]);
    std::sort(ids.begin(), ids.end());
    ids.erase(std::unique(ids.begin(), ids.end()), ids.end());
    std::vector<int32_t> missing;
    int64_t need = 0;
    for (int32_t a : ids) {
        if (p->adapters.count(a)) continue;
        auto h = r->host.find(a);
        if (h == r->host.end())
            return fail(SGMV_ERR_NOT_RESIDENT, "residency_prepare: adapter " + std::to_string(a) +
                                                   " is neither resident nor registered");
        missing.push_back(a);
        need += adapter_pages(p, h->second.rank);
    }
    int64_t evictable = 0;  // pages of resident adapters the batch does not use
    for (const auto& kv : p->adapters)
        if (!std::binary_search(ids.begin(), ids.end(), kv.first)) evictable += kv.second.pt_count;
    if (need > (int64_t)p->free_pages.size() + evictable)
        return fail(SGMV_ERR_OUT_OF_PAGES, "residency_prepare: the batch's adapters do not fit in the pool");
    r->stats.hits += (int64_t)(ids.size() - missing.size());
    r->stats.misses += (int64_t)missing.size();
    for (int32_t a : ids)
        if (p->adapters.count(a)) r->used[a] = tick;

    // evict least recently used adapters outside the batch until the misses fit
    while (need > (int64_t)p->free_pages.size()) {
        int32_t victim = -1;
        uint64_t oldest = UINT64_MAX;
        for (const auto& kv : p->adapters) {
            if (std::binary_search(ids.begin(), ids.end(), kv.first)) continue;
            auto u = r->used.find(kv.first);
            const uint64_t t = u == r->used.end() ? 0 : u->second;
            if (t < oldest || (t == oldest && kv.first < victim)) {
                oldest = t;
                victim = kv.first;
            }
        }
        if (victim < 0) break;
        release(p, victim);
        r->used.erase(victim);
        ++r->stats.evictions;
    }

    const bool dev = p->device >= 0;
    if (dev && !missing.empty()) {
        SGMV_CUDA_TRY(cudaSetDevice(p->device));
        // pages and page-table entries given up by evicted adapters may still be read
        // by work already queued on the compute stream: the copies that overwrite
        // them wait for it
        SGMV_CUDA_TRY(cudaEventRecord(r->before, compute_stream));
        SGMV_CUDA_TRY(cudaStreamWaitEvent(copy_stream, r->before, 0));
    }
    for (int32_t a : missing) {
        const sgmv_residency::Host& h = r->host.at(a);
        AdapterRec rec;
        if (!place(p, a, h.rank, &rec))
            return fail(SGMV_ERR_OUT_OF_PAGES, "residency_prepare: page table is fragmented");
        // a failed copy returns this adapter's placement to the free lists (adapters loaded
        // before it in this call stay resident)
        int64_t loaded_bytes = 0;
        auto copy_in = [&]() -> sgmv_status {
            if (!dev || rec.pt_count == 0) return SGMV_OK;
            SGMV_CUDA_TRY(cudaMemcpyAsync(p->pt_dev + rec.pt_begin, p->pt_host.data() + rec.pt_begin,
                                          (size_t)rec.pt_count * sizeof(int32_t), cudaMemcpyHostToDevice,
                                          copy_stream));
            for (int i = 0; i < p->n_proj; ++i) {
                for (int m = 0; m < 2; ++m) {
                    const int64_t cols = m == 0 ? p->d_in[i] : p->d_out[i];
                    const size_t bytes = (size_t)h.rank * cols * 2;
                    // the staging buffer is reused in stream order: each copy follows the
                    // previous scatter on the copy stream
                    SGMV_CUDA_TRY(cudaMemcpyAsync(r->staging, m == 0 ? h.A[i] : h.B[i], bytes,
                                                  cudaMemcpyHostToDevice, copy_stream));
                    SGMV_CUDA_TRY(write_matrix(p, static_cast<const uint16_t*>(r->staging), h.rank, cols, m == 1,
                                               m == 0 ? rec.a_pt[i] : rec.b_pt[i], copy_stream));
                    loaded_bytes += (int64_t)bytes;
                }
            }
            return SGMV_OK;
        };
        const sgmv_status st = copy_in();
        if (st != SGMV_OK) {
            unplace(p, rec);
            return st;
        }
        r->stats.bytes_loaded += loaded_bytes;
        p->adapters[a] = std::move(rec);
        r->used[a] = tick;
    }
    if (dev && !missing.empty()) {
        SGMV_CUDA_TRY(cudaEventRecord(r->after, copy_stream));
        SGMV_CUDA_TRY(cudaStreamWaitEvent(compute_stream, r->after, 0));
    }
    if (loaded) *loaded = (int32_t)missing.size();
    return SGMV_OK;
}

extern "C" sgmv_status sgmv_residency_get_stats(const sgmv_residency* r, sgmv_residency_stats* out) {
    if (!r || !out) return fail(SGMV_ERR_INVALID, "residency_get_stats: NULL argument");
    *out = r->stats;
    return SGMV_OK;
}
