// Thin inline-PTX wrappers for sm_100a: mbarriers, bulk async copies (no
// multicast), thread-block-cluster shared memory, cp.async, the tcgen05
// tensor-core / tensor-memory instructions, and the warp-level ldmatrix / mma.sync
// pair the SIMT kernels use for their small contractions.  Every wait here is bounded.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace sgmv {

// Device error bits (see sgmv_check_errors in include/sgmv.h).
enum : uint32_t {
    kErrPage = 1u,     // page id outside the pool
    kErrToken = 2u,    // token row outside the batch
    kErrTimeout = 4u,  // a bounded wait gave up
    kErrRows = 8u,     // segment rows outside the plan
};

// Roughly one second of SM clocks at ~2 GHz: any wait longer than this is a bug.
constexpr long long kWaitLimitCycles = 2000000000LL;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Wait for the phase with the given parity to complete.  Returns false (and
// sets kErrTimeout in *err) if it did not complete within kWaitLimitCycles.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned int* err) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > kWaitLimitCycles) {
            atomicOr(err, kErrTimeout);
            return false;
        }
    }
    return true;
}

// ------------------------------------------------------- bulk async copies
// Global -> this CTA's shared memory, completion counted on `bar` in bytes.
// `bytes` is a multiple of 16; both addresses are 16-byte aligned.
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Add `bytes` to the transaction count the current phase of `bar` waits for
// (no arrival).
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
// This CTA's shared memory -> global, tracked by the thread's bulk groups.
// Both addresses 16-byte aligned, `bytes` a multiple of 16.
__device__ __forceinline__ void bulk_s2g(void* dst_gmem, const void* src_smem, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst_gmem),
                 "r"(smem_u32(src_smem)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// The thread's bulk stores have finished reading shared memory (all groups, or
// all but the newest one).
__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read_but1() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
// The thread's bulk stores are complete (written to global memory).
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// 2-D tiled TMA copies (no multicast).  `map` is the address of a tensor map
// held in kernel parameters; x (innermost, elements) times the element size is
// a multiple of 16 bytes; a store never starts at a negative coordinate.
__device__ __forceinline__ void tma_load_2d(void* dst_smem, const void* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst_smem)),
        "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tma_store_2d(const void* map, int x, int y, const void* src_smem) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(map), "r"(x),
                 "r"(y), "r"(smem_u32(src_smem))
                 : "memory");
}
// Barrier `id` among `count` threads that also returns the AND of `v` over them.
__device__ __forceinline__ bool named_bar_and(int id, int count, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

// ------------------------------------------------------ cp.async (16 bytes)
__device__ __forceinline__ void cp_async16(void* dst_smem, const void* src_gmem, bool valid) {
    // src-size 0 writes sixteen zero bytes and reads nothing.
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst_smem)), "l"(src_gmem),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
// 8- and 4-byte copies (through L1: the .cg form takes only 16 bytes).
__device__ __forceinline__ void cp_async8(void* dst_smem, const void* src_gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(dst_smem)), "l"(src_gmem) : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst_smem, const void* src_gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst_smem)), "l"(src_gmem) : "memory");
}
// A copy of B bytes (16, 8 or 4) that is always valid.
template <int B>
__device__ __forceinline__ void cp_async_n(void* dst_smem, const void* src_gmem) {
    if constexpr (B == 16) cp_async16(dst_smem, src_gmem, true);
    else if constexpr (B == 8) cp_async8(dst_smem, src_gmem);
    else cp_async4(dst_smem, src_gmem);
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// Arrive on `bar` once all cp.async copies this thread issued so far have
// completed; the arrival counts against the count the barrier was created with.
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Barrier `id` (1..15) among `count` threads (a multiple of 32).
__device__ __forceinline__ void named_bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Programmatic dependent launch: let the next kernel of the stream be scheduled (its
// CTAs start as resources free up), and wait until the preceding kernel has completed
// and its memory operations are visible (returns at once without such a dependency).
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ cluster
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory location in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_cluster(uint32_t local_smem, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_smem), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}
// 16 bytes from a cluster shared-memory address (16-byte aligned).
__device__ __forceinline__ float4 ld_cluster_v4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}
// Arrive once on `bar` when all previously issued tcgen05.mma of this thread complete.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}
// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane
// (base lane + i), columns [col, col+32).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
          "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, no swizzle ("interleaved" canonical
// layout: 8 rows x 16 bytes core matrices).  lbo = byte distance between
// core matrices along K, sbo = along M/N.  Version bits 46-47 = 1 (sm_100).
__device__ __forceinline__ uint64_t smem_desc_noswizzle(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;
    // base offset 0, lbo mode 0, layout type 0 (no swizzle)
    return d;
}
// Shared-memory matrix descriptor, 128-byte swizzle: atoms of 8 rows x 128
// bytes whose 16-byte chunks are permuted by XOR with the row index (bits 4-6
// of the address XOR bits 7-9), atoms 1024-byte aligned.  K-major operands:
// lbo unused (1), sbo = stride of 8-row groups; MN-major operands: lbo = stride
// of 64-element MN atoms, sbo = stride of 8-row K groups.  Layout type 2 in
// bits 61-63, version 1 in bits 46-47.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}
// Byte offset of 16-byte chunk `chunk` (0-7) of row `row` inside a 128B-swizzled atom.
__host__ __device__ __forceinline__ uint32_t sw128_off(uint32_t row, uint32_t chunk) {
    return (row & 7u) * 128u + ((chunk ^ (row & 7u)) & 7u) * 16u;
}

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
    return (1u << 4)                           // D format: f32
           | (1u << 7)                         // A format: bf16
           | (1u << 10)                        // B format: bf16
           | ((a_mn_major ? 1u : 0u) << 15)    // A major
           | ((b_mn_major ? 1u : 0u) << 16)    // B major
           | ((uint32_t)(N >> 3) << 17)        // N / 8
           | ((uint32_t)(M >> 4) << 24);       // M / 16
}

// ------------------------------------------------------------------ bf16
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ void unpack8(const uint4& q, float (&f)[8]) {
    f[0] = bf16lo(q.x); f[1] = bf16hi(q.x);
    f[2] = bf16lo(q.y); f[3] = bf16hi(q.y);
    f[4] = bf16lo(q.z); f[5] = bf16hi(q.z);
    f[6] = bf16lo(q.w); f[7] = bf16hi(q.w);
}

// Eight E4M3 codes (byte i = value i) to fp32, exactly: each pair goes through
// the hardware E4M3x2 -> f16x2 conversion (every E4M3 value is an f16 value).
__device__ __forceinline__ void fp8x8_to_f32(const uint2& q, float (&f)[8]) {
    const uint32_t w[2] = {q.x, q.y};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        uint32_t hh;
        const uint16_t pair = (uint16_t)(w[h >> 1] >> (16 * (h & 1)));
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(hh) : "h"(pair));
        float lo, hi;
        asm("cvt.f32.f16 %0, %1;" : "=f"(lo) : "h"((uint16_t)(hh & 0xFFFFu)));
        asm("cvt.f32.f16 %0, %1;" : "=f"(hi) : "h"((uint16_t)(hh >> 16)));
        f[2 * h] = lo;
        f[2 * h + 1] = hi;
    }
}

// Eight INT4 codes (two's complement nibbles, value i in bits 4i..4i+3) to fp32,
// exactly: with n = nibble ^ 8 (0..15), the float whose bits are 0x4B000000 | n
// is 2^23 + n, and 2^23 + n - (2^23 + 8) = n - 8 is the nibble's signed value.
__device__ __forceinline__ void int4x8_to_f32(uint32_t q, float (&f)[8]) {
    const uint32_t flipped = q ^ 0x88888888u;
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = __uint_as_float(0x4B000000u | ((flipped >> (4 * i)) & 0xFu)) - 8388616.0f;
}

// Eight INT4 codes as position-scaled fp32: f[i] = q_i * 16^(i % 4), exactly, in two
// operations a value.  With n = nibble ^ 8, the float with bits 0x4B000000 | (n << 4j)
// (j = i % 4, the nibble kept in place inside the low 16 bits) is 2^23 + n 16^j, an
// integer below 2^24; subtracting 2^23 + 8 * 16^j is exact and leaves (n - 8) 16^j.
// The caller undoes the factor 16^j on the other operand (x) or on the sum, both exact
// power-of-two scalings.
__device__ __forceinline__ void int4x8_to_f32_pos(uint32_t q, float (&f)[8]) {
    const uint32_t lo = q ^ 0x88888888u, hi = lo >> 16;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float c = 8388608.0f + 8.0f * (float)(1u << (4 * i));
        f[i] = __uint_as_float(0x4B000000u | (lo & (0xFu << (4 * i)))) - c;
        f[i + 4] = __uint_as_float(0x4B000000u | (hi & (0xFu << (4 * i)))) - c;
    }
}
// 16^-(i % 4): the factor that int4x8_to_f32_pos leaves on value i
__device__ __forceinline__ float int4_pos_unscale(int i) {
    return i % 4 == 0 ? 1.0f : i % 4 == 1 ? 0.0625f : i % 4 == 2 ? 0.00390625f : 0.000244140625f;
}

// ------------------------------------------------------------------ warp-level mma
// ldmatrix: lanes 8i..8i+7 give the row addresses (16 bytes each) of 8x8 matrix i;
// lane l receives, of every matrix, the pair (row l/4, columns 2(l%4), 2(l%4)+1), or with
// .trans the pair (rows 2(l%4), 2(l%4)+1, column l/4).
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t (&r)[2]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(addr));
}
// D(16x8, fp32) += A(16x16, bf16, row-major fragment) x B(16x8, bf16, column fragment).
// Fragments, with g = lane / 4 and t = lane % 4: a = {A[g][2t..], A[g+8][2t..], A[g][2t+8..],
// A[g+8][2t+8..]}, b = {B[2t..][g], B[2t+8..][g]}, d = {D[g][2t], D[g][2t+1], D[g+8][2t],
// D[g+8][2t+1]}; each 32-bit register holds two bf16, the lower index in the low half.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Two fp32 to a bf16 pair (round to nearest even), lo in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
           ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
}

// Eight stored weights of format WF at p (16, 8 or 4 bytes) to fp32.
template <int WF>
__device__ __forceinline__ void load_w8(const uint8_t* p, float (&f)[8]) {
    if constexpr (WF == 0) unpack8(*reinterpret_cast<const uint4*>(p), f);
    else if constexpr (WF == 1) fp8x8_to_f32(*reinterpret_cast<const uint2*>(p), f);
    else int4x8_to_f32(*reinterpret_cast<const uint32_t*>(p), f);
}

}  // namespace sgmv
