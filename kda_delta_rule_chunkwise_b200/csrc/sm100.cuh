// Thin inline-PTX wrappers for the sm_100a features the prefill kernels use:
// tcgen05 (TMEM allocation, MMA, commit, TMEM<->register moves, fences),
// UMMA shared-memory / instruction descriptors, and bulk async copies.
// Descriptor bit layouts follow the PTX ISA description of tcgen05 matrix
// descriptors (start address >> 4 in bits 0-13, leading byte offset >> 4 in
// 16-29, stride byte offset >> 4 in 32-45, version 1 in bits 46-47, swizzle
// mode in bits 61-63) and of the kind::f16 instruction descriptor.
#pragma once

#include <stdint.h>

#include "kda_common.cuh"

namespace kda {
namespace sm100 {

// ------------------------------------------------------------ descriptors

enum Swizzle : uint32_t { SW_NONE = 0, SW_128B = 2, SW_64B = 4, SW_32B = 6 };

// Shared-memory matrix descriptor.  `addr` is a shared-window byte address.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo_bytes,
                                              uint32_t sbo_bytes, Swizzle sw) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;                 // descriptor version for sm_100
    d |= (uint64_t)sw << 61;
    return d;
}

// Instruction descriptor, fp32 accumulate, dense.  `fmt` is the A/B element
// format (A and B always share it): kind::f16 -> 0 = fp16, 1 = bf16;
// kind::tf32 -> 2 = tf32.  a_mn / b_mn: 0 = K-major, 1 = MN-major.
enum : uint32_t { FMT_F16 = 0, FMT_BF16 = 1, FMT_TF32 = 2 };
__host__ __device__ constexpr uint32_t idesc(uint32_t fmt, int M, int N, int a_mn, int b_mn) {
    return (1u << 4)                        // D format: f32
           | (fmt << 7)                     // A format
           | (fmt << 10)                    // B format (same type as A)
           | ((uint32_t)a_mn << 15)         // A major
           | ((uint32_t)b_mn << 16)         // B major
           | ((uint32_t)(N >> 3) << 17)     // N / 8
           | ((uint32_t)(M >> 4) << 24);    // M / 16
}

// ------------------------------------------------------------ TMEM

// Whole warp: allocate `ncols` TMEM columns; the base address is written to *dst_smem.
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Make generic-proxy shared-memory writes visible to the async proxy (MMA reads).
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem], 16-bit inputs (K = 16 per instruction);
// single thread issues.  The idesc must name the same 16-bit type for A and B.
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t id, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(id), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[smem] * B[smem], tf32 inputs stored as 32-bit words
// (K = 8 per instruction).
__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t id, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(id), "r"(accumulate)
        : "memory");
}

// Round an fp32 value to tf32 (nearest, ties away), low 13 mantissa bits zero.
__device__ __forceinline__ float to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return __uint_as_float(r);
}

// Arrive (once) on an mbarrier when all prior tcgen05 ops of this thread complete.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// 32 lanes x 32 bits, 16 consecutive columns: thread i gets lane (base+i).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&r)[16]) {
    uint32_t u[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]),
          "=r"(u[7]), "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]),
          "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) r[i] = __uint_as_float(u[i]);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(__float_as_uint(r[0])), "r"(__float_as_uint(r[1])), "r"(__float_as_uint(r[2])),
        "r"(__float_as_uint(r[3])), "r"(__float_as_uint(r[4])), "r"(__float_as_uint(r[5])),
        "r"(__float_as_uint(r[6])), "r"(__float_as_uint(r[7])), "r"(__float_as_uint(r[8])),
        "r"(__float_as_uint(r[9])), "r"(__float_as_uint(r[10])), "r"(__float_as_uint(r[11])),
        "r"(__float_as_uint(r[12])), "r"(__float_as_uint(r[13])), "r"(__float_as_uint(r[14])),
        "r"(__float_as_uint(r[15]))
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// TMEM address of (lane, column) relative to an allocation base.
__device__ __forceinline__ uint32_t taddr(uint32_t base, uint32_t lane, uint32_t col) {
    return base + (lane << 16) + col;
}

// ------------------------------------------------------------ bulk copies

// 1-D bulk copy global -> shared, completing `bytes` of tx on `bar`.
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst_smem, const void *src, uint32_t bytes,
                                         uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, "
        "[%3];" ::"r"(smem_u32(dst_smem)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// 1-D bulk copy shared -> global in this thread's bulk group (commit with
// bulk_commit).  Both addresses 16-byte aligned, bytes a multiple of 16; the
// shared source must have been made visible to the async proxy.
__device__ __forceinline__ void bulk_s2g(void *dst, const void *src_smem, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                 "r"(smem_u32(src_smem)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until this thread's bulk stores have read their shared-memory sources.
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until this thread's bulk stores have completed.
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// TMA tile load of a 3-D box (coordinates innermost first) described by a tensor
// map passed as a __grid_constant__ kernel parameter, into this CTA's shared
// memory, completing its bytes as tx on `bar`.  No multicast.  The innermost
// coordinate times the element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_3d(void *dst_smem, const void *tmap, int c0, int c1,
                                            int c2, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst_smem)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

// 16-byte async copy global -> shared with zero fill beyond src_bytes (0 or 16).
__device__ __forceinline__ void cp_async16(void *dst_smem, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst_smem)),
                 "l"(src), "r"(src_bytes)
                 : "memory");
}

// Close the current group of this thread's cp.async copies.
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}

// Wait until at most one of this thread's committed cp.async groups is pending.
__device__ __forceinline__ void cp_async_wait_group1() {
    asm volatile("cp.async.wait_group 1;" ::: "memory");
}

// Wait until all of this thread's prior cp.async copies have landed.
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// The mbarrier receives one arrival when all prior cp.async of this thread land.
__device__ __forceinline__ void cp_async_arrive(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// ------------------------------------------------------------ smem layouts

// Byte offset of element (row, col) in a K-major, 128-byte-swizzled 32-bit
// (tf32) tile whose rows hold 32 elements (one 128-byte line) per K-block;
// same swizzle rule as below.
__host__ __device__ __forceinline__ uint32_t sw128_kmajor_off32(uint32_t row, uint32_t col,
                                                                uint32_t kblock_bytes) {
    const uint32_t kb = col >> 5, c = col & 31u;
    const uint32_t chunk = (c >> 2) ^ (row & 7u);
    return kb * kblock_bytes + (row >> 3) * 1024u + (row & 7u) * 128u + chunk * 16u +
           (c & 3u) * 4u;
}

// Byte offset of element (row, col) in a K-major, 128-byte-swizzled 16-bit
// tile whose rows hold 64 elements (one 128-byte line) per K-block:
// 8-row groups are 1024 bytes apart, K-blocks `kblock_bytes` apart.
// The 16-byte chunk index is XOR-ed with (row % 8); the tile base must be
// 1024-byte aligned.
__host__ __device__ __forceinline__ uint32_t sw128_kmajor_off(uint32_t row, uint32_t col,
                                                              uint32_t kblock_bytes) {
    const uint32_t kb = col >> 6, c = col & 63u;
    const uint32_t chunk = (c >> 3) ^ (row & 7u);
    return kb * kblock_bytes + (row >> 3) * 1024u + (row & 7u) * 128u + chunk * 16u +
           (c & 7u) * 2u;
}

// Byte offset of element (mn, k) in an MN-major, 128-byte-swizzled 16-bit tile:
// 64 MN-contiguous elements per 128-byte line, k rows 128 bytes apart,
// 8-row k groups 1024 bytes apart, 64-wide MN blocks `mnblock_bytes` apart.
__host__ __device__ __forceinline__ uint32_t sw128_mnmajor_off(uint32_t mn, uint32_t k,
                                                               uint32_t mnblock_bytes) {
    const uint32_t mb = mn >> 6, m = mn & 63u;
    const uint32_t chunk = (m >> 3) ^ (k & 7u);
    return mb * mnblock_bytes + (k >> 3) * 1024u + (k & 7u) * 128u + chunk * 16u +
           (m & 7u) * 2u;
}

// Byte offset of element (mn, k) in an MN-major 16-bit tile without swizzle:
// 8x8 core matrices (8 MN elements x 8 k rows, 128 contiguous bytes),
// MN-adjacent core matrices 128 bytes apart, k-adjacent ones `kgroup_bytes` apart.
__host__ __device__ __forceinline__ uint32_t interleave_mnmajor_off(uint32_t mn, uint32_t k,
                                                                    uint32_t kgroup_bytes) {
    return (k >> 3) * kgroup_bytes + (mn >> 3) * 128u + (k & 7u) * 16u + (mn & 7u) * 2u;
}

}  // namespace sm100
}  // namespace kda
