// 5th-generation tensor core (tcgen05) helpers for sm_100a: shared-memory operand descriptors,
// the single-thread MMA with its accumulator in tensor memory (TMEM), completion through an
// mbarrier, and the warp-wide TMEM loads.
//
// Operand layout used here (both A and B "K-major", bf16): a [rows][128] tile whose rows are
// split into two 64-element halves; half h is a block of rows x 128 bytes (row r at r * 128
// bytes, so eight rows fill one 1024-byte swizzle atom), and within a row the 16-byte chunk c
// (elements 8c .. 8c + 7 of the half) is stored at chunk position c ^ (r % 8).  This is the
// 128-byte-swizzle canonical layout the tensor core reads; the tile must start on a 1024-byte
// boundary.  ldmatrix reads it without bank conflicts (eight rows of one chunk column land in
// eight different 16-byte bank groups).
#pragma once
#include "carve_mma.cuh"

namespace carve {

// element offset of (row r, column c) in a [rows][128] bf16 tile of the layout above
__host__ __device__ __forceinline__ int umma_off(int r, int c, int rows) {
    return (c >> 6) * (rows * 64) + r * 64 + ((((c >> 3) & 7) ^ (r & 7)) << 3) + (c & 7);
}

// Shared-memory descriptor of a K-major, 128-byte-swizzled operand slice starting at byte
// address `saddr` (the 16 K-elements of one MMA: the start advances 32 bytes per slice inside a
// half, and by rows * 128 bytes to the second half): 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4)      // start address, 16-byte units
           | ((uint64_t)1u << 16)                   // leading-dimension offset (unused when swizzled)
           | ((uint64_t)(1024u >> 4) << 32)         // stride between 8-row groups
           | ((uint64_t)1u << 46)                   // descriptor version of sm_100
           | ((uint64_t)2u << 61);                  // 128-byte swizzle
}

// Instruction descriptor of kind::f16: bf16 A and B (both K-major), fp32 accumulator, M x N.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N) {
    return (1u << 4)                        // accumulator fp32
           | (1u << 7) | (1u << 10)         // A, B bf16
           | ((uint32_t)(N >> 3) << 17)     // N / 8
           | ((uint32_t)(M >> 4) << 24);    // M / 16
}

// D (TMEM) = A B^T (+ D when `accumulate`), issued by one thread.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive (once) on `bar` when every MMA this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(smem_u32(bar))
                 : "memory");
}

// Ordering of tensor-core operations against thread synchronisation (barriers, mbarrier waits).
__device__ __forceinline__ void tc_fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

// TMEM allocation (one whole warp): the base address is written to shared memory at `dst`.
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(dst)), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols) : "memory");
}

// Warp-wide load of TMEM lanes lane0 .. lane0 + 15 (lane0 = this warp's lane quarter base, + 16
// for the upper half), columns col0 .. col0 + 63: thread t receives, for each group j of eight
// columns, (lane t/4, columns 2(t%4), 2(t%4)+1) and (lane t/4 + 8, the same columns), i.e. the
// accumulator fragment of an m16n8 mma.sync tile.
__device__ __forceinline__ void tmem_ld_frags8(uint32_t taddr, float (&d)[8][4]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
          "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
    // the registers are tied to the wait, so that nothing reads them before the load has landed
    asm volatile("tcgen05.wait::ld.sync.aligned;\n"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
                   "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]),
                   "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                   "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) d[j][e] = __uint_as_float(r[4 * j + e]);
}

// ldmatrix fragments from a tile of the layout above ([rows][128], `rows` rows): load_a on an
// [m][k] tile, load_b_kn on a [k][n] tile (see carve_mma.cuh for the fragment conventions)
__device__ __forceinline__ void load_a_um(uint32_t (&a)[4], const __nv_bfloat16 *base, int rows, int m0, int k0,
                                          int lane) {
    const int r = m0 + (lane & 15), k = k0 + (lane >> 4) * 8;
    ldsm_x4(a, smem_u32(base + umma_off(r, k, rows)));
}
__device__ __forceinline__ void load_b_kn_um(uint32_t (&b)[4], const __nv_bfloat16 *base, int rows, int n0, int k0,
                                             int lane) {
    const int k = k0 + (lane & 7) + (((lane >> 3) & 1) << 3), n = n0 + ((lane >> 4) << 3);
    ldsm_x4_t(b, smem_u32(base + umma_off(k, n, rows)));
}

}  // namespace carve
