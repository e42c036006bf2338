// Tensor-core, bulk-copy and barrier helpers for the CARVE tensor-core kernels (sm_100a).
//
// Fragment conventions (bf16 m16n8k16, fp32 accumulate), lane l, g = l / 4, c = l % 4:
//   C/D (16x8 fp32):  d0 (row g,   col 2c), d1 (row g,   col 2c+1),
//                     d2 (row g+8, col 2c), d3 (row g+8, col 2c+1)
//   A (16x16 bf16):   a0 (row g, k 2c..2c+1), a1 (row g+8, k 2c..), a2 (row g, k 2c+8..),
//                     a3 (row g+8, k 2c+8..)
//   B (16x8 bf16):    b0 (k 2c..2c+1, col g), b1 (k 2c+8.., col g)
// Two adjacent C tiles (cols n0..n0+15) therefore repack into one A fragment without any
// data movement between lanes.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace carve {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// bf16x2 operand times a pair of factors (rounded to bf16), one packed multiply
__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t v, float f_lo, float f_hi) {
    const uint32_t f = pack_bf16(f_lo, f_hi);
    const __nv_bfloat162 r =
        __hmul2(*reinterpret_cast<const __nv_bfloat162 *>(&v), *reinterpret_cast<const __nv_bfloat162 *>(&f));
    return *reinterpret_cast<const uint32_t *>(&r);
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// A fragment (16x16) of a row-major [m][k] bf16 tile: rows m0.., cols k0.. (ld in elements)
__device__ __forceinline__ void load_a(uint32_t (&a)[4], const __nv_bfloat16 *base, int ld, int m0, int k0, int lane) {
    const int r = m0 + (lane & 15), k = k0 + (lane >> 4) * 8;
    ldsm_x4(a, smem_u32(base + r * ld + k));
}

// A fragment (16x16) of A = X^T where X is a row-major [k][m] tile (rows k0.., cols m0..)
__device__ __forceinline__ void load_a_t(uint32_t (&a)[4], const __nv_bfloat16 *base, int ld, int m0, int k0, int lane) {
    const int mat = lane >> 3, r = lane & 7;
    const int k = k0 + r + ((mat >> 1) << 3), m = m0 + ((mat & 1) << 3);
    ldsm_x4_t(a, smem_u32(base + k * ld + m));
}

// B fragments of two n-tiles (n0.., n0+8..) x 16 k from an [n][k] tile (k contiguous):
// b[0], b[1] -> tile n0;  b[2], b[3] -> tile n0+8
__device__ __forceinline__ void load_b_nk(uint32_t (&b)[4], const __nv_bfloat16 *base, int ld, int n0, int k0, int lane) {
    const int n = n0 + (lane & 7) + ((lane >> 4) << 3), k = k0 + ((lane >> 3) & 1) * 8;
    ldsm_x4(b, smem_u32(base + n * ld + k));
}

// B fragments of two n-tiles from a [k][n] tile (n contiguous), via the transposing load
__device__ __forceinline__ void load_b_kn(uint32_t (&b)[4], const __nv_bfloat16 *base, int ld, int n0, int k0, int lane) {
    const int k = k0 + (lane & 7) + (((lane >> 3) & 1) << 3), n = n0 + ((lane >> 4) << 3);
    ldsm_x4_t(b, smem_u32(base + k * ld + n));
}

// Four 8x8 bf16 matrices to shared memory (the inverse of ldsm_x4): lane l gives the address of
// row l % 8 of matrix l / 8; register i holds matrix i in the fragment layout above.
__device__ __forceinline__ void stsm_x4(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1,%2,%3,%4};\n" ::"r"(addr), "r"(r0), "r"(r1),
                 "r"(r2), "r"(r3)
                 : "memory");
}
// The same with each matrix stored transposed: lane l addresses row l % 8 of the stored
// (transposed) matrix l / 8.
__device__ __forceinline__ void stsm_x4_t(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1,%2,%3,%4};\n" ::"r"(addr), "r"(r0),
                 "r"(r1), "r"(r2), "r"(r3)
                 : "memory");
}

// C fragments of a warp's 16 rows x (8 * nt2 * 2) columns, stored transposed into a row-major
// [column][row] tile (ld elements per stored row) at stored columns m0 .. m0 + 15: tile j holds
// columns 8j .. 8j + 7; two tiles per stmatrix
template <int NT>
__device__ __forceinline__ void store_frags_t(__nv_bfloat16 *base, int ld, int m0, const float (*y)[4], int lane) {
    const int mi = lane >> 3, r = lane & 7;
#pragma unroll
    for (int p = 0; p < NT / 2; ++p) {
        const int row = 8 * (2 * p + (mi >> 1)) + r;   // stored row = original column
        stsm_x4_t(smem_u32(base + row * ld + m0 + 8 * (mi & 1)), pack_bf16(y[2 * p][0], y[2 * p][1]),
                  pack_bf16(y[2 * p][2], y[2 * p][3]), pack_bf16(y[2 * p + 1][0], y[2 * p + 1][1]),
                  pack_bf16(y[2 * p + 1][2], y[2 * p + 1][3]));
    }
}

// ---- swizzled [rows][128] bf16 tiles (256-byte rows, no padding): the 16-byte chunk c of
//      row r is stored at chunk c ^ (r & 7), so the eight rows of an 8x8 ldmatrix always hit
//      eight different bank groups
__device__ __forceinline__ int swz128(int r, int c) {   // element offset of (row r, column c)
    return r * 128 + ((((c >> 3) ^ (r & 7))) << 3) + (c & 7);
}

// load_a on a swizzled [m][k] tile
__device__ __forceinline__ void load_a_swz(uint32_t (&a)[4], const __nv_bfloat16 *base, int m0, int k0, int lane) {
    const int r = m0 + (lane & 15), k = k0 + (lane >> 4) * 8;
    ldsm_x4(a, smem_u32(base + swz128(r, k)));
}

// load_b_nk on a swizzled [n][k] tile
__device__ __forceinline__ void load_b_nk_swz(uint32_t (&b)[4], const __nv_bfloat16 *base, int n0, int k0, int lane) {
    const int n = n0 + (lane & 7) + ((lane >> 4) << 3), k = k0 + ((lane >> 3) & 1) * 8;
    ldsm_x4(b, smem_u32(base + swz128(n, k)));
}

// load_b_kn on a swizzled [k][n] tile
__device__ __forceinline__ void load_b_kn_swz(uint32_t (&b)[4], const __nv_bfloat16 *base, int n0, int k0, int lane) {
    const int k = k0 + (lane & 7) + (((lane >> 3) & 1) << 3), n = n0 + ((lane >> 4) << 3);
    ldsm_x4_t(b, smem_u32(base + swz128(k, n)));
}

// ---- mbarrier + bulk copy (global -> shared through the TMA engine) ------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;\n" ::); }

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(bytes));
}

// Bounded wait on phase `parity`.  Returns false if the limit ran out (the caller records it).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t limit = 1u << 26) {
    const uint32_t a = smem_u32(bar);
    for (uint32_t it = 0; it < limit; ++it) {
        uint32_t done;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(done)
            : "r"(a), "r"(parity));
        if (done) return true;
    }
    return false;
}

// 1-D bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned) into shared
// memory, completing on `bar` as transaction bytes.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// 1-D bulk copy of `bytes` from shared memory to global memory (same alignment rules), in
// the thread's current bulk group.  The writes of other threads to the source must be made
// visible to the copy engine first (fence_proxy_async + a barrier).
__device__ __forceinline__ void bulk_s2g(void *dst, const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;\n" ::"l"(dst), "r"(smem_u32(src)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;\n" ::: "memory"); }
// Wait until at most N of this thread's bulk groups still read their shared-memory source.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;\n" ::"n"(N) : "memory");
}
// Wait until at most N of this thread's bulk groups are incomplete.
template <int N>
__device__ __forceinline__ void bulk_wait() {
    asm volatile("cp.async.bulk.wait_group %0;\n" ::"n"(N) : "memory");
}
// Order this thread's generic-proxy shared-memory writes before later bulk copies.
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }

// Tiled TMA load of a 3-D box (coordinates innermost first) into shared memory, completing
// on `bar` as transaction bytes.  c0 * element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int c0, int c1, int c2, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];\n" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Host: tensor map over a [rows, H, inner] token-major tensor (inner = channels, contiguous),
// box = [box_rows tokens, 1 head, inner channels]; elem_bytes 2 (bf16) or 4 (fp32).
cudaError_t make_token_tile_map(CUtensorMap *map, const void *base, int elem_bytes, int inner, int H,
                                long long rows, int box_rows);

}  // namespace carve
