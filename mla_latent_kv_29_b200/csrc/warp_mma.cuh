// Warp-level bf16 tensor-core tiles (mma.sync m16n8k16, fp32 accumulate) for
// the small, weight-bandwidth-bound GEMMs around the attention: the query
// absorption, the value up-projection and the cache-append projection. Their
// M is the number of new tokens (tens), far below a tcgen05 tile.
//
// Shared-memory operands are row-major with a row stride of (columns + 8)
// elements, which keeps ldmatrix reads free of bank conflicts.
#pragma once

#include <stdint.h>

namespace mla {
namespace wmma16 {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

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

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// One warp accumulates a 16 x 64 tile: acc[nt][.] += A[r0:r0+16, k0:k0+16] * B[k0:k0+16, c0 + 8nt : +8]
// for nt < 8. A is row-major [rows][lda]; B is either row-major [k][ldb]
// (KN layout) or row-major [n][ldb] with k contiguous (NK layout).
template <bool kBisNK>
__device__ __forceinline__ void warp_tile_k16(float (&acc)[8][4], const uint16_t* As, int lda, int r0,
                                              const uint16_t* Bs, int ldb, int c0, int k0) {
    const int lane = threadIdx.x & 31;
    uint32_t a[4];
    ldsm_x4(smem_u32(As + (r0 + (lane & 15)) * lda + k0 + 8 * (lane >> 4)), a);
    const int mi = lane >> 3, ri = lane & 7;  // which 8x8 matrix this lane addresses, and its row
#pragma unroll
    for (int np = 0; np < 4; ++np) {  // pairs of n-tiles
        uint32_t b[4];
        const int n = c0 + 16 * np + 8 * (mi >> 1);
        const int k = k0 + 8 * (mi & 1);
        if (kBisNK) {
            ldsm_x4(smem_u32(Bs + (n + ri) * ldb + k), b);
        } else {
            ldsm_x4_trans(smem_u32(Bs + (k + ri) * ldb + n), b);
        }
        mma16816(acc[2 * np], a, b[0], b[1]);
        mma16816(acc[2 * np + 1], a, b[2], b[3]);
    }
}

}  // namespace wmma16
}  // namespace mla
