// efla_mma_sync.cuh -- warp-level bf16 tensor-core tiles (mma.sync m16n8k16, fp32
// accumulation) with operands read from padded shared memory by ldmatrix, and cp.async
// tile loads.  Used by the auxiliary kernels (the backward's chunk kernels, the segmented
// scan's correction); the forward's chunk products run on tcgen05 (sm100.cuh).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace efla {
namespace mmas {

using bf16 = __nv_bfloat16;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(smem_addr(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(smem_addr(p)));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// acc (16 rows from m0, 8 NT columns from n0) += A(., K) B(K, .), bf16 operands in shared memory.
//   A: AT = false, A[m][k] = a[m * lda + k];  AT = true, A[m][k] = a[k * lda + m].
//   B: BT = false, B[k][n] = b[n * ldb + k];  BT = true, B[k][n] = b[k * ldb + n].
// ldmatrix (with .trans for the transposed storages) delivers the mma fragments directly.
template <int NT, bool AT, bool BT>
__device__ __forceinline__ void warp_mma(float (&acc)[NT][4], const bf16* a, int lda, const bf16* b, int ldb,
                                         int m0, int n0, int K, int lane) {
    static_assert(NT % 2 == 0, "n tiles come in pairs");
    const int r = lane & 7, j = lane >> 3;
    for (int k0 = 0; k0 < K; k0 += 16) {
        uint32_t af[4];
        if constexpr (!AT) ldsm_x4(af, a + (m0 + r + (j & 1) * 8) * lda + k0 + (j >> 1) * 8);
        else ldsm_x4_t(af, a + (k0 + r + (j >> 1) * 8) * lda + m0 + (j & 1) * 8);
#pragma unroll
        for (int nt = 0; nt < NT; nt += 2) {
            uint32_t bf[4];
            const int nb = n0 + 8 * nt;
            if constexpr (!BT) ldsm_x4(bf, b + (nb + r + (j >> 1) * 8) * ldb + k0 + (j & 1) * 8);
            else ldsm_x4_t(bf, b + (k0 + r + (j & 1) * 8) * ldb + nb + (j >> 1) * 8);
            mma16816(acc[nt], af, bf[0], bf[1]);
            mma16816(acc[nt + 1], af, bf[2], bf[3]);
        }
    }
}

template <int NT>
__device__ __forceinline__ void zero_acc(float (&acc)[NT][4]) {
#pragma unroll
    for (int i = 0; i < NT; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
}

// Visit the accumulator elements: f(row, col, value&) with row = m0 + g (+8), col = n0 + 8 nt + 2 t (+1).
template <int NT, typename F>
__device__ __forceinline__ void for_acc(float (&acc)[NT][4], int m0, int n0, int lane, F f) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) f(m0 + g + (e >> 1) * 8, n0 + 8 * nt + 2 * t + (e & 1), acc[nt][e]);
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// rows x cols bf16 from global (row stride gstride elements, rows past nvalid zero) into
// shared memory (row stride lds), 16-byte pieces spread over nthreads threads.
__device__ __forceinline__ void load_tile(bf16* dst, int lds, const bf16* src, long gstride, int rows, int cols,
                                          int nvalid, int tid, int nthreads) {
    const int per_row = cols / 8;
    for (int e = tid; e < rows * per_row; e += nthreads) {
        const int rr = e / per_row, cc = (e % per_row) * 8;
        bf16* d = dst + rr * lds + cc;
        if (rr < nvalid) cp_async16(d, src + rr * gstride + cc);
        else *reinterpret_cast<uint4*>(d) = make_uint4(0u, 0u, 0u, 0u);
    }
}

}  // namespace mmas
}  // namespace efla
