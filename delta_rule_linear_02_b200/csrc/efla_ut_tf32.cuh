// efla_ut_tf32.cuh -- the UT transform of one 64-token chunk: X = (I + A)^{-1}.
//
// Exact Flow Linear Attention, Section 3.3 applies the UT transform to the chunk
// recurrence: with A = strictly-lower(diag(alpha) K K^T), the chunk's rank-1 writes are
// Delta = T (V - K S) for T = (I + A)^{-1} diag(alpha) (row convention).  This header
// builds X = (I + A)^{-1}; the caller applies diag(alpha).
#pragma once

#include <stdint.h>

#include "sm100.cuh"

namespace efla {
namespace ut {

using sm100::bar_sync;
constexpr int LDX = 68;          // fp32 row stride of At and X (16-byte aligned rows)

// X = (I + A)^{-1} for the 64 x 64 strictly-lower A, by NT >= 128 threads (ptid, named barrier NB),
// with
//   At[j * LDX + i] = A[i][j] (i > j)  -- only that part of At is read.
// X's strictly-upper 16 x 16 blocks are zero from the start of the kernel.
//   (1) 16 x 16 diagonal blocks by forward substitution, one thread per column (fp32);
//   (2) 32 x 32 merges X21 = -X22 (A21 X11);  (3) the 64 x 64 merge the same way.
// In (2) and (3) a warp forms the Y = A21 X11 it needs as Y^T = X11^T A21^T, whose
// accumulators are already the B fragments of X21 = -X22 Y: Y never goes through shared
// memory, and each merge level is one barrier phase.
// The merge products run as warp-level TF32 tensor-core tiles (m16n8k8, fp32
// accumulation): operands are read from shared memory once per warp fragment instead of
// once per output, which is what bounds a CUDA-core solve.  TF32 operands (10-bit
// mantissa, round-to-nearest) are finer than the bf16 rounding T receives afterwards.
// Tiles that multiply a structural zero block of a triangular factor are skipped.

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// D += A(16x8, row) B(8x8, col), TF32 in, fp32 accumulate
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Store a 16 x 16 fragment (times `scale`) at dst[r * LDX + c].
__device__ __forceinline__ void warp_st16x16(float* __restrict__ dst, const float (&c)[2][4], float scale, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        *reinterpret_cast<float2*>(dst + g * LDX + 8 * nt + 2 * t) = make_float2(scale * c[nt][0], scale * c[nt][1]);
        *reinterpret_cast<float2*>(dst + (g + 8) * LDX + 8 * nt + 2 * t) = make_float2(scale * c[nt][2], scale * c[nt][3]);
    }
}

// One warp: Y^T = X11^T A21^T for the 8-column tiles j < NTILE of Y^T (columns 8 j .. 8 j + 7
// of Y^T are rows of Y), Y^T rows n = 0..15, over k-steps [k0, k1):
//   X11^T(n, m) = x11[m * LDX + n],   A21^T(m, k) = a21t[m * LDX + k].
// Within a k-step the MMA's k slots t and t + 4 take columns k = 2t and 2t + 1 of the
// step (the same permutation for A and B leaves the sum unchanged).  With the row stride
// of 68 floats (4 mod 32 banks) the k-strided loads then hit bank 8t + g + const, all 32
// lanes distinct, and a row-strided A operand is read as float2 pairs (warp_mm_yreg).  The
// permutation also makes the accumulator of tile j (rows n = g, g + 8, columns 2t,
// 2t + 1) exactly the B fragment of Y for k-step j of a following product.
template <int NTILE>
__device__ __forceinline__ void warp_yt(float (&yt)[NTILE][4], const float* __restrict__ x11,
                                        const float* __restrict__ a21t, int k0, int k1, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int j = 0; j < NTILE; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) yt[j][e] = 0.f;
    for (int ks = k0; ks < k1; ++ks) {
        const int k = 8 * ks + 2 * t;
        uint32_t a[4];
        a[0] = to_tf32(x11[k * LDX + g]);
        a[1] = to_tf32(x11[k * LDX + g + 8]);
        a[2] = to_tf32(x11[(k + 1) * LDX + g]);
        a[3] = to_tf32(x11[(k + 1) * LDX + g + 8]);
#pragma unroll
        for (int j = 0; j < NTILE; ++j) {
            uint32_t b[2];
            b[0] = to_tf32(a21t[k * LDX + 8 * j + g]);
            b[1] = to_tf32(a21t[(k + 1) * LDX + 8 * j + g]);
            mma_tf32(yt[j], a, b);
        }
    }
}

// One warp: C(16 x 16) = sum over k-steps [0, KS) of A(16 x 8) Y(8 x 16), A(r, k) = a_base[r * LDX + k]
// (float2 pairs), Y from the Y^T accumulators of warp_yt (no shared-memory round trip).
template <int KS>
__device__ __forceinline__ void warp_mm_yreg(float (&c)[2][4], const float* __restrict__ a_base,
                                             const float (&yt)[KS][4], int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) c[nt][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
        const int k = 8 * ks + 2 * t;
        const float2 lo = *reinterpret_cast<const float2*>(a_base + g * LDX + k);
        const float2 hi = *reinterpret_cast<const float2*>(a_base + (g + 8) * LDX + k);
        uint32_t a[4];
        a[0] = to_tf32(lo.x);
        a[1] = to_tf32(hi.x);
        a[2] = to_tf32(lo.y);
        a[3] = to_tf32(hi.y);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            uint32_t b[2];
            b[0] = to_tf32(yt[ks][2 * nt]);
            b[1] = to_tf32(yt[ks][2 * nt + 1]);
            mma_tf32(c[nt], a, b);
        }
    }
}

template <int NB, int NT>
__device__ __forceinline__ void ut_solve(float* __restrict__ At, float* __restrict__ X, int ptid) {
    static_assert(NT >= 128, "the solve uses four warps");
    const int pw = ptid >> 5, lane = ptid & 31;
    if (ptid < 64) {   // (1) column c of diagonal block b; A rows read four at a time
        const int b = ptid >> 4, c = ptid & 15;
        const float* Ab = At + (16 * b) * LDX + 16 * b;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = (i == c) ? 1.f : 0.f;
#pragma unroll
        for (int j = 0; j < 15; ++j) {
            const float xj = x[j];
#pragma unroll
            for (int m = (j + 1) >> 2; m < 4; ++m) {
                const float4 a = *reinterpret_cast<const float4*>(Ab + j * LDX + 4 * m);
                const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (4 * m + e > j) x[4 * m + e] = fmaf(-av[e], xj, x[4 * m + e]);
            }
        }
        float* Xb = X + (16 * b) * LDX + 16 * b + c;
#pragma unroll
        for (int i = 0; i < 16; ++i) Xb[i * LDX] = x[i];
    }
    bar_sync(NB, NT);
    if (pw < 2) {      // (2) super-block pw: Y = A21 X11 (as Y^T, in registers), X21 = -X22 Y
        const int r0 = 32 * pw + 16, c0 = 32 * pw;
        float yt[2][4], acc[2][4];
        warp_yt<2>(yt, X + c0 * LDX + c0, At + c0 * LDX + r0, 0, 2, lane);
        warp_mm_yreg<2>(acc, X + r0 * LDX + r0, yt, lane);
        warp_st16x16(X + r0 * LDX + c0, acc, -1.f, lane);
    }
    bar_sync(NB, NT);
    if (pw < 4) {      // (3) tile (wr, wc) of the 64 x 64 merge: X21 = -X22 (A21 X11), 32 x 32 blocks;
                       //     X11[m][n] = 0 for m < 16 wc, X22[i][k] = 0 for k > 16 wr + 15
        const int wr = pw >> 1, wc = pw & 1;
        float acc[2][4];
        if (wr == 0) {
            float yt[2][4];
            warp_yt<2>(yt, X + 16 * wc, At + 32, 2 * wc, 4, lane);
            warp_mm_yreg<2>(acc, X + 32 * LDX + 32, yt, lane);
        } else {
            float yt[4][4];
            warp_yt<4>(yt, X + 16 * wc, At + 32, 2 * wc, 4, lane);
            warp_mm_yreg<4>(acc, X + 48 * LDX + 32, yt, lane);
        }
        warp_st16x16(X + (32 + 16 * wr) * LDX + 16 * wc, acc, -1.f, lane);
    }
    bar_sync(NB, NT);
}

}  // namespace ut
}  // namespace efla
