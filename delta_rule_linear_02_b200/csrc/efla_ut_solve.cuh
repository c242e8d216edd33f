// efla_ut_solve.cuh -- the UT transform of one 64-token chunk in fp32 shared memory.
//
// Exact Flow Linear Attention, Section 3.3 applies the UT transform to the chunk
// recurrence.  Inside a chunk (row convention, S is d_k x d_v) the writes
// delta_r = alpha_r (v_r - S_{r-1}^T k_r) satisfy (I + A) Delta = diag(alpha) (V - K S)
// with A = strictly-lower(diag(alpha) K K^T), so Delta = T (V - K S) for
//     T = (I + A)^{-1} diag(alpha).
// (I + A) is unit lower triangular.  Its inverse is built by block doubling:
//   16x16 diagonal blocks by forward substitution (one thread per column), then
//   [[X11, 0], [L21, X22]]^{-1}-style merges X21 = -X22 L21 X11 at 32 and at 64.
#pragma once

namespace efla {

// A: 64x64 fp32, strictly lower part used (row stride LD).  alpha[64].
// X: output 64x64 (row stride LD) = T.  Y: 64x64 scratch (row stride LD).
// Called by all NT threads of the block; contains __syncthreads().
template <int NT>
__device__ __forceinline__ void ut_inverse64(const float* __restrict__ A,
                                             const float* __restrict__ alpha,
                                             float* __restrict__ X, float* __restrict__ Y, int LD,
                                             int tid) {
    // clear the strictly-upper off-diagonal 16-blocks (never written below)
    for (int e = tid; e < 64 * 64; e += NT) {
        const int i = e >> 6, c = e & 63;
        if ((c >> 4) > (i >> 4)) X[i * LD + c] = 0.f;
    }
    // (1) the four 16x16 diagonal blocks: column c of block b by thread 16b + c
    if (tid < 64) {
        const int b = tid >> 4, c = tid & 15;
        const float* Ab = A + (16 * b) * LD + 16 * b;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = (i == c) ? 1.f : 0.f;
#pragma unroll
        for (int i = 1; i < 16; ++i) {
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < i; ++j) s = fmaf(Ab[i * LD + j], x[j], s);
            if (i > c) x[i] = -s;
        }
        float* Xb = X + (16 * b) * LD + 16 * b + c;
#pragma unroll
        for (int i = 0; i < 16; ++i) Xb[i * LD] = x[i];
    }
    __syncthreads();
    // (2) merge to 32x32 blocks s = 0, 1:  X21 = -X22 (A21 X11)
    for (int e = tid; e < 512; e += NT) {
        const int s = e >> 8, i = (e >> 4) & 15, c = e & 15;
        const int r0 = 32 * s + 16, c0 = 32 * s;
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) acc = fmaf(A[(r0 + i) * LD + c0 + j], X[(c0 + j) * LD + c0 + c], acc);
        Y[(r0 + i) * LD + c0 + c] = acc;
    }
    __syncthreads();
    for (int e = tid; e < 512; e += NT) {
        const int s = e >> 8, i = (e >> 4) & 15, c = e & 15;
        const int r0 = 32 * s + 16, c0 = 32 * s;
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) acc = fmaf(X[(r0 + i) * LD + r0 + j], Y[(r0 + j) * LD + c0 + c], acc);
        X[(r0 + i) * LD + c0 + c] = -acc;
    }
    __syncthreads();
    // (3) merge to 64x64:  X21 = -X22 (A21 X11) with 32x32 blocks
    for (int e = tid; e < 1024; e += NT) {
        const int i = e >> 5, c = e & 31;
        float acc = 0.f;
#pragma unroll 8
        for (int j = c & ~15; j < 32; ++j) acc = fmaf(A[(32 + i) * LD + j], X[j * LD + c], acc);
        Y[(32 + i) * LD + c] = acc;
    }
    __syncthreads();
    for (int e = tid; e < 1024; e += NT) {
        const int i = e >> 5, c = e & 31;
        float acc = 0.f;
#pragma unroll 8
        for (int j = 0; j <= (i | 15); ++j) acc = fmaf(X[(32 + i) * LD + 32 + j], Y[(32 + j) * LD + c], acc);
        X[(32 + i) * LD + c] = -acc;
    }
    __syncthreads();
    // (4) T = X diag(alpha)
    for (int e = tid; e < 64 * 64; e += NT) {
        const int i = e >> 6, c = e & 63;
        X[i * LD + c] *= alpha[c];
    }
    __syncthreads();
}

}  // namespace efla
