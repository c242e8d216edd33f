// efla_chunk_simt.cu -- chunkwise EFLA forward on fp32 CUDA cores.
//
// The fp32 path: fp32 inputs must match the fp64 oracle to 1e-4, which TF32 tensor-core
// operands cannot promise, so every product here is an FFMA.  One CTA owns one (b, h)
// stream and one 64-column slice of d_v; the state slice S (d_k x 64, fp32) stays in
// shared memory across the whole sequence.
//
// Per 64-token chunk (Exact Flow Linear Attention, Section 3.3; row convention):
//   alpha_r = gate(beta_r, ||k_r||^2)                      (Section 3.2 / 3.4)
//   A = strictly-lower(diag(alpha) K K^T),  T = (I + A)^{-1} diag(alpha)   (UT transform)
//   X = V - K S,   Delta = T X                             (the chunk's rank-1 writes)
//   O = Q S + (Q K^T, lower incl. diagonal) Delta          (read-out after each write)
//   S <- S + K^T Delta
// Tokens past T are zero-filled (k = 0, beta = 0: alpha = 0, an exact no-op).
//
// Gated flow (Section 3.4, Gated EFLA; per-token log-decay g, cumulative G_r = g_0 + .. + g_r
// inside the chunk, Gam_r = e^{G_r}, write gate abar_r):
//   A[r][s] = alpha_r (Gam_r / Gam_s) k_r . k_s (s < r),  X = (I + A)^{-1}
//   Delta = X (diag(abar) V - diag(alpha Gam) K S)
//   O = diag(Gam) Q S + (Q K^T (.) Gam_r / Gam_s, lower incl. diagonal) Delta
//   S <- Gam_last S + K^T diag(Gam_last / Gam) Delta
#include "efla_common.cuh"
#include "efla_kernels.h"
#include "efla_ut_solve.cuh"

namespace efla {

namespace {
constexpr int kC = 64;          // chunk length
constexpr int kNT = 256;        // threads
constexpr int kLD = 65;         // row stride of 64-wide fp32 tiles (conflict-free columns)

// acc[i][j] += sum_kk A(ty + 16 i, kk) * B(kk, tx + 16 j)
//   AT: A stored transposed (A(r, kk) = A[kk * lda + r]);  BT: B(kk, c) = B[c * ldb + kk]
template <int MT, int KD, bool AT, bool BT>
__device__ __forceinline__ void mm(float (&acc)[MT][4], const float* __restrict__ A, int lda,
                                   const float* __restrict__ B, int ldb, int ty, int tx) {
#pragma unroll 4
    for (int kk = 0; kk < KD; ++kk) {
        float a[MT], b[4];
#pragma unroll
        for (int i = 0; i < MT; ++i) a[i] = AT ? A[kk * lda + ty + 16 * i] : A[(ty + 16 * i) * lda + kk];
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = BT ? B[(tx + 16 * j) * ldb + kk] : B[kk * ldb + tx + 16 * j];
#pragma unroll
        for (int i = 0; i < MT; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
}

template <int MT>
__device__ __forceinline__ void zero(float (&acc)[MT][4]) {
#pragma unroll
    for (int i = 0; i < MT; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
}

template <int D>
struct SimtSmem {
    static constexpr int kKD = D + 1;                 // K, Q row stride
    static constexpr int kK = 0;
    static constexpr int kQ = kK + kC * kKD;
    static constexpr int kV = kQ + kC * kKD;
    static constexpr int kS = kV + kC * kLD;          // D x 64 state slice
    static constexpr int kT = kS + D * kLD;
    static constexpr int kP = kT + kC * kLD;
    static constexpr int kA = kP + kC * kLD;          // A, then Delta
    static constexpr int kX = kA + kC * kLD;          // solve scratch, then X = V - K S
    static constexpr int kAlpha = kX + kC * kLD;
    static constexpr int kBeta = kAlpha + kC;
    static constexpr int kAbar = kBeta + kC;          // gated flow: write gate, cumulative log-decay, ones
    static constexpr int kGcum = kAbar + kC;
    static constexpr int kOnes = kGcum + kC;
    static constexpr int kFloats = kOnes + kC;
    static constexpr size_t kBytes = sizeof(float) * kFloats;
};

template <typename Tin, int D, bool kGated = false>
__global__ void __launch_bounds__(kNT, 1) chunk_simt_kernel(const Tin* __restrict__ q,
                                                            const Tin* __restrict__ k,
                                                            const Tin* __restrict__ v,
                                                            const Tin* __restrict__ beta,
                                                            const float* __restrict__ S0,
                                                            Tin* __restrict__ o,
                                                            float* __restrict__ S_T, Seqs seqs, int Tdim,
                                                            int rule, const float* __restrict__ gdec = nullptr) {
    using L = SimtSmem<D>;
    constexpr int NSL = D / 64;                 // d_v slices per stream
    extern __shared__ float smem[];
    float* Ks = smem + L::kK;
    float* Qs = smem + L::kQ;
    float* Vs = smem + L::kV;
    float* Ss = smem + L::kS;
    float* Ts = smem + L::kT;
    float* Ps = smem + L::kP;
    float* As = smem + L::kA;
    float* Xs = smem + L::kX;
    float* al = smem + L::kAlpha;
    float* bt = smem + L::kBeta;
    float* ab = smem + L::kAbar;
    float* gc = smem + L::kGcum;
    float* ones = smem + L::kOnes;

    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    if constexpr (kGated) {
        if (tid < kC) ones[tid] = 1.f;
    }
    const long bh = blockIdx.x / NSL;           // stream (state index)
    const int col0 = (blockIdx.x % NSL) * 64;   // first d_v column of this slice
    const StreamJob jb = seqs.job(bh);
    const int T = jb.len;

    // initial state slice
    for (int e = tid; e < D * 64; e += kNT) {
        const int i = e >> 6, j = e & 63;
        Ss[i * kLD + j] = S0 ? S0[(bh * D + i) * D + col0 + j] : 0.f;
    }

    const long base = (long)jb.z * Tdim + jb.y0;  // first token row of this stream
    for (int r0 = 0; r0 < T; r0 += kC) {
        const int n = min(kC, T - r0);
        __syncthreads();                        // previous chunk is done with K, Q, V
        // ---- load the chunk (zero rows past T)
        for (int e = tid; e < kC * (D / 4); e += kNT) {
            const int r = e / (D / 4), c4 = (e % (D / 4)) * 4;
            float4 kk = make_float4(0.f, 0.f, 0.f, 0.f), qq = kk;
            if (r < n) {
                kk = load4(k + (base + r0 + r) * D + c4);
                qq = load4(q + (base + r0 + r) * D + c4);
            }
            float* kd = Ks + r * L::kKD + c4;
            float* qd = Qs + r * L::kKD + c4;
            kd[0] = kk.x; kd[1] = kk.y; kd[2] = kk.z; kd[3] = kk.w;
            qd[0] = qq.x; qd[1] = qq.y; qd[2] = qq.z; qd[3] = qq.w;
        }
        for (int e = tid; e < kC * 16; e += kNT) {
            const int r = e >> 4, c4 = (e & 15) * 4;
            float4 vv = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r < n) vv = load4(v + (base + r0 + r) * D + col0 + c4);
            float* vd = Vs + r * kLD + c4;
            vd[0] = vv.x; vd[1] = vv.y; vd[2] = vv.z; vd[3] = vv.w;
        }
        if (tid < kC) bt[tid] = (tid < n) ? Elem<Tin>::to_f(beta[base + r0 + tid]) : 0.f;
        if constexpr (kGated) {
            if (tid < kC) gc[tid] = (tid < n) ? gdec[base + r0 + tid] : 0.f;
        }
        __syncthreads();
        if constexpr (kGated) {   // log-decay of token r -> cumulative G_r (one warp, shuffle scan)
            if (tid < 32) {
                const float a0 = gc[2 * tid], a1 = gc[2 * tid + 1];
                float run = a0 + a1;                // inclusive scan of the pair sums
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, run, off);
                    if (tid >= off) run += y;
                }
                float before = __shfl_up_sync(0xffffffffu, run, 1);
                if (tid == 0) before = 0.f;
                ab[2 * tid] = before + a0;          // staged in ab, moved to gc below
                ab[2 * tid + 1] = (before + a0) + a1;
            }
            __syncthreads();
            // ab holds G_r for now; the raw g_r stays in gc until the write gate is formed
        }

        // ---- gate: lambda_r = ||k_r||^2 (4 threads per row), alpha_r
        {
            const int r = tid >> 2, part = tid & 3;
            float lam = 0.f;
            for (int d = part; d < D; d += 4) lam = fmaf(Ks[r * L::kKD + d], Ks[r * L::kKD + d], lam);
            lam += __shfl_xor_sync(0xffffffffu, lam, 1);
            lam += __shfl_xor_sync(0xffffffffu, lam, 2);
            if constexpr (kGated) {
                const float graw = gc[r], gcum = ab[r];
                __syncwarp();
                if (part == 0) {
                    al[r] = rule_alpha(rule, bt[r], lam);
                    ab[r] = rule_write_gate(rule, bt[r], lam, graw);
                    gc[r] = gcum;
                }
            } else {
                if (part == 0) al[r] = rule_alpha(rule, bt[r], lam);
            }
        }
        // ---- G = K K^T and P = Q K^T
        float g[4][4], p[4][4];
        zero(g);
        zero(p);
        mm<4, D, false, true>(g, Ks, L::kKD, Ks, L::kKD, ty, tx);
        mm<4, D, false, true>(p, Qs, L::kKD, Ks, L::kKD, ty, tx);
        __syncthreads();                        // alpha visible
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = ty + 16 * i;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = tx + 16 * j;
                if constexpr (kGated) {
                    const float dcy = (c <= r) ? expf(gc[r] - gc[c]) : 0.f;   // Gam_r / Gam_c
                    As[r * kLD + c] = (c < r) ? al[r] * dcy * g[i][j] : 0.f;
                    Ps[r * kLD + c] = (c <= r) ? dcy * p[i][j] : 0.f;
                } else {
                    As[r * kLD + c] = (c < r) ? al[r] * g[i][j] : 0.f;
                    Ps[r * kLD + c] = (c <= r) ? p[i][j] : 0.f;
                }
            }
        }
        __syncthreads();
        // ---- T = (I + A)^{-1} diag(alpha)   (gated: T = (I + A)^{-1}, the diagonals go on the right side)
        ut_inverse64<kNT>(As, kGated ? ones : al, Ts, Xs, kLD, tid);
        // ---- X = V - K S   (gated: diag(abar) V - diag(alpha Gam) K S)
        {
            float x[4][4];
            zero(x);
            mm<4, D, false, false>(x, Ks, L::kKD, Ss, kLD, ty, tx);
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int r = ty + 16 * i, c = tx + 16 * j;
                    if constexpr (kGated)
                        Xs[r * kLD + c] = ab[r] * Vs[r * kLD + c] - al[r] * expf(gc[r]) * x[i][j];
                    else
                        Xs[r * kLD + c] = Vs[r * kLD + c] - x[i][j];
                }
        }
        __syncthreads();
        // ---- Delta = T X  (into As)
        {
            float d[4][4];
            zero(d);
            mm<4, kC, false, false>(d, Ts, kLD, Xs, kLD, ty, tx);
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) As[(ty + 16 * i) * kLD + tx + 16 * j] = d[i][j];
        }
        __syncthreads();
        // ---- O = Q S + P Delta   (gated: diag(Gam) Q S + P Delta)
        {
            float oo[4][4];
            zero(oo);
            mm<4, D, false, false>(oo, Qs, L::kKD, Ss, kLD, ty, tx);
            if constexpr (kGated) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float gm = expf(gc[ty + 16 * i]);
#pragma unroll
                    for (int j = 0; j < 4; ++j) oo[i][j] *= gm;
                }
            }
            mm<4, kC, false, false>(oo, Ps, kLD, As, kLD, ty, tx);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = ty + 16 * i;
                if (r < n) {
                    Tin* orow = o + (base + r0 + r) * D + col0;
#pragma unroll
                    for (int j = 0; j < 4; ++j) orow[tx + 16 * j] = Elem<Tin>::from_f(oo[i][j]);
                }
            }
        }
        __syncthreads();                        // every read of the old S is done
        if constexpr (kGated) {                 // Delta rows scaled by Gam_last / Gam_r
            const float glast = gc[kC - 1];
            for (int e = tid; e < kC * 64; e += kNT) {
                const int r = e >> 6, c = e & 63;
                As[r * kLD + c] *= expf(glast - gc[r]);
            }
            __syncthreads();
        }
        // ---- S <- S + K^T Delta   (gated: Gam_last S + K^T diag(Gam_last / Gam) Delta)
        {
            float s[D / 16][4];
            zero(s);
            mm<D / 16, kC, true, false>(s, Ks, L::kKD, As, kLD, ty, tx);
            float keep = 1.f;
            if constexpr (kGated) keep = expf(gc[kC - 1]);
#pragma unroll
            for (int i = 0; i < D / 16; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float& st = Ss[(ty + 16 * i) * kLD + tx + 16 * j];
                    if constexpr (kGated)
                        st = fmaf(keep, st, s[i][j]);
                    else
                        st += s[i][j];
                }
        }
    }
    __syncthreads();
    if (S_T) {
        for (int e = tid; e < D * 64; e += kNT) {
            const int i = e >> 6, j = e & 63;
            S_T[(bh * D + i) * D + col0 + j] = Ss[i * kLD + j];
        }
    }
}

template <typename Tin, int D, bool kGated>
cudaError_t launch_t(const void* q, const void* k, const void* v, const void* beta, const float* S0,
                     void* o, float* S_T, const Seqs& seqs, long nstreams, int Tdim, int rule, const float* g,
                     cudaStream_t stream) {
    using L = SimtSmem<D>;
    auto kern = chunk_simt_kernel<Tin, D, kGated>;
    static std::atomic<uint64_t> smem_set{0};
    cudaError_t err = set_smem_limit_once(kern, (int)L::kBytes, smem_set);
    if (err != cudaSuccess) return err;
    kern<<<(unsigned)(nstreams * (D / 64)), kNT, L::kBytes, stream>>>(
        (const Tin*)q, (const Tin*)k, (const Tin*)v, (const Tin*)beta, S0, (Tin*)o, S_T, seqs, Tdim, rule, g);
    return cudaGetLastError();
}

template <typename Tin, int D>
cudaError_t launch_g(const void* q, const void* k, const void* v, const void* beta, const float* S0,
                     void* o, float* S_T, const Seqs& seqs, long nstreams, int Tdim, int rule, const float* g,
                     cudaStream_t stream) {
    return g ? launch_t<Tin, D, true>(q, k, v, beta, S0, o, S_T, seqs, nstreams, Tdim, rule, g, stream)
             : launch_t<Tin, D, false>(q, k, v, beta, S0, o, S_T, seqs, nstreams, Tdim, rule, nullptr, stream);
}
}  // namespace

cudaError_t launch_chunk_simt(const void* q, const void* k, const void* v, const void* beta,
                              const float* S0, void* o, float* S_T, const Seqs& seqs, long nstreams, int Tdim,
                              int D, bool bf16, int rule, cudaStream_t stream, const float* g) {
    if (bf16)
        return D == 128 ? launch_g<__nv_bfloat16, 128>(q, k, v, beta, S0, o, S_T, seqs, nstreams, Tdim, rule, g, stream)
                        : launch_g<__nv_bfloat16, 64>(q, k, v, beta, S0, o, S_T, seqs, nstreams, Tdim, rule, g, stream);
    return D == 128 ? launch_g<float, 128>(q, k, v, beta, S0, o, S_T, seqs, nstreams, Tdim, rule, g, stream)
                    : launch_g<float, 64>(q, k, v, beta, S0, o, S_T, seqs, nstreams, Tdim, rule, g, stream);
}

}  // namespace efla
