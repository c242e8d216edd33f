// efla_bwd.cu -- reverse-mode pass of the exact-flow recurrence (training), fp32 state.
//
// Exact Flow Linear Attention, Section 3.2 (the rank-1 update with the exact-flow gate),
// differentiated for training (Section 4.6 reports training throughput; the pages print
// no backward formulas, so this is the chain rule of the recurrence).  Row convention,
// S is d_k x d_v, with r_t = S_{t-1}^T k_t - v_t:
//     S_t = S_{t-1} - alpha_t k_t r_t^T,     o_t = S_t^T q_t.
// Reverse sweep with G = dL/dS_t, from G = dS_T:
//     G += q_t dO_t^T;   dq_t = S_t dO_t;   g = G^T k_t;   dv_t = alpha_t g;
//     dalpha_t = -g . r_t;   S_{t-1} = S_t + alpha_t k_t r_t^T;
//     dk_t = -alpha_t (G r_t + S_{t-1} g) + dalpha_t (d alpha / d lambda) 2 k_t;
//     dbeta_t = dalpha_t (d alpha / d beta);   G -= alpha_t k_t g^T;   dS0 = G.
//
// Layout of the work: one CTA per (stream, 32-column slice of d_v), the slice of S and of
// G in registers (column j of the update needs only column j of S, r and g).  A forward
// sweep stores r_t (this slice) in the workspace; the reverse sweep rebuilds S_{t-1} from
// S_t by adding the stored rank-1 write back, which is exact algebra (no inverse).  Row
// sums over the slice (dq, dk, dalpha) are partial per slice and accumulate with atomics
// into zeroed fp32 buffers; the gate's terms, which need the full dalpha_t, are added by a
// last per-token kernel.
#include "efla_common.cuh"
#include "efla_kernels.h"

namespace efla {

namespace {
constexpr int kCols = 32;      // state columns per CTA
constexpr int kThreads = 256;  // 8 column quads x 32 row groups

__global__ void zero_kernel(float* __restrict__ p, long n) {
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) p[i] = 0.f;
}

// lambda = ||k||^2 by one warp (every warp computes it for itself: no barrier needed)
template <typename Tin, int D>
__device__ __forceinline__ float warp_norm2(const Tin* kh, int lane) {
    float lam = 0.f;
#pragma unroll
    for (int i = lane; i < D; i += 32) {
        const float x = Elem<Tin>::to_f(kh[i]);
        lam = fmaf(x, x, lam);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) lam += __shfl_xor_sync(0xffffffffu, lam, off);
    return lam;
}

__device__ __forceinline__ float4 f4_fma(float a, float4 x, float4 y) {
    return make_float4(fmaf(a, x.x, y.x), fmaf(a, x.y, y.y), fmaf(a, x.z, y.z), fmaf(a, x.w, y.w));
}
__device__ __forceinline__ float dot4(float4 a, float4 b) {
    return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}
// sum of a float4 over the 32 row groups of the CTA (rows within a warp by shuffles, then
// across the eight warps through `red`, a buffer used on alternate tokens)
__device__ __forceinline__ float4 rows_sum(float4 p, float4 (*red)[8], int warp, int lane, int cq) {
#pragma unroll
    for (int off = 8; off < 32; off <<= 1) {
        p.x += __shfl_xor_sync(0xffffffffu, p.x, off);
        p.y += __shfl_xor_sync(0xffffffffu, p.y, off);
        p.z += __shfl_xor_sync(0xffffffffu, p.z, off);
        p.w += __shfl_xor_sync(0xffffffffu, p.w, off);
    }
    if (lane < 8) red[warp][lane] = p;
    __syncthreads();
    float4 s = red[0][cq];
#pragma unroll
    for (int w = 1; w < 8; ++w) {
        const float4 a = red[w][cq];
        s.x += a.x; s.y += a.y; s.z += a.z; s.w += a.w;
    }
    return s;
}
// sum over the eight column quads of a warp (lanes differing in their low three bits)
__device__ __forceinline__ float quads_sum(float x) {
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

template <typename Tin, int D>
__global__ void __launch_bounds__(kThreads) bwd_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                                                       const Tin* __restrict__ v, const Tin* __restrict__ beta,
                                                       const float* __restrict__ S0, const Tin* __restrict__ dO,
                                                       const float* __restrict__ dST, float* __restrict__ dq,
                                                       float* __restrict__ dk, float* __restrict__ dv,
                                                       float* __restrict__ dS0, float* __restrict__ R,
                                                       float* __restrict__ dalpha, int T, int rule) {
    constexpr int RPT = D / 32;
    constexpr int SLICES = D / kCols;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cq = tid & 7, rg = tid >> 3;
    const long bh = blockIdx.x / SLICES;
    const int j0 = (blockIdx.x % SLICES) * kCols + cq * 4;
    __shared__ float4 red[2][8][8];

    const Tin* qb = q + bh * (long)T * D;
    const Tin* kb = k + bh * (long)T * D;
    const Tin* vb = v + bh * (long)T * D;
    const Tin* ob = dO + bh * (long)T * D;
    const Tin* bb = beta + bh * (long)T;
    float* Rb = R + bh * (long)T * D;

    float4 s[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m)
        s[m] = S0 ? *reinterpret_cast<const float4*>(S0 + (bh * D + rg + 32 * m) * (long)D + j0)
                  : make_float4(0.f, 0.f, 0.f, 0.f);

    // ---- forward sweep: S_T, and r_t of this slice for every token
    for (int t = 0; t < T; ++t) {
        const Tin* kh = kb + (long)t * D;
        float kr[RPT];
#pragma unroll
        for (int m = 0; m < RPT; ++m) kr[m] = Elem<Tin>::to_f(kh[rg + 32 * m]);
        const float4 vv = load4(vb + (long)t * D + j0);
        const float alpha = rule_alpha(rule, Elem<Tin>::to_f(bb[t]), warp_norm2<Tin, D>(kh, lane));
        float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int m = 0; m < RPT; ++m) p = f4_fma(kr[m], s[m], p);
        float4 r = rows_sum(p, red[t & 1], warp, lane, cq);
        r.x -= vv.x; r.y -= vv.y; r.z -= vv.z; r.w -= vv.w;
        if (rg == 0) *reinterpret_cast<float4*>(Rb + (long)t * D + j0) = r;
#pragma unroll
        for (int m = 0; m < RPT; ++m) s[m] = f4_fma(-alpha * kr[m], r, s[m]);
    }

    // ---- reverse sweep (the barrier keeps its first row sum off the buffer the forward
    // sweep's last one may still be reading; it also orders the r_t stores before their loads)
    __syncthreads();
    float4 G[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m)
        G[m] = dST ? *reinterpret_cast<const float4*>(dST + (bh * D + rg + 32 * m) * (long)D + j0)
                   : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int t = T - 1; t >= 0; --t) {
        const Tin* kh = kb + (long)t * D;
        const Tin* qh = qb + (long)t * D;
        float kr[RPT], qr[RPT];
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            kr[m] = Elem<Tin>::to_f(kh[rg + 32 * m]);
            qr[m] = Elem<Tin>::to_f(qh[rg + 32 * m]);
        }
        const float4 d_o = load4(ob + (long)t * D + j0);
        const float4 r = *reinterpret_cast<const float4*>(Rb + (long)t * D + j0);
        const float alpha = rule_alpha(rule, Elem<Tin>::to_f(bb[t]), warp_norm2<Tin, D>(kh, lane));
        float* dqt = dq + (bh * (long)T + t) * D;
        float* dkt = dk + (bh * (long)T + t) * D;

        // o_t = S_t^T q_t: G += q dO^T, dq = S_t dO (this slice's columns)
        float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            G[m] = f4_fma(qr[m], d_o, G[m]);
            const float a = quads_sum(dot4(s[m], d_o));
            if (cq == 0) atomicAdd(dqt + rg + 32 * m, a);
            p = f4_fma(kr[m], G[m], p);
        }
        // g = G^T k (full column sums)
        const float4 g = rows_sum(p, red[t & 1], warp, lane, cq);
        const float da = quads_sum(-dot4(g, r));        // the same in every row group
        if (rg == 0) {
            *reinterpret_cast<float4*>(dv + (bh * (long)T + t) * D + j0) =
                make_float4(alpha * g.x, alpha * g.y, alpha * g.z, alpha * g.w);
            if (lane == 0) atomicAdd(dalpha + bh * (long)T + t, da);
        }
        // S_{t-1} = S_t + alpha k r^T; dk (this slice) = -alpha (G r + S_{t-1} g); G -= alpha k g^T
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            s[m] = f4_fma(alpha * kr[m], r, s[m]);
            const float a = quads_sum(dot4(G[m], r) + dot4(s[m], g));
            if (cq == 0) atomicAdd(dkt + rg + 32 * m, -alpha * a);
            G[m] = f4_fma(-alpha * kr[m], g, G[m]);
        }
    }
    if (dS0) {
#pragma unroll
        for (int m = 0; m < RPT; ++m) *reinterpret_cast<float4*>(dS0 + (bh * D + rg + 32 * m) * (long)D + j0) = G[m];
    }
}

// the gate's share: dbeta_t = dalpha_t dalpha/dbeta, dk_t += dalpha_t dalpha/dlambda 2 k_t
// (one warp per token)
template <typename Tin, int D>
__global__ void bwd_gate_kernel(const Tin* __restrict__ k, const Tin* __restrict__ beta,
                                const float* __restrict__ dalpha, float* __restrict__ dk,
                                float* __restrict__ dbeta, long ntok, int rule) {
    const long tok = blockIdx.x * (long)(blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (tok >= ntok) return;
    const Tin* kh = k + tok * D;
    const float lam = warp_norm2<Tin, D>(kh, lane);
    const float b = Elem<Tin>::to_f(beta[tok]);
    const float da = dalpha[tok];
    float dadb = 1.f, dadl = 0.f;
    if (rule != kRuleEuler) {
        dadb = expf(-b * lam);
        dadl = gate_dalpha_dlambda(b, lam);
    }
    if (lane == 0) dbeta[tok] = da * dadb;
    const float c = 2.f * da * dadl;
#pragma unroll
    for (int i = lane; i < D; i += 32) dk[tok * D + i] = fmaf(c, Elem<Tin>::to_f(kh[i]), dk[tok * D + i]);
}

template <typename Tin, int D>
cudaError_t launch_bwd_t(const void* q, const void* k, const void* v, const void* beta, const float* S0,
                         const void* dO, const float* dST, float* dq, float* dk, float* dv, float* dbeta,
                         float* dS0, long BH, int T, int rule, float* R, float* dalpha, cudaStream_t stream) {
    const long ntok = BH * T;
    zero_kernel<<<592, 256, 0, stream>>>(dq, ntok * D);
    zero_kernel<<<592, 256, 0, stream>>>(dk, ntok * D);
    zero_kernel<<<148, 256, 0, stream>>>(dalpha, ntok);
    bwd_kernel<Tin, D><<<(unsigned)(BH * (D / kCols)), kThreads, 0, stream>>>(
        (const Tin*)q, (const Tin*)k, (const Tin*)v, (const Tin*)beta, S0, (const Tin*)dO, dST, dq, dk, dv, dS0, R,
        dalpha, T, rule);
    bwd_gate_kernel<Tin, D><<<(unsigned)((ntok + 7) / 8), 256, 0, stream>>>((const Tin*)k, (const Tin*)beta, dalpha,
                                                                          dk, dbeta, ntok, rule);
    return cudaGetLastError();
}
}  // namespace

size_t bwd_workspace_bytes(long BH, int T, int D) {
    return (size_t)BH * T * D * sizeof(float) + (size_t)BH * T * sizeof(float);
}

cudaError_t launch_bwd(const void* q, const void* k, const void* v, const void* beta, const float* S0,
                       const void* dO, const float* dST, float* dq, float* dk, float* dv, float* dbeta, float* dS0,
                       long BH, int T, int D, bool bf16, int rule, void* workspace, cudaStream_t stream) {
    float* R = static_cast<float*>(workspace);
    float* dalpha = R + (size_t)BH * T * D;
    if (bf16) {
        return D == 128 ? launch_bwd_t<__nv_bfloat16, 128>(q, k, v, beta, S0, dO, dST, dq, dk, dv, dbeta, dS0, BH, T,
                                                          rule, R, dalpha, stream)
                        : launch_bwd_t<__nv_bfloat16, 64>(q, k, v, beta, S0, dO, dST, dq, dk, dv, dbeta, dS0, BH, T,
                                                         rule, R, dalpha, stream);
    }
    return D == 128 ? launch_bwd_t<float, 128>(q, k, v, beta, S0, dO, dST, dq, dk, dv, dbeta, dS0, BH, T, rule, R,
                                               dalpha, stream)
                    : launch_bwd_t<float, 64>(q, k, v, beta, S0, dO, dST, dq, dk, dv, dbeta, dS0, BH, T, rule, R,
                                              dalpha, stream);
}

}  // namespace efla
