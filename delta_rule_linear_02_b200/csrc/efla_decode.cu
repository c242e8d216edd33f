// efla_decode.cu -- one recurrent (decode) token for N*H streams, state updated in place.
//
// Exact Flow Linear Attention, Section 3.2 (update with the exact-flow gate) in the
// recurrent form; the read-out o_t = S_t^T q_t is taken after the write.  With
// r = k^T S, p = q^T S, c = q.k and e = r - v (row convention, S is d_k x d_v):
//     S_new = S - alpha k e^T,      o = S_new^T q = p - alpha c e.
// The gated flow (Section 3.4, Gated EFLA) with decay d = e^g and write gate abar:
//     S_new = d S - k w^T,  w = d alpha r - abar v,   o = d p - c w
// (d = 1 and abar = alpha give the line above).
// Column j of S_new depends only on column j of S, so each CTA owns a 32-column slice
// of one head's state and streams it exactly once through registers: one HBM read and
// one HBM write of the 4*d_k*d_v-byte state per token, the bound for this step.
#include "efla_common.cuh"
#include "efla_kernels.h"

namespace efla {

namespace {
constexpr int kCols = 32;      // state columns per CTA
constexpr int kThreads = 256;  // 8 column-quads x 32 row groups

template <typename Tin, int D, bool kGated = false>
__global__ void __launch_bounds__(kThreads) decode_kernel(const Tin* __restrict__ q,
                                                          const Tin* __restrict__ k,
                                                          const Tin* __restrict__ v,
                                                          const Tin* __restrict__ beta,
                                                          float* __restrict__ S,
                                                          Tin* __restrict__ o, int rule,
                                                          const float* __restrict__ gdec = nullptr) {
    constexpr int RPT = D / 32;                 // rows per thread
    constexpr int SLICES = D / kCols;
    const int t = threadIdx.x;
    const int cq = t & 7;                       // float4 column within the slice
    const int rg = t >> 3;                      // row group 0..31
    const int warp = t >> 5, lane = t & 31;
    const long head = blockIdx.x / SLICES;
    const int j0 = (blockIdx.x % SLICES) * kCols + cq * 4;

    float* Sh = S + head * (long)D * D;
    // 1. stream the state tile in first: the loads are independent of everything else
    float4 s[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) s[m] = __ldcs(reinterpret_cast<const float4*>(Sh + (long)(rg + 32 * m) * D + j0));

    const Tin* qh = q + head * D;
    const Tin* kh = k + head * D;
    float kr[RPT], qr[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        kr[m] = Elem<Tin>::to_f(kh[rg + 32 * m]);
        qr[m] = Elem<Tin>::to_f(qh[rg + 32 * m]);
    }
    const float4 vv = load4(v + head * D + j0);

    __shared__ float4 red_r[8][8];
    __shared__ float4 red_p[8][8];
    __shared__ float sh_alpha, sh_c, sh_abar, sh_dec;

    // 2. lambda = ||k||^2 and c = q.k over the full key, by warp 0
    if (warp == 0) {
        float lam = 0.f, c = 0.f;
#pragma unroll
        for (int i = lane; i < D; i += 32) {
            const float ki = Elem<Tin>::to_f(kh[i]);
            lam = fmaf(ki, ki, lam);
            c = fmaf(Elem<Tin>::to_f(qh[i]), ki, c);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            lam += __shfl_xor_sync(0xffffffffu, lam, off);
            c += __shfl_xor_sync(0xffffffffu, c, off);
        }
        if (lane == 0) {
            const float bt = Elem<Tin>::to_f(beta[head]);
            sh_alpha = rule_alpha(rule, bt, lam);
            sh_c = c;
            if constexpr (kGated) {
                const float gh = gdec[head];
                sh_abar = rule_write_gate(rule, bt, lam, gh);
                sh_dec = expf(gh);
            }
        }
    }

    // 3. partial r = k^T S and p = q^T S over this thread's rows, then over the warp
    float4 r = make_float4(0.f, 0.f, 0.f, 0.f), p = r;
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        r.x = fmaf(kr[m], s[m].x, r.x); r.y = fmaf(kr[m], s[m].y, r.y);
        r.z = fmaf(kr[m], s[m].z, r.z); r.w = fmaf(kr[m], s[m].w, r.w);
        p.x = fmaf(qr[m], s[m].x, p.x); p.y = fmaf(qr[m], s[m].y, p.y);
        p.z = fmaf(qr[m], s[m].z, p.z); p.w = fmaf(qr[m], s[m].w, p.w);
    }
#pragma unroll
    for (int off = 8; off < 32; off <<= 1) {
        r.x += __shfl_xor_sync(0xffffffffu, r.x, off); r.y += __shfl_xor_sync(0xffffffffu, r.y, off);
        r.z += __shfl_xor_sync(0xffffffffu, r.z, off); r.w += __shfl_xor_sync(0xffffffffu, r.w, off);
        p.x += __shfl_xor_sync(0xffffffffu, p.x, off); p.y += __shfl_xor_sync(0xffffffffu, p.y, off);
        p.z += __shfl_xor_sync(0xffffffffu, p.z, off); p.w += __shfl_xor_sync(0xffffffffu, p.w, off);
    }
    if (lane < 8) {
        red_r[warp][lane] = r;
        red_p[warp][lane] = p;
    }
    __syncthreads();

    // 4. full column sums (every thread, for its own column quad)
    r = red_r[0][cq];
    p = red_p[0][cq];
#pragma unroll
    for (int w = 1; w < 8; ++w) {
        const float4 a = red_r[w][cq], b = red_p[w][cq];
        r.x += a.x; r.y += a.y; r.z += a.z; r.w += a.w;
        p.x += b.x; p.y += b.y; p.z += b.z; p.w += b.w;
    }
    const float alpha = sh_alpha, c = sh_c;
    if constexpr (kGated) {
        // w = d alpha r - abar v;  S_new = d S - k w^T;  o = d p - c w
        const float dec = sh_dec, da = sh_dec * sh_alpha, ab = sh_abar;
        const float4 w = make_float4(fmaf(da, r.x, -ab * vv.x), fmaf(da, r.y, -ab * vv.y),
                                     fmaf(da, r.z, -ab * vv.z), fmaf(da, r.w, -ab * vv.w));
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            const float km = kr[m];
            float4 u = s[m];
            u.x = fmaf(-km, w.x, dec * u.x); u.y = fmaf(-km, w.y, dec * u.y);
            u.z = fmaf(-km, w.z, dec * u.z); u.w = fmaf(-km, w.w, dec * u.w);
            __stcs(reinterpret_cast<float4*>(Sh + (long)(rg + 32 * m) * D + j0), u);
        }
        if (rg == 0)
            store4(o + head * D + j0, make_float4(fmaf(-c, w.x, dec * p.x), fmaf(-c, w.y, dec * p.y),
                                                  fmaf(-c, w.z, dec * p.z), fmaf(-c, w.w, dec * p.w)));
        return;
    }
    const float4 e = make_float4(r.x - vv.x, r.y - vv.y, r.z - vv.z, r.w - vv.w);

    // 5. rank-1 write S -= alpha k e^T, streamed back
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const float ak = alpha * kr[m];
        float4 u = s[m];
        u.x = fmaf(-ak, e.x, u.x); u.y = fmaf(-ak, e.y, u.y);
        u.z = fmaf(-ak, e.z, u.z); u.w = fmaf(-ak, e.w, u.w);
        __stcs(reinterpret_cast<float4*>(Sh + (long)(rg + 32 * m) * D + j0), u);
    }
    // 6. read-out after the write: o = p - alpha c e
    if (rg == 0) {
        const float ac = alpha * c;
        store4(o + head * D + j0, make_float4(fmaf(-ac, e.x, p.x), fmaf(-ac, e.y, p.y),
                                              fmaf(-ac, e.z, p.z), fmaf(-ac, e.w, p.w)));
    }
}

template <typename Tin, int D>
cudaError_t launch_decode_t(const void* q, const void* k, const void* v, const void* beta,
                            float* S, void* o, long NH, int rule, const float* g, cudaStream_t stream) {
    const long blocks = NH * (D / kCols);
    if (g)
        decode_kernel<Tin, D, true><<<(unsigned)blocks, kThreads, 0, stream>>>(
            (const Tin*)q, (const Tin*)k, (const Tin*)v, (const Tin*)beta, S, (Tin*)o, rule, g);
    else
        decode_kernel<Tin, D><<<(unsigned)blocks, kThreads, 0, stream>>>(
            (const Tin*)q, (const Tin*)k, (const Tin*)v, (const Tin*)beta, S, (Tin*)o, rule);
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_decode(const void* q, const void* k, const void* v, const void* beta, float* S,
                          void* o, long NH, int D, bool bf16, int rule, cudaStream_t stream, const float* g) {
    if (bf16) {
        return D == 128 ? launch_decode_t<__nv_bfloat16, 128>(q, k, v, beta, S, o, NH, rule, g, stream)
                        : launch_decode_t<__nv_bfloat16, 64>(q, k, v, beta, S, o, NH, rule, g, stream);
    }
    return D == 128 ? launch_decode_t<float, 128>(q, k, v, beta, S, o, NH, rule, g, stream)
                    : launch_decode_t<float, 64>(q, k, v, beta, S, o, NH, rule, g, stream);
}

}  // namespace efla
