// efla_gate.cu -- the exact-flow gate alone: lambda = ||k||^2 (fp32 accumulation) and
// alpha = (1 - exp(-beta*lambda)) / lambda per token (Exact Flow Linear Attention,
// Section 3.2 and Section 3.4).  One warp per token, 16-byte loads, shuffle reduction.
#include "efla_common.cuh"
#include "efla_kernels.h"

namespace efla {

template <typename Tin>
__global__ void __launch_bounds__(256) gate_kernel(const Tin* __restrict__ k,
                                                   const Tin* __restrict__ beta,
                                                   float* __restrict__ alpha, long n, int dk) {
    const int lane = threadIdx.x & 31;
    const long tok = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (tok >= n) return;
    const Tin* kr = k + tok * (long)dk;
    float lam = 0.f;
    for (int i = lane * 4; i < dk; i += 128) {
        float4 x = load4(kr + i);
        lam = fmaf(x.x, x.x, lam);
        lam = fmaf(x.y, x.y, lam);
        lam = fmaf(x.z, x.z, lam);
        lam = fmaf(x.w, x.w, lam);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lam += __shfl_xor_sync(0xffffffffu, lam, o);
    if (lane == 0) alpha[tok] = gate_alpha(Elem<Tin>::to_f(beta[tok]), lam);
}

cudaError_t launch_gate(const void* k, const void* beta, float* alpha, long n, int dk, bool bf16,
                        cudaStream_t stream) {
    const int warps = 8;
    const long blocks = (n + warps - 1) / warps;
    if (bf16)
        gate_kernel<__nv_bfloat16><<<(unsigned)blocks, warps * 32, 0, stream>>>(
            (const __nv_bfloat16*)k, (const __nv_bfloat16*)beta, alpha, n, dk);
    else
        gate_kernel<float><<<(unsigned)blocks, warps * 32, 0, stream>>>(
            (const float*)k, (const float*)beta, alpha, n, dk);
    return cudaGetLastError();
}

}  // namespace efla
