// efla_common.cuh -- element access and the exact-flow gate, shared by the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace efla {

// ---------------------------------------------------------------- element access
template <typename T> struct Elem;

template <> struct Elem<float> {
    static __device__ __forceinline__ float to_f(float x) { return x; }
    static __device__ __forceinline__ float from_f(float x) { return x; }
};

template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
    static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// Load 4 consecutive elements (16-byte aligned for float, 8-byte for bf16) as floats.
__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
    uint2 u = *reinterpret_cast<const uint2*>(p);
    float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.x));
    float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ void store4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
}

// ---------------------------------------------------------------- the gate
// Exact Flow Linear Attention, Section 3.2: the closed-form flow keeps the delta rule's
// rank-1 write with beta replaced by alpha = (1 - exp(-beta*lambda)) / lambda, where
// lambda = ||k||^2 (Section 3.4; the nonzero eigenvalue of A = k k^T, App. D).
// For |x| = |beta*lambda| < 2^-10 the series 1 - x/2 + x^2/6 of (1 - e^{-x})/x is used
// (truncation error below x^3/24 < 4e-11 relative): it keeps full precision when x is
// subnormal and gives alpha = beta exactly at lambda = 0, the limit of the formula.
// The step size the rule writes with: the exact flow's gate, or beta itself for the Euler
// (delta-rule) step the exact flow replaces (Exact Flow Linear Attention, Section 2).
constexpr int kRuleExact = 0, kRuleEuler = 1;
__device__ __forceinline__ float gate_alpha(float beta, float lambda);
__device__ __forceinline__ float rule_alpha(int rule, float beta, float lambda) {
    return rule == kRuleEuler ? beta : gate_alpha(beta, lambda);
}

__device__ __forceinline__ float gate_alpha(float beta, float lambda) {
    const float x = beta * lambda;
    if (fabsf(x) < 0.0009765625f) {
        return beta * (1.0f - x * (0.5f - x * (1.0f / 6.0f)));
    }
    return -expm1f(-x) / lambda;
}

// d alpha / d lambda of the exact gate in fp32: (beta e^{-x} - alpha) / lambda, x = beta*lambda,
// by its series beta^2 sum_{n>=1} (-1)^n n x^{n-1} / (n+1)! for |x| < 1/16 (where the
// difference cancels; truncation below x^6 / 840 relative), limit -beta^2/2 at lambda = 0.
__device__ __forceinline__ float gate_dalpha_dlambda(float beta, float lambda) {
    const float x = beta * lambda;
    if (fabsf(x) < 0.0625f)
        return beta * beta *
               (-0.5f + x * (1.0f / 3.0f - x * (1.0f / 8.0f - x * (1.0f / 30.0f - x * (1.0f / 144.0f - x * (1.0f / 840.0f))))));
    return (beta * expf(-x) + expm1f(-x) / lambda) / lambda;
}

// The gate's derivatives for the backward pass: dalpha/dbeta = e^{-beta lambda} and
// dalpha/dlambda above (the Euler rule: 1 and 0).
__device__ __forceinline__ void gate_derivatives(int rule, float beta, float lambda, float alpha, float* dadb,
                                                 float* dadl) {
    (void)alpha;
    if (rule == kRuleEuler) {
        *dadb = 1.f;
        *dadl = 0.f;
        return;
    }
    *dadb = expf(-beta * lambda);
    *dadl = gate_dalpha_dlambda(beta, lambda);
}

// The gated flow (Gated EFLA, Section 3.4): a per-token log-decay g joins the ODE over the
// token's unit interval, dS/dtau = g S - beta (k k^T S - k v^T).  The flow keeps alpha for the
// rank-1 contraction, decays the state by e^g, and writes with
//     abar = beta phi1(beta lambda - g),   phi1(x) = (1 - e^{-x}) / x,
// which equals alpha at g = 0.  phi1 uses the same short series as gate_alpha near x = 0.
// Under the Euler rule (the gated delta rule) the write uses beta.
__device__ __forceinline__ float phi1(float x) {
    if (fabsf(x) < 0.0009765625f) return 1.0f - x * (0.5f - x * (1.0f / 6.0f));
    return -expm1f(-x) / x;
}
__device__ __forceinline__ float rule_write_gate(int rule, float beta, float lambda, float g) {
    return rule == kRuleEuler ? beta : beta * phi1(beta * lambda - g);
}

// ---------------------------------------------------------------- streams and tiles
// One recurrence ("stream") per (sequence, head).  Dense batches: stream bh of B*H, each T
// tokens, tensors [B*H][T][d].  Packed variable-length batches (Section 3.3's chunking per
// sequence): N sequences of one head-major stream per head, tensors [H][total_T][d], sequence
// n at tokens cu[n] .. cu[n+1] of every head; stream n*H + h; chunks restart at each
// sequence start, so a sequence's tail chunk is padded with alpha = 0 (its rows past the
// sequence end belong to the next sequence and are never written).
struct StreamJob {
    int z;          // index along the outer tensor dimension: bh (dense) or h (packed)
    int y0;         // first token of the stream within that row
    int len;        // tokens
    long tile0;     // UT tile of the stream's chunk 0
};
struct Seqs {
    const int* cu;        // packed: N+1 offsets (device); null for dense batches
    const int* tileoff;   // packed: N+1 prefix sums of the sequences' chunk counts
    int N, H;             // packed: sequences, heads
    int T;                // dense: tokens per stream
    long total_tiles;     // packed: tileoff[N] (per head)
    __device__ __forceinline__ StreamJob job(long s) const {
        if (!cu) return StreamJob{(int)s, 0, T, s * (long)((T + 63) / 64)};
        const int n = (int)(s / H), h = (int)(s % H);
        return StreamJob{h, cu[n], cu[n + 1] - cu[n], (long)h * total_tiles + tileoff[n]};
    }
    // UT tile i -> its stream's job and chunk
    __device__ __forceinline__ StreamJob tile(long i, int* chunk) const {
        if (!cu) {
            const int nc = (T + 63) / 64;
            *chunk = (int)(i % nc);
            return StreamJob{(int)(i / nc), 0, T, i - *chunk};
        }
        const int h = (int)(i / total_tiles);
        const int j = (int)(i % total_tiles);
        int lo = 0, hi = N;                   // largest n with tileoff[n] <= j (sequences with chunks)
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (tileoff[mid] <= j) lo = mid; else hi = mid;
        }
        *chunk = j - tileoff[lo];
        return StreamJob{h, cu[lo], cu[lo + 1] - cu[lo], (long)h * total_tiles + tileoff[lo]};
    }
};

// Device error word values (kept in the caller's workspace).
enum : uint32_t { kDevOk = 0u, kDevTimeout = 1u, kDevBounds = 2u };

// ---------------------------------------------------------------- checked builds
// Built with -DEFLA_CHECKED=1 (delta_rule_linear_02_b200/build.py --checked, a separate
// library), the tensor-core forward's kernels test every generic global access and every
// computed shared-memory store against the extent of its buffer; a violation sets
// kDevBounds in the error word and the access is skipped (no trap, no assert).  In the
// normal build the tests compile away.
#ifndef EFLA_CHECKED
#define EFLA_CHECKED 0
#endif
struct Span {
    const void* p = nullptr;
    size_t bytes = 0;
};
__device__ __forceinline__ bool span_ok(uint32_t* err, Span s, const void* q, size_t n) {
#if EFLA_CHECKED
    const uintptr_t a = reinterpret_cast<uintptr_t>(s.p), b = reinterpret_cast<uintptr_t>(q);
    if (s.p && b >= a && b + n <= a + s.bytes) return true;
    atomicOr(err, kDevBounds);
    return false;
#else
    (void)err; (void)s; (void)q; (void)n;
    return true;
#endif
}
// an offset into a CTA's shared-memory map of `limit` bytes
__device__ __forceinline__ bool smem_ok(uint32_t* err, uint32_t off, uint32_t n, uint32_t limit) {
#if EFLA_CHECKED
    if (off + n <= limit) return true;
    atomicOr(err, kDevBounds);
    return false;
#else
    (void)err; (void)off; (void)n; (void)limit;
    return true;
#endif
}

// A kernel's dynamic shared-memory limit is a per-device attribute that persists, so it
// is set once per device (bit `dev` of `done`); setting it on every launch would add a
// driver call to each forward.
template <typename Kernel>
inline cudaError_t set_smem_limit_once(Kernel kernel, int bytes, std::atomic<uint64_t>& done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0;
    if (bit && (done.load(std::memory_order_relaxed) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_relaxed);
    return e;
}

}  // namespace efla
