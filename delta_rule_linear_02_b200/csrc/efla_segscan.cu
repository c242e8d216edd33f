// efla_segscan.cu -- the segmented scan's combine and output correction (bf16, d = 128).
//
// Exact Flow Linear Attention, Section 3.3: a chunk maps the entering state affinely,
// S -> (I - K^T W) S + K^T U, so a whole segment of chunks does too:
//     S_out = Phi S_in + S_loc,   O = O_loc + R S_in,
// where S_loc, O_loc are the segment run from a zero state and Phi, R the same run with
// V = 0 from S = I (its final state and its outputs).  The chain kernel produces all four
// for every segment at once (SegPlan in efla_kernels.h); here
//   combine:  S_in(1) = S_loc(0), S_in(g+1) = Phi(g) S_in(g) + S_loc(g), S_T = S_in(G)   (fp32)
//   correct:  o[t] += R[t] S_in(g) for the tokens t of every segment g >= 1   (bf16 MMA,
//             fp32 accumulation: R and S_in as bf16 operands, like every chunk product;
//             the combine hands S_in(g) over transposed in bf16)
#include "efla_common.cuh"
#include "efla_kernels.h"
#include "efla_mma_sync.cuh"

namespace efla {

namespace {
constexpr int kD = 128;

// One CTA per (stream, 32-column block): the column block of S_in(g) evolves on its own.
__global__ void __launch_bounds__(256) seg_combine_kernel(SegPlan seg, float* __restrict__ S_T,
                                                          __nv_bfloat16* __restrict__ SinT) {
    __shared__ float cur[kD][33];                   // S_in(g)[:, block], padded
    __shared__ float pk[kD][33];                    // a 32-column slab of Phi(g)
    const long s = blockIdx.x >> 2;
    const int j0 = (blockIdx.x & 3) * 32;
    const int t = threadIdx.x;
    const size_t mat = (size_t)kD * kD;
    const float* sloc = seg.Sloc + (size_t)s * seg.G * mat;
    const float* phi = seg.Phi + (size_t)s * seg.G * mat;
    // S_in(g) for the correction: bf16, transposed (SinT[g][n][k] = S_in(g)[k][n])
    __nv_bfloat16* sint = SinT + (size_t)s * seg.G * mat;
    for (int e = t; e < kD * 32; e += 256) {         // S_in(1) = S_loc(0)
        const int i = e >> 5, j = e & 31;
        const float x = sloc[(size_t)i * kD + j0 + j];
        cur[i][j] = x;
        if (seg.G > 1) sint[mat + (size_t)(j0 + j) * kD + i] = __float2bfloat16_rn(x);
    }
    __syncthreads();
    for (int g = 1; g < seg.G; ++g) {
        // out = Phi(g) cur + S_loc(g): thread t owns rows (t >> 3) + 32 r, columns 4 (t & 7) .. +3
        float acc[4][4];
        const int rb = t >> 3, cb = (t & 7) * 4;
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[r][c] = sloc[g * mat + (size_t)(rb + 32 * r) * kD + j0 + cb + c];
        const float* P = phi + g * mat;
        for (int k0 = 0; k0 < kD; k0 += 32) {        // Phi[:, k0 .. k0 + 31] through shared memory
            __syncthreads();
            for (int e = t; e < kD * 32; e += 256) {
                const int i = e >> 5, kk = e & 31;
                pk[i][kk] = P[(size_t)i * kD + k0 + kk];
            }
            __syncthreads();
#pragma unroll 4
            for (int kk = 0; kk < 32; ++kk) {
                float b[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) b[c] = cur[k0 + kk][cb + c];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const float a = pk[rb + 32 * r][kk];
#pragma unroll
                    for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(a, b[c], acc[r][c]);
                }
            }
        }
        __syncthreads();                             // every read of cur is done
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int i = rb + 32 * r, j = cb + c;
                cur[i][j] = acc[r][c];
                if (g + 1 < seg.G) sint[(g + 1) * mat + (size_t)(j0 + j) * kD + i] = __float2bfloat16_rn(acc[r][c]);
            }
        __syncthreads();
    }
    if (S_T) {
        for (int e = t; e < kD * 32; e += 256) {
            const int i = e >> 5, j = e & 31;
            S_T[(size_t)s * mat + (size_t)i * kD + j0 + j] = cur[i][j];
        }
    }
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

constexpr int LW = kD + 8;     // bf16 row stride of the 128-wide tiles (conflict-free ldmatrix rows)
constexpr int kTilesPerCta = 4;

// One CTA (8 warps) per (stream, run of 4 64-token tiles of segments >= 1): S_in^T of the
// tiles' segment once, then o_tile += R_tile S_in for each tile.  Warp w: rows 16 (w % 4),
// columns 64 (w / 4).  A run never straddles segments (segments are whole multiples of 4
// tiles, or the run ends where its segment ends).
__global__ void __launch_bounds__(256) seg_correct_kernel(SegPlan seg, const __nv_bfloat16* __restrict__ SinT,
                                                          __nv_bfloat16* __restrict__ o, int T, int runs_per) {
    using namespace mmas;
    extern __shared__ __align__(16) uint8_t seg_smem[];
    bf16* St = reinterpret_cast<bf16*>(seg_smem);    // kD x LW: S_in^T
    bf16* Rt = St + kD * LW;                          // 2 x (64 x LW): R tiles, double-buffered
    float* Ct = reinterpret_cast<float*>(Rt + 2 * 64 * LW);   // 64 x (kD + 4): R S_in of a tile, fp32
    const long s = blockIdx.x / runs_per;
    const int run = (int)(blockIdx.x % runs_per);
    const int L = seg.seg_chunks * 64;
    const int runs_seg = (seg.seg_chunks + kTilesPerCta - 1) / kTilesPerCta;   // runs per segment
    const int g = 1 + run / runs_seg;
    const int t_first = g * L + (run % runs_seg) * kTilesPerCta * 64;
    const int t_end = min(T, min((g + 1) * L, t_first + kTilesPerCta * 64));
    if (g >= seg.G || t_first >= t_end) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wm = 16 * (warp & 3), wn = 64 * (warp >> 2);
    load_tile(St, LW, SinT + ((size_t)s * seg.G + g) * kD * kD, kD, kD, kD, kD, tid, 256);
    const bf16* Rg = seg.R + (size_t)s * T * kD;
    auto issue = [&](int t0, bf16* dst) { load_tile(dst, LW, Rg + (size_t)t0 * kD, kD, 64, kD, min(64, t_end - t0), tid, 256); };
    issue(t_first, Rt);
    cp_async_commit();
    int buf = 0;
    for (int t0 = t_first; t0 < t_end; t0 += 64, buf ^= 1) {
        if (t0 + 64 < t_end) {
            issue(t0 + 64, Rt + (buf ^ 1) * 64 * LW);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        float acc[8][4];
        zero_acc(acc);
        warp_mma<8, false, false>(acc, Rt + buf * 64 * LW, LW, St, LW, wm, wn, kD, lane);
        for_acc(acc, wm, wn, lane, [&](int r, int c, float& x) { Ct[r * (kD + 4) + c] = x; });
        __syncthreads();                              // the tile's R S_in is staged; this R buffer is free
        // o += R S_in with 16-byte accesses: 8 consecutive bf16 of a row per thread and step
        const int nrow = min(64, t_end - t0);
        bf16* Og = o + ((size_t)s * T + t0) * kD;
        for (int e = tid; e < 64 * (kD / 8); e += 256) {
            const int r = e / (kD / 8), c = (e % (kD / 8)) * 8;
            if (r < nrow) {
                uint4* p = reinterpret_cast<uint4*>(Og + (size_t)r * kD + c);
                uint4 cur = *p;
                const float* add = Ct + r * (kD + 4) + c;
                uint32_t* w = reinterpret_cast<uint32_t*>(&cur);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(w + m));
                    w[m] = pack2(f.x + add[2 * m], f.y + add[2 * m + 1]);
                }
                *p = cur;
            }
        }
        __syncthreads();                              // Ct is rewritten by the next tile
    }
}
}  // namespace

cudaError_t launch_seg_combine(const SegPlan& seg, const float* S0, float* S_T, void* SinT, long nstreams,
                               cudaStream_t stream) {
    (void)S0;   // segment 0 starts from S0 inside the chain kernel; its final state is S_loc(0)
    seg_combine_kernel<<<(unsigned)(nstreams * 4), 256, 0, stream>>>(seg, S_T, static_cast<__nv_bfloat16*>(SinT));
    return cudaGetLastError();
}

cudaError_t launch_seg_correct(const SegPlan& seg, const void* SinT, __nv_bfloat16* o, long nstreams, int T,
                               cudaStream_t stream) {
    const int runs_seg = (seg.seg_chunks + kTilesPerCta - 1) / kTilesPerCta;
    const int runs_per = runs_seg * (seg.G - 1);
    if (runs_per <= 0) return cudaSuccess;
    constexpr int smem = (kD + 2 * 64) * LW * 2 + 64 * (kD + 4) * 4;
    static std::atomic<uint64_t> smem_set{0};
    cudaError_t e = set_smem_limit_once(seg_correct_kernel, smem, smem_set);
    if (e != cudaSuccess) return e;
    seg_correct_kernel<<<(unsigned)(nstreams * runs_per), 256, smem, stream>>>(
        seg, static_cast<const __nv_bfloat16*>(SinT), o, T, runs_per);
    return cudaGetLastError();
}

}  // namespace efla
