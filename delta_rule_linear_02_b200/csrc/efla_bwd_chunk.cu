// efla_bwd_chunk.cu -- the backward pass through the chunkwise (UT) form, bf16 d = 128.
//
// Exact Flow Linear Attention, Section 3.3 computes a chunk as dense products; its reverse
// mode differentiates those products (row convention; S the chunk's entering state, dS'
// the gradient of its leaving state):
//   forward:  G = K K^T, A = strict_tril(diag(alpha) G), X = (I + A)^{-1}, T = X diag(alpha),
//             R = V - K S, Delta = T R, P = tril_incl(Q K^T), O = Q S + P Delta,
//             S' = S + K^T Delta
//   reverse:  dDelta = P^T dO + K dS',   dR = T^T dDelta = dV,
//             dS = dS' + Q^T dO - K^T dR                       (carried to the previous chunk)
//             dP = tril_incl(dO Delta^T),  dQ = dO S^T + dP K,  dT = dDelta R^T,
//             dalpha_j = sum_i dT_ij X_ij + sum_s dA_js G_js,  dA = strict_tril(-X^T dT diag(alpha) X^T),
//             dK = Delta dS'^T + dP^T Q - dR S^T + (dG + dG^T) K + dalpha (dalpha/dlambda) 2 K,
//             dG = diag(alpha) dA,  dbeta = dalpha dalpha/dbeta.
// Three launches after the UT transforms (efla_ut.cu):
//   1. the forward chain (efla_chunk_tc.cu) storing every chunk's entering state S (bf16);
//   2. bwd_chain_kernel: one CTA per (stream, 64-column half of d_v) walks the chunks in
//      reverse, carrying its half of dS in the MMA accumulators (the columns of dS evolve
//      independently), and stores each chunk's dS' (bf16);
//   3. bwd_tile_kernel: one CTA per (stream, chunk), all chunks at once: every gradient of
//      the chunk from its S and dS'.
// Products are warp-level bf16 tensor-core tiles (mma.sync m16n8k16, fp32 accumulation;
// operands read with ldmatrix from padded shared memory); the triangular solve that gives X
// again is fp32 on CUDA cores.  Operands pass through bf16 as in the forward, so the
// gradients carry bf16-operand rounding (relative Frobenius error ~1e-2), not fp32's.
#include "efla_common.cuh"
#include "efla_kernels.h"
#include "efla_mma_sync.cuh"
#include "efla_ut_solve.cuh"

namespace efla {

namespace {
using namespace mmas;
constexpr int kD = 128, kC = 64;
constexpr int LW = kD + 8;     // bf16 row stride of 128-wide tiles (272 B: conflict-free ldmatrix rows)
constexpr int LH = 64 + 8;     // bf16 row stride of 64-wide tiles (144 B)
constexpr int LF = 65;         // fp32 row stride of the solve's 64 x 64 tiles

// ============================================================================ reverse chain
// One CTA (8 warps) per (stream, d_v half).  Per chunk, walking backwards:
//   store dS' (the carried gradient, bf16) for the tile kernel;
//   P = tril(Q K^T);  dDelta = P^T dO + K dS';  -dR = -(T^T dDelta);  dS += Q^T dO + K^T (-dR).
// Warp w carries rows 16 w .. 16 w + 15 of the dS half in its accumulators.
struct ChainSmem {
    static constexpr int Q = 0;                          // per stage: Q, K (64 x LW), T (64 x LH), dO (64 x LH)
    static constexpr int K = Q + kC * LW;
    static constexpr int T = K + kC * LW;
    static constexpr int DO = T + kC * LH;
    static constexpr int STAGE = DO + kC * LH;           // bf16 elements per stage
    static constexpr int P = 2 * STAGE;
    static constexpr int DD = P + kC * LH;               // dDelta
    static constexpr int NR = DD + kC * LH;              // -dR
    static constexpr int DS = NR + kC * LH;              // dS (bf16), 128 x LH
    static constexpr int ELEMS = DS + kD * LH;
    static constexpr size_t BYTES = sizeof(bf16) * ELEMS;
};

__global__ void __launch_bounds__(256, 1)
bwd_chain_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ dO,
                 const bf16* __restrict__ Tt, const float* __restrict__ dST, bf16* __restrict__ dSp,
                 float* __restrict__ dS0, int T) {
    extern __shared__ __align__(16) bf16 sh[];
    using L = ChainSmem;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long bh = blockIdx.x >> 1;
    const int col0 = (blockIdx.x & 1) * 64;
    const int nchunks = (T + kC - 1) / kC;
    const long tile0 = bh * nchunks;
    auto stage = [&](int c) { return sh + (c & 1) * L::STAGE; };
    auto issue = [&](int c) {   // chunk c's Q, K, T and dO half into its stage
        bf16* st = stage(c);
        const int nv = min(kC, T - c * kC);
        const size_t row0 = (size_t)bh * T + (size_t)c * kC;
        load_tile(st + L::Q, LW, q + row0 * kD, kD, kC, kD, nv, tid, 256);
        load_tile(st + L::K, LW, k + row0 * kD, kD, kC, kD, nv, tid, 256);
        load_tile(st + L::T, LH, Tt + (size_t)(tile0 + c) * kC * kC, kC, kC, kC, kC, tid, 256);
        load_tile(st + L::DO, LH, dO + row0 * kD + col0, kD, kC, 64, nv, tid, 256);
        cp_async_commit();
    };
    // the carried gradient: dS_T's half (or zero)
    float ds[8][4];
    zero_acc(ds);
    if (dST) for_acc(ds, 16 * warp, 0, lane, [&](int r, int c, float& v) { v = dST[((size_t)bh * kD + r) * kD + col0 + c]; });
    bf16* dsb = sh + L::DS;
    auto write_ds = [&]() {
        for_acc(ds, 16 * warp, 0, lane, [&](int r, int c, float& v) { dsb[r * LH + c] = __float2bfloat16_rn(v); });
    };
    write_ds();
    issue(nchunks - 1);
    for (int c = nchunks - 1; c >= 0; --c) {
        if (c > 0) {
            issue(c - 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();                                   // stage c landed, dS' (bf16) complete
        const bf16* st = stage(c);
        // dS' for the tile kernel (this half's 64 columns of the 128 x 128 matrix)
        for (int e = tid; e < kD * 8; e += 256) {
            const int rr = e >> 3, cc = (e & 7) * 8;
            *reinterpret_cast<uint4*>(dSp + ((size_t)(tile0 + c) * kD + rr) * kD + col0 + cc) =
                *reinterpret_cast<const uint4*>(dsb + rr * LH + cc);
        }
        {   // P = tril_incl(Q K^T): warp w -> rows 16 (w % 4), columns 32 (w / 4)
            float acc[4][4];
            zero_acc(acc);
            const int m0 = 16 * (warp & 3), n0 = 32 * (warp >> 2);
            warp_mma<4, false, false>(acc, st + L::Q, LW, st + L::K, LW, m0, n0, kD, lane);
            for_acc(acc, m0, n0, lane, [&](int r, int c2, float& v) {
                sh[L::P + r * LH + c2] = __float2bfloat16_rn(c2 <= r ? v : 0.f);
            });
        }
        __syncthreads();
        {   // dDelta = P^T dO + K dS'
            float acc[4][4];
            zero_acc(acc);
            const int m0 = 16 * (warp & 3), n0 = 32 * (warp >> 2);
            warp_mma<4, true, true>(acc, sh + L::P, LH, st + L::DO, LH, m0, n0, kC, lane);
            warp_mma<4, false, true>(acc, st + L::K, LW, dsb, LH, m0, n0, kD, lane);
            for_acc(acc, m0, n0, lane, [&](int r, int c2, float& v) { sh[L::DD + r * LH + c2] = __float2bfloat16_rn(v); });
        }
        __syncthreads();
        {   // -dR = -(T^T dDelta)
            float acc[4][4];
            zero_acc(acc);
            const int m0 = 16 * (warp & 3), n0 = 32 * (warp >> 2);
            warp_mma<4, true, true>(acc, st + L::T, LH, sh + L::DD, LH, m0, n0, kC, lane);
            for_acc(acc, m0, n0, lane, [&](int r, int c2, float& v) { sh[L::NR + r * LH + c2] = __float2bfloat16_rn(-v); });
        }
        __syncthreads();
        // dS += Q^T dO + K^T (-dR): rows 16 w .. of the 128 x 64 half
        warp_mma<8, true, true>(ds, st + L::Q, LW, st + L::DO, LH, 16 * warp, 0, kC, lane);
        warp_mma<8, true, true>(ds, st + L::K, LW, sh + L::NR, LH, 16 * warp, 0, kC, lane);
        __syncthreads();                                   // every read of dS' and of stage c is done
        write_ds();
    }
    if (dS0) for_acc(ds, 16 * warp, 0, lane, [&](int r, int c, float& v) { dS0[((size_t)bh * kD + r) * kD + col0 + c] = v; });
}

// ============================================================================ per-chunk gradients
// One CTA (8 warps) per (stream, chunk).  64 x 128 products: warp w -> rows 16 (w % 4), columns
// 64 (w / 4); 64 x 64 products: columns 32 (w / 4).  Shared memory: the S tile's bytes host
// the solve's fp32 A and scratch before S is loaded, and dT and dX X^T after its last use.
struct TileSmem {
    // bf16 tiles (element offsets)
    static constexpr int K = 0, Q = K + kC * LW, VR = Q + kC * LW, DO = VR + kC * LW, DEL = DO + kC * LW;
    static constexpr int S = DEL + kC * LW;              // 128 x LW: S (fp32 A and scratch around it)
    static constexpr int DSP = S + kD * LW;              // 128 x LW: dS', later dDelta (rows 0-63), -dR (64-127)
    static constexpr int TB = DSP + kD * LW;             // 64 x LH: T
    static constexpr int PB = TB + kC * LH;              // 64 x LH: P, later dP
    static constexpr int GB = PB + kC * LH;              // 64 x LH: G, later dG + dG^T
    static constexpr int BF16_END = GB + kC * LH;
    // fp32 (float offsets from the end of the bf16 part)
    static constexpr int FX = 0;
    static constexpr int ALPHA = FX + kC * LF, BETA = ALPHA + kC, DALPHA = BETA + kC, LAM = DALPHA + kC, ONES = LAM + kC;
    static constexpr int F32_END = ONES + kC;
    static constexpr size_t BYTES = sizeof(bf16) * BF16_END + sizeof(float) * F32_END;
    static_assert(2 * kC * LF * sizeof(float) <= kD * LW * sizeof(bf16), "fp32 A and scratch fit in the S tile");
    static_assert(BYTES <= 232448, "shared memory");
};

__global__ void __launch_bounds__(256, 1)
bwd_tile_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
                const bf16* __restrict__ beta, const bf16* __restrict__ dO, const bf16* __restrict__ states,
                const bf16* __restrict__ dSp, float* __restrict__ dq, float* __restrict__ dk, float* __restrict__ dv,
                float* __restrict__ dbeta, int T, int rule) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    using L = TileSmem;
    bf16* sh = reinterpret_cast<bf16*>(smem_raw);
    float* sf = reinterpret_cast<float*>(smem_raw + sizeof(bf16) * L::BF16_END);
    float* fA = reinterpret_cast<float*>(sh + L::S);      // aliases the S tile (see above)
    float* fY = fA + kC * LF;
    float* fX = sf + L::FX;
    float *al = sf + L::ALPHA, *bt = sf + L::BETA, *dal = sf + L::DALPHA, *lam = sf + L::LAM, *ones = sf + L::ONES;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nchunks = (T + kC - 1) / kC;
    const long tile = blockIdx.x;
    const long bh = tile / nchunks;
    const int c = (int)(tile % nchunks);
    const int nv = min(kC, T - c * kC);
    const size_t row0 = (size_t)bh * T + (size_t)c * kC;
    const int wm = 16 * (warp & 3);                  // this warp's row block
    const int wn = 64 * (warp >> 2), wn64 = 32 * (warp >> 2);

    load_tile(sh + L::K, LW, k + row0 * kD, kD, kC, kD, nv, tid, 256);
    cp_async_commit();
    load_tile(sh + L::Q, LW, q + row0 * kD, kD, kC, kD, nv, tid, 256);
    load_tile(sh + L::VR, LW, v + row0 * kD, kD, kC, kD, nv, tid, 256);
    load_tile(sh + L::DO, LW, dO + row0 * kD, kD, kC, kD, nv, tid, 256);
    load_tile(sh + L::DSP, LW, dSp + (size_t)tile * kD * kD, kD, kD, kD, kD, tid, 256);
    cp_async_commit();
    if (tid < kC) {
        bt[tid] = tid < nv ? __bfloat162float(beta[row0 + tid]) : 0.f;
        ones[tid] = 1.f;
        dal[tid] = 0.f;
    }
    cp_async_wait<1>();
    __syncthreads();                                 // K landed
    {   // G = K K^T (fp32 into fY), lambda from its diagonal
        float acc[4][4];
        zero_acc(acc);
        warp_mma<4, false, false>(acc, sh + L::K, LW, sh + L::K, LW, wm, wn64, kD, lane);
        for_acc(acc, wm, wn64, lane, [&](int r, int c2, float& x) {
            fY[r * LF + c2] = x;
            sh[L::GB + r * LH + c2] = __float2bfloat16_rn(x);
        });
    }
    __syncthreads();
    if (tid < kC) {
        lam[tid] = fY[tid * LF + tid];
        al[tid] = rule_alpha(rule, bt[tid], lam[tid]);
    }
    __syncthreads();
    for (int e = tid; e < kC * kC; e += 256) {       // A = strict_tril(diag(alpha) G)
        const int r = e >> 6, s2 = e & 63;
        fA[r * LF + s2] = s2 < r ? al[r] * fY[r * LF + s2] : 0.f;
    }
    __syncthreads();
    ut_inverse64<256>(fA, ones, fX, fY, LF, tid);    // X = (I + A)^{-1} (ends with a barrier)
    // the S tile is free of the solve: load the chunk's entering state
    load_tile(sh + L::S, LW, states + (size_t)tile * kD * kD, kD, kD, kD, kD, tid, 256);
    cp_async_commit();
    for (int e = tid; e < kC * kC; e += 256) {       // T = X diag(alpha), bf16
        const int r = e >> 6, s2 = e & 63;
        sh[L::TB + r * LH + s2] = __float2bfloat16_rn(fX[r * LF + s2] * al[s2]);
    }
    cp_async_wait<0>();
    __syncthreads();                                 // everything landed, T written
    float dqa[8][4], dka[8][4];
    zero_acc(dqa);
    zero_acc(dka);
    {   // R = V - K S (bf16 over V);  dQ = dO S^T (+ dP K below)
        float acc[8][4];
        zero_acc(acc);
        warp_mma<8, false, true>(acc, sh + L::K, LW, sh + L::S, LW, wm, wn, kD, lane);
        warp_mma<8, false, false>(dqa, sh + L::DO, LW, sh + L::S, LW, wm, wn, kD, lane);
        for_acc(acc, wm, wn, lane, [&](int r, int c2, float& x) {
            bf16* p = sh + L::VR + r * LW + c2;
            *p = __float2bfloat16_rn(__bfloat162float(*p) - x);
        });
    }
    {   // P = tril_incl(Q K^T)
        float acc[4][4];
        zero_acc(acc);
        warp_mma<4, false, false>(acc, sh + L::Q, LW, sh + L::K, LW, wm, wn64, kD, lane);
        for_acc(acc, wm, wn64, lane, [&](int r, int c2, float& x) {
            sh[L::PB + r * LH + c2] = __float2bfloat16_rn(c2 <= r ? x : 0.f);
        });
    }
    __syncthreads();
    {   // Delta = T R
        float acc[8][4];
        zero_acc(acc);
        warp_mma<8, false, true>(acc, sh + L::TB, LH, sh + L::VR, LW, wm, wn, kC, lane);
        for_acc(acc, wm, wn, lane, [&](int r, int c2, float& x) { sh[L::DEL + r * LW + c2] = __float2bfloat16_rn(x); });
    }
    __syncthreads();
    {   // dDelta = P^T dO + K dS';  dK = Delta dS'^T (+ more below).  dS' is then dead.
        float acc[8][4];
        zero_acc(acc);
        warp_mma<8, true, true>(acc, sh + L::PB, LH, sh + L::DO, LW, wm, wn, kC, lane);
        warp_mma<8, false, true>(acc, sh + L::K, LW, sh + L::DSP, LW, wm, wn, kD, lane);
        warp_mma<8, false, false>(dka, sh + L::DEL, LW, sh + L::DSP, LW, wm, wn, kD, lane);
        __syncthreads();
        for_acc(acc, wm, wn, lane, [&](int r, int c2, float& x) { sh[L::DSP + r * LW + c2] = __float2bfloat16_rn(x); });
    }
    __syncthreads();
    const bf16* dD = sh + L::DSP;                    // dDelta, rows 0-63 of the old dS' tile
    bf16* nR = sh + L::DSP + kC * LW;                // -dR, rows 64-127 of the old dS' tile
    {   // dR = T^T dDelta = dV, and -dR (bf16) for dK -= dR S^T
        float acc[8][4];
        zero_acc(acc);
        warp_mma<8, true, true>(acc, sh + L::TB, LH, dD, LW, wm, wn, kC, lane);
        for_acc(acc, wm, wn, lane, [&](int r, int c2, float& x) {
            if (r < nv) dv[(row0 + r) * kD + c2] = x;
            nR[r * LW + c2] = __float2bfloat16_rn(-x);
        });
    }
    {   // dP = tril_incl(dO Delta^T) over P (dead since dDelta)
        float acc[4][4];
        zero_acc(acc);
        warp_mma<4, false, false>(acc, sh + L::DO, LW, sh + L::DEL, LW, wm, wn64, kD, lane);
        for_acc(acc, wm, wn64, lane, [&](int r, int c2, float& x) {
            sh[L::PB + r * LH + c2] = __float2bfloat16_rn(c2 <= r ? x : 0.f);
        });
    }
    __syncthreads();
    // dK -= dR S^T (S's last use);  dQ += dP K
    warp_mma<8, false, false>(dka, nR, LW, sh + L::S, LW, wm, wn, kD, lane);
    warp_mma<8, false, true>(dqa, sh + L::PB, LH, sh + L::K, LW, wm, wn, kC, lane);
    for_acc(dqa, wm, wn, lane, [&](int r, int c2, float& x) {
        if (r < nv) dq[(row0 + r) * kD + c2] = x;
    });
    float dta[4][4];                                 // dT = dDelta R^T
    zero_acc(dta);
    warp_mma<4, false, false>(dta, dD, LW, sh + L::VR, LW, wm, wn64, kD, lane);
    __syncthreads();                                 // S is dead: fp32 dT over it
    for_acc(dta, wm, wn64, lane, [&](int r, int c2, float& x) { fA[r * LF + c2] = x; });
    __syncthreads();
    // ---- through T = X diag(alpha) and X = (I + A)^{-1}, fp32 on CUDA cores
    if (tid < kC) {                                  // dalpha_j = sum_i dT_ij X_ij
        float sacc = 0.f;
        for (int i = 0; i < kC; ++i) sacc = fmaf(fA[i * LF + tid], fX[i * LF + tid], sacc);
        dal[tid] = sacc;
    }
    __syncthreads();
    for (int e = tid; e < kC * kC; e += 256) {       // dX = dT diag(alpha), in place
        const int r = e >> 6, s2 = e & 63;
        fA[r * LF + s2] *= al[s2];
    }
    __syncthreads();
    // 64 x 64 x 64 fp32 products on CUDA cores, 4 x 4 outputs per thread (rows 4 (tid / 16),
    // columns 4 (tid % 16)): per k, 4 + 4 shared loads for 16 FMAs
    const int r4 = 4 * (tid >> 4), c4 = 4 * (tid & 15);
    {   // W = dX X^T into fY:  W[r][c] = sum_m dX[r][m] X[c][m]
        float w[4][4] = {};
        for (int m = 0; m < kC; ++m) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = fA[(r4 + i) * LF + m];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = fX[(c4 + j) * LF + m];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) w[i][j] = fmaf(a[i], b[j], w[i][j]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) fY[(r4 + i) * LF + c4 + j] = w[i][j];
    }
    __syncthreads();
    {   // dA = strict_tril(-X^T W) over fA:  dA[r][c] = -sum_m X[m][r] W[m][c];  dalpha_r += sum_{s<r} dA_rs G_rs
        float w[4][4] = {};
        for (int m = 0; m < kC; ++m) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = fX[m * LF + r4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = fY[m * LF + c4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) w[i][j] = fmaf(a[i], b[j], w[i][j]);
        }
        // (fA, the dX tile, is not read here: it is overwritten at once)
        float part[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            part[i] = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = r4 + i, s2 = c4 + j;
                const float da = s2 < r ? -w[i][j] : 0.f;
                fA[r * LF + s2] = da;
                part[i] = fmaf(da, __bfloat162float(sh[L::GB + r * LH + s2]), part[i]);
            }
        }
        // the 16 column blocks of a row block sit in 16 consecutive lanes: sum over them
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int off = 1; off < 16; off <<= 1) part[i] += __shfl_xor_sync(0xffffffffu, part[i], off);
        }
        if ((tid & 15) == 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i) dal[r4 + i] += part[i];
        }
    }
    __syncthreads();
    for (int e = tid; e < kC * kC; e += 256) {       // dG + dG^T with dG = diag(alpha) dA, bf16 over G
        const int r = e >> 6, s2 = e & 63;
        const float x = (s2 < r ? al[r] * fA[r * LF + s2] : 0.f) + (r < s2 ? al[s2] * fA[s2 * LF + r] : 0.f);
        sh[L::GB + r * LH + s2] = __float2bfloat16_rn(x);
    }
    __syncthreads();
    // dK += dP^T Q + (dG + dG^T) K, then the gate's lambda term; dbeta
    warp_mma<8, true, true>(dka, sh + L::PB, LH, sh + L::Q, LW, wm, wn, kC, lane);
    warp_mma<8, false, true>(dka, sh + L::GB, LH, sh + L::K, LW, wm, wn, kC, lane);
    if (tid < kC) {
        float dadb, dadl;
        gate_derivatives(rule, bt[tid], lam[tid], al[tid], &dadb, &dadl);
        if (tid < nv) dbeta[row0 + tid] = dal[tid] * dadb;
        lam[tid] = 2.f * dal[tid] * dadl;            // the coefficient of k in dk's gate term
    }
    __syncthreads();
    for_acc(dka, wm, wn, lane, [&](int r, int c2, float& x) {
        if (r < nv) dk[(row0 + r) * kD + c2] = x + lam[r] * __bfloat162float(sh[L::K + r * LW + c2]);
    });
}
}  // namespace

size_t bwd_chunk_workspace_bytes(long BH, int T) {
    const long ntiles = BH * ((T + kC - 1) / kC);
    return (size_t)ntiles * (kC * kC + 2 * kD * kD) * sizeof(bf16);   // T, S and dS' per tile
}

cudaError_t launch_bwd_chunk(const void* q, const void* k, const void* v, const void* beta, const float* S0,
                             const void* dO, const float* dST, float* dq, float* dk, float* dv, float* dbeta,
                             float* dS0, long BH, int T, int rule, uint32_t* err, void* scratch, cudaStream_t stream) {
    const int nchunks = (T + kC - 1) / kC;
    const long ntiles = BH * nchunks;
    bf16* Tt = static_cast<bf16*>(scratch);
    bf16* states = Tt + (size_t)ntiles * kC * kC;
    bf16* dSp = states + (size_t)ntiles * kD * kD;
    // 1. UT transforms and the forward chain, storing every chunk's entering state
    SegPlan plan;
    plan.states = states;
    Seqs seqs{nullptr, nullptr, 0, 0, T, 0};
    cudaError_t e = launch_chunk_tc(q, k, v, beta, S0, nullptr, nullptr, seqs, BH, BH, T, ntiles, err, Tt, rule,
                                    stream, nullptr, plan);
    if (e != cudaSuccess) return e;
    // 2. the reverse chain
    static std::atomic<uint64_t> smem_chain{0}, smem_tile{0};
    e = set_smem_limit_once(bwd_chain_kernel, (int)ChainSmem::BYTES, smem_chain);
    if (e != cudaSuccess) return e;
    bwd_chain_kernel<<<(unsigned)(BH * 2), 256, ChainSmem::BYTES, stream>>>(
        (const bf16*)q, (const bf16*)k, (const bf16*)dO, Tt, dST, dSp, dS0, T);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // 3. every chunk's gradients
    e = set_smem_limit_once(bwd_tile_kernel, (int)TileSmem::BYTES, smem_tile);
    if (e != cudaSuccess) return e;
    bwd_tile_kernel<<<(unsigned)ntiles, 256, TileSmem::BYTES, stream>>>(
        (const bf16*)q, (const bf16*)k, (const bf16*)v, (const bf16*)beta, (const bf16*)dO, states, dSp, dq, dk, dv,
        dbeta, T, rule);
    return cudaGetLastError();
}

}  // namespace efla