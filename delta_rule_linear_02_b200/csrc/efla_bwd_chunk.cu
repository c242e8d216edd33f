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
//   1. the UT transforms keeping X = (I + A)^{-1} (fp32) beside T, and the forward chain
//      (efla_chunk_tc.cu) storing every chunk's entering state S (bf16) -- or, for training,
//      the same residuals saved by the forward (efla_chunk_fwd_save);
//   2. bwd_chain_kernel: one CTA per (stream, 64-column half of d_v) walks the chunks in
//      reverse, carrying its half of dS in the MMA accumulators (the columns of dS evolve
//      independently), and stores each chunk's dS' (bf16);
//   3. bwd_tile_kernel: one CTA per (stream, chunk), all chunks at once: every gradient of
//      the chunk from its S and dS'.
// Both kernels' bf16 products are tcgen05 MMAs (operands in shared memory, fp32 accumulators
// in tensor memory); only dA's two small fp32 products are TF32 mma.sync tiles.  Operands pass
// through bf16 as in the forward, so the gradients carry bf16-operand rounding (relative
// Frobenius error ~1e-2), not fp32's.
#include "efla_common.cuh"
#include "efla_kernels.h"
#include "efla_tma.cuh"
#include "efla_ut_tf32.cuh"
#include "sm100.cuh"

namespace efla {

namespace {
using bf16 = __nv_bfloat16;
constexpr int kD = 128, kC = 64;

// The extents of the buffers the two backward kernels address directly (checked builds test
// each access against them; see efla_common.cuh).
struct BwdSpans {
    Span beta, dq, dk, dv, dbeta, dst, ds0, x;
};

// ============================================================================ per-chunk gradients
// One CTA (8 warps) per (stream, chunk), every product on the 5th-generation tensor cores
// (tcgen05, bf16 operands in shared memory, fp32 accumulators in tensor memory).
//
// Products whose rows index d are computed transposed (M = 128 = d, N = 64 tokens): the
// accumulator then fills all 128 TMEM lanes, an N = 64 MMA costs less than an N = 128 one,
// and each epilogue thread owns one d-row of 64 tokens, which it writes as one 128-byte
// swizzled row (bf16) or, for the fp32 gradients, as one column of dq / dk / dv (a warp's
// 32 lanes are 32 consecutive d: 128 contiguous bytes per token).  Token x token products
// (G, P, dP, dT) are M = 64 or ride in the rows 64-127 of a stacked M = 128 product.
// Operand shapes (row convention, t and s tokens, i = d_k, j = d_v):
//   [G; P~] = [K; Q] K^T          R^T = V^T - S^T K^T          dQ^T = S dO^T + K^T dP^T
//   Delta^T = R^T T^T             dDelta^T = dO^T P + dS'^T K^T
//   dK^T = dS' Delta^T + S (-dR^T) + Q^T dP + K^T (dG + dG^T)
//   dR^T = dDelta^T T (= dV^T)    dP = tril_incl(dO Delta^T)   dT = dDelta R^T
// Shared-memory tiles are 128-byte swizzled rows of 64 elements: token-major tiles (K, Q, V,
// dO: 64 rows per 64-column atom) serve as K-major operands over d or MN-major ones over
// tokens, d-major tiles (S, dS', R^T, Delta^T, dDelta^T, -dR^T: 128 rows) the other way
// round, so no operand is ever transposed in memory.  X = (I + A)^{-1} (fp32) and T (bf16)
// come from the UT transform; the two 64^3 products of dA = strict_tril(-X^T dX X^T) run on
// the TF32 tensor path, dalpha and dG on CUDA cores.  Phases are sequential: one warp issues a
// phase's MMAs and commits them to one mbarrier; all warps wait (bounded), run the
// epilogue, and meet at a block barrier.
namespace tb {
constexpr uint32_t TILE = 8192;
constexpr uint32_t KQ = 0;                 // [K a0 | Q a0 | K a1 | Q a1]: rows 0-63 K, 64-127 Q of [K; Q]
constexpr uint32_t V = 32768;              // [V a0 | V a1]; later dT^T, dX^T, dA (fp32)
constexpr uint32_t DO = 49152;             // [dO a0 | dO a1]
constexpr uint32_t DSP = 65536;            // dS' [a0 | a1] (128 rows each); later dDelta^T and -dR^T
constexpr uint32_t SS = 98304;             // S [a0 | a1]
constexpr uint32_t TT = 131072;            // T (bf16 [t][s]); later X^T (fp32)
constexpr uint32_t PP = 139264;            // P, later dP (bf16 [t][s])
constexpr uint32_t RT = 147456;            // R^T (128 rows)
constexpr uint32_t DL = 164864;            // Delta^T (128 rows)
constexpr uint32_t DG = 181248;            // G (bf16 [t][s]), later dG + dG^T
constexpr int LX = 68;                     // row stride of the fp32 64 x 64 tiles (16-byte rows; the UT
                                           // transform's X arrives in this layout)
constexpr uint32_t F32 = 64 * LX * 4;      // bytes of one of them
constexpr uint32_t FX = 189440;            // X (fp32)
constexpr uint32_t FXT = TT;               // X^T
constexpr uint32_t FW = TT + F32;          // W = dX X^T
constexpr uint32_t FDT = V;                // dT^T, then dX^T, then dA
constexpr uint32_t FDA2 = FDT + F32;       // dA^T (over dO and the first dS' atom, both dead by then)
constexpr uint32_t SMALL = FX + F32;       // alpha, beta, dalpha, lambda, (unused), two partial sums (fp32 [64] each)
constexpr uint32_t BAR = SMALL + 7 * 256;  // mbarriers: the tile's inputs, MMA commits
constexpr uint32_t MISC = BAR + 6 * 8;     // TMEM base, abort flag
constexpr uint32_t SMEM_BYTES = MISC + 16 + 1024;
static_assert(64 * LX * 4 == kUtXBytes, "X as the UT transform writes it");
static_assert(FDT + F32 <= DSP && FW + F32 <= DG && FDA2 + F32 <= DSP + 2 * TILE,
              "fp32 tiles stay inside dead regions");
static_assert(SMEM_BYTES <= 232448, "shared memory");
// TMEM columns (fp32 accumulators, 64 columns each)
constexpr uint32_t C_GP = 0, C_SK = 64, C_DQ = 128, C_DL = 192, C_DD = 256, C_DK = 320, C_DR = 384, C_COLS = 512;
// the tile's inputs, on five barriers in the order the first products need them
enum : int { L_KQ = 0, L_VTX = 2, L_S = 3, L_DSP = 4, L_DO = 5 };   // (1: the MMA commits)
constexpr uint32_t KQ_BYTES = 32768, S_BYTES = 32768, DSP_BYTES = 32768, DO_BYTES = 16384;
constexpr uint32_t VTX_BYTES = 16384 + 8192 + 64 * 68 * 4;          // V, T, X: from the second epilogue on

// nk k-steps of K = 16 with A and B in shared memory; operand k-step ks starts at
// base + (ks / 4) * atom + (ks % 4) * step (K-major: step 32 bytes inside a 64-column atom;
// MN-major: step 16 rows = 2048 bytes, atom 64 rows = 8192 bytes; lbo = distance between
// 64-element MN blocks of an MN-major operand).  Called by a whole converged warp; the lane
// elect.sync picks builds the descriptors and issues all nk MMAs (one branch per product:
// about half the code of an elect.sync per MMA, in kernels whose phases each run once).
__device__ __forceinline__ void mma_ss(uint32_t d, uint32_t a, uint32_t a_atom, uint32_t a_step, uint32_t a_lbo,
                                       uint32_t b, uint32_t b_atom, uint32_t b_step, uint32_t b_lbo, uint32_t idesc,
                                       int nk, bool acc) {
    if (sm100::elect_one()) {
        const uint64_t da = sm100::sdesc_sw128(a, a_lbo, 1024), db = sm100::sdesc_sw128(b, b_lbo, 1024);
#pragma unroll
        for (int ks = 0; ks < nk; ++ks)
            sm100::mma_bf16(d, da + (((ks >> 2) * a_atom + (ks & 3) * a_step) >> 4),
                            db + (((ks >> 2) * b_atom + (ks & 3) * b_step) >> 4), idesc, acc || ks > 0);
    }
    __syncwarp();
}
constexpr uint32_t K_MAJ = 0, MN_MAJ = 1;
__host__ __device__ constexpr uint32_t idesc(int M, uint32_t a, uint32_t b) {
    return sm100::idesc_bf16(M, 64, a == MN_MAJ, b == MN_MAJ);
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
// 32 floats -> row `r`, 16-byte chunks c0 .. c0 + 3 of a 128-byte-swizzled tile at `tile`
__device__ __forceinline__ void st_row32(uint8_t* tile, uint32_t r, uint32_t c0, const float* v) {
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        uint4 u;
        u.x = pack2(v[8 * m], v[8 * m + 1]);
        u.y = pack2(v[8 * m + 2], v[8 * m + 3]);
        u.z = pack2(v[8 * m + 4], v[8 * m + 5]);
        u.w = pack2(v[8 * m + 6], v[8 * m + 7]);
        *reinterpret_cast<uint4*>(tile + sm100::sw128_off(r, c0 + m)) = u;
    }
}
// element (r, c) of a token-major tile of 64-column atoms `atom` bytes apart
__device__ __forceinline__ float ld_tok(const uint8_t* tile, uint32_t atom, int r, int c) {
    const uint8_t* p = tile + (c >> 6) * atom + sm100::sw128_off(r, (c & 63) >> 3) + (c & 7) * 2;
    return __bfloat162float(*reinterpret_cast<const bf16*>(p));
}

// C (64 x 64) = sum_m P[m][r] Q[m][c] for the fp32 tiles P, Q (row stride LX), on the TF32
// tensor path (mma.sync m16n8k8; operands rounded to TF32, 10-bit mantissa, finer than the
// bf16 operands of the other products).  Warp w: rows 16 (w % 4) .. + 15, columns
// 32 (w / 4) .. + 31 (four 8-column tiles); acc[nt] holds C[r0 + g][c] and C[r0 + g + 8][c]
// for c = c0 + 8 nt + 2 t, + 1 (g = lane / 4, t = lane % 4).  The k slots t and t + 4 of a
// k-step take m = 2 t and 2 t + 1: with LX = 4 (mod 32) every operand load of a warp then
// hits 32 distinct banks.
__device__ __forceinline__ void gemm_tn64_tc(const float* __restrict__ P, const float* __restrict__ Q,
                                             float (&acc)[4][4], int warp, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const int r0 = 16 * (warp & 3), c0 = 32 * (warp >> 2);
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
#pragma unroll 2
    for (int k0 = 0; k0 < 64; k0 += 8) {
        const float* p0 = P + (k0 + 2 * t) * LX + r0 + g;
        const float av[4] = {p0[0], p0[8], p0[LX], p0[LX + 8]};
        uint32_t a[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) a[e] = ut::to_tf32(av[e]);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const float* q0 = Q + (k0 + 2 * t) * LX + c0 + 8 * nt + g;
            uint32_t b[2] = {ut::to_tf32(q0[0]), ut::to_tf32(q0[LX])};
            ut::mma_tf32(acc[nt], a, b);
        }
    }
}
}  // namespace tb

__global__ void __launch_bounds__(256, 1)
bwd_tile_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                const __grid_constant__ CUtensorMap tm_s, const __grid_constant__ CUtensorMap tm_dsp,
                const __grid_constant__ CUtensorMap tm_t, const float* __restrict__ Xg,
                const bf16* __restrict__ beta, float* __restrict__ dq, float* __restrict__ dk, float* __restrict__ dv,
                float* __restrict__ dbeta, int T, int rule, uint32_t* __restrict__ err, unsigned long long limit_ns,
                BwdSpans spans) {
    using namespace tb;
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + BAR);    // 1: MMA commits, the others the tile's inputs
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + MISC);
    volatile int* abort = reinterpret_cast<volatile int*>(sm + MISC + 4);
    float* fX = reinterpret_cast<float*>(sm + FX);
    float* fXT = reinterpret_cast<float*>(sm + FXT);
    float* fW = reinterpret_cast<float*>(sm + FW);
    float* fdT = reinterpret_cast<float*>(sm + FDT);
    float* fdA2 = reinterpret_cast<float*>(sm + FDA2);
    float* al = reinterpret_cast<float*>(sm + SMALL);
    float *bt = al + 64, *dal = al + 128, *lam = al + 192, *part = al + 320;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3, h = warp >> 2;                    // TMEM lane quarter, column half
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    const int row = 32 * q + lane;                            // accumulator row (M = 128)
    const int nchunks = (T + 63) / 64;
    const long tile = blockIdx.x;
    const long bh = tile / nchunks;
    const int c = (int)(tile % nchunks), t0 = c * 64;
    const int nv = min(64, T - t0);
    const size_t row0 = (size_t)bh * T + t0;

    if (tid == 0) {
        for (int i = 0; i < 6; ++i) mbar_init(bar + i, 1);
        *abort = 0;
        fence_mbar_init();
        // each of the first products starts once its operands have landed; V, T and X land
        // while those products run
        mbar_arrive_expect_tx(bar + L_KQ, KQ_BYTES);
        mbar_arrive_expect_tx(bar + L_S, S_BYTES);
        mbar_arrive_expect_tx(bar + L_DSP, DSP_BYTES);
        mbar_arrive_expect_tx(bar + L_DO, DO_BYTES);
        mbar_arrive_expect_tx(bar + L_VTX, VTX_BYTES);
        tma_load_3d(sm + KQ, &tm_k, bar + L_KQ, 0, t0, (int)bh);
        tma_load_3d(sm + KQ + 2 * TILE, &tm_k, bar + L_KQ, 64, t0, (int)bh);
        tma_load_3d(sm + KQ + TILE, &tm_q, bar + L_KQ, 0, t0, (int)bh);
        tma_load_3d(sm + KQ + 3 * TILE, &tm_q, bar + L_KQ, 64, t0, (int)bh);
        tma_load_2d(sm + SS, &tm_s, bar + L_S, 0, (int)(tile * 128));
        tma_load_2d(sm + SS + 2 * TILE, &tm_s, bar + L_S, 64, (int)(tile * 128));
        tma_load_2d(sm + DSP, &tm_dsp, bar + L_DSP, 0, (int)(tile * 128));
        tma_load_2d(sm + DSP + 2 * TILE, &tm_dsp, bar + L_DSP, 64, (int)(tile * 128));
        tma_load_3d(sm + DO, &tm_do, bar + L_DO, 0, t0, (int)bh);
        tma_load_3d(sm + DO + TILE, &tm_do, bar + L_DO, 64, t0, (int)bh);
        uint64_t* rest = bar + L_VTX;
        tma_load_3d(sm + V, &tm_v, rest, 0, t0, (int)bh);
        tma_load_3d(sm + V + TILE, &tm_v, rest, 64, t0, (int)bh);
        tma_load_2d(sm + TT, &tm_t, rest, 0, (int)(tile * 64));
        const float* xs = Xg + tile * (64 * LX);
        if (span_ok(err, spans.x, xs, 64 * LX * 4)) bulk_load(sm + FX, xs, 64 * LX * 4, rest);
    }
    const float beta_t = tid < nv && span_ok(err, spans.beta, beta + row0 + tid, 2)   // in flight during the setup
                             ? __bfloat162float(beta[row0 + tid]) : 0.f;
    if (warp == 0) {
        tmem_alloc(tmem_slot, C_COLS);
        tmem_relinquish();
    }
    if (tid < 64) {
        bt[tid] = beta_t;
        dal[tid] = 0.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;
    // bounded waits; once one has run out every later wait is skipped (the outputs are then
    // invalid and the error word says so), so the block still reaches every barrier
    auto wait = [&](int i, uint32_t parity) {
        if (*abort) return;
        if (!mbar_wait(bar + i, parity, limit_ns)) *abort = 1;
        tc_fence_after();
    };
    uint32_t mma_phase = 0;
    auto wait_mma = [&]() { wait(1, mma_phase & 1); ++mma_phase; };
    auto commit = [&]() { mma_commit_elect(bar + 1); };
    // the next phase's operands written by this block's threads -> visible to the tensor core
    auto handoff = [&]() {
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    };

    // ---- 1. [G; P~] = [K; Q] K^T;  dDelta^T = dS'^T K^T (+ dO^T P below);  S^T K^T;  dQ^T = S dO^T
    //      (every thread waits on each input barrier; warp 0 issues each product as its operands land)
    wait(L_KQ, 0);
    if (warp == 0)
        mma_ss(tm + C_GP, sb + KQ, 2 * TILE, 32, 16, sb + KQ, 2 * TILE, 32, 16, idesc(128, K_MAJ, K_MAJ), 8, false);
    wait(L_S, 0);
    if (warp == 0)
        mma_ss(tm + C_SK, sb + SS, TILE, 2048, 2 * TILE, sb + KQ, 2 * TILE, 32, 16, idesc(128, MN_MAJ, K_MAJ), 8,
               false);
    wait(L_DSP, 0);
    if (warp == 0)
        mma_ss(tm + C_DD, sb + DSP, TILE, 2048, 2 * TILE, sb + KQ, 2 * TILE, 32, 16, idesc(128, MN_MAJ, K_MAJ), 8,
               false);
    wait(L_DO, 0);
    if (warp == 0) {
        mma_ss(tm + C_DQ, sb + SS, 2 * TILE, 32, 16, sb + DO, TILE, 32, 16, idesc(128, K_MAJ, K_MAJ), 8, false);
        commit();
    }
    wait_mma();
    float g[32];
    tmem_ld32_wait(tm + lane_off + C_GP + 32 * h, g);
    if (q < 2) {          // G row `row`: bf16 copy, lambda and alpha from its diagonal
        st_row32(sm + DG, row, 4 * h, g);
        if (q == h) {
            float dg = 0.f;
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (j == lane) dg = g[j];
            lam[row] = dg;
            al[row] = rule_alpha(rule, bt[row], dg);
        }
    } else {              // P = tril_incl(Q K^T), query row t = row - 64
        const int t = row - 64;
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (32 * h + j > t) g[j] = 0.f;
        st_row32(sm + PP, t, 4 * h, g);
    }
    handoff();
    // ---- 2. dDelta^T += dO^T P;  R^T = V^T - S^T K^T.  T and X = (I + A)^{-1} come from the
    //         UT transform of the forward (its fp32 X and bf16 T), not from a solve here.
    if (warp == 0) {
        mma_ss(tm + C_DD, sb + DO, TILE, 2048, TILE, sb + PP, TILE, 2048, TILE, idesc(128, MN_MAJ, MN_MAJ), 4, true);
        commit();
    }
    {
        wait_mma();       // dO^T P has landed
        wait(L_VTX, 0);   // V, T and X have landed
        float r[32];
        tmem_ld32_wait(tm + lane_off + C_SK + 32 * h, r);
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = ld_tok(sm + V, TILE, 32 * h + j, row) - r[j];
        st_row32(sm + RT, row, 4 * h, r);
    }
    handoff();
    // ---- 3. Delta^T = R^T T^T
    if (warp == 0) {
        mma_ss(tm + C_DL, sb + RT, 0, 32, 16, sb + TT, 0, 32, 16, idesc(128, K_MAJ, K_MAJ), 4, false);
        commit();
    }
    wait_mma();
    {
        float x[32];
        tmem_ld32_wait(tm + lane_off + C_DL + 32 * h, x);
        st_row32(sm + DL, row, 4 * h, x);
    }
    handoff();
    // ---- 4. dK^T = dS' Delta^T;  dP~ = dO Delta^T (M = 64)
    if (warp == 0) {
        mma_ss(tm + C_DK, sb + DSP, 2 * TILE, 32, 16, sb + DL, TILE, 2048, TILE, idesc(128, K_MAJ, MN_MAJ), 8, false);
        mma_ss(tm + C_GP, sb + DO, TILE, 32, 16, sb + DL, TILE, 2048, TILE, idesc(64, K_MAJ, MN_MAJ), 8, false);
        commit();
    }
    wait_mma();
    {   // dDelta^T (dS' is dead) -> DSP rows 0-127;  dP = tril_incl(dP~) (rows 16 q + lane, lanes < 16)
        float x[32];
        tmem_ld32_wait(tm + lane_off + C_DD + 32 * h, x);
        st_row32(sm + DSP, row, 4 * h, x);
        tmem_ld32_wait(tm + lane_off + C_GP + 32 * h, x);
        if (lane < 16) {
            const int t = 16 * q + lane;
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (32 * h + j > t) x[j] = 0.f;
            st_row32(sm + PP, t, 4 * h, x);
        }
    }
    handoff();
    // ---- 5. dR^T = dDelta^T T;  dT = dDelta R^T (M = 64);  dQ^T += K^T dP^T;  dK^T += Q^T dP
    if (warp == 0) {
        mma_ss(tm + C_DR, sb + DSP, 0, 32, 16, sb + TT, 0, 2048, TILE, idesc(128, K_MAJ, MN_MAJ), 4, false);
        mma_ss(tm + C_SK, sb + DSP, TILE, 2048, TILE, sb + RT, TILE, 2048, TILE, idesc(64, MN_MAJ, MN_MAJ), 8, false);
        mma_ss(tm + C_DQ, sb + KQ, 0, 2048, 2 * TILE, sb + PP, 0, 32, 16, idesc(128, MN_MAJ, K_MAJ), 4, true);
        mma_ss(tm + C_DK, sb + KQ + TILE, 0, 2048, 2 * TILE, sb + PP, 0, 2048, TILE, idesc(128, MN_MAJ, MN_MAJ), 4,
               true);
        commit();
    }
    wait_mma();
    {
        float x[32], y[32], z[32];
        tmem_ld32x3_wait(tm + lane_off + C_DR + 32 * h, tm + lane_off + C_DQ + 32 * h, tm + lane_off + C_SK + 32 * h,
                         x, y, z);
        // dV = dR: dv[token][j] for this thread's j = row (a warp stores 32 consecutive floats)
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (32 * h + j < nv && span_ok(err, spans.dv, dv + (row0 + 32 * h + j) * 128 + row, 4))
                dv[(row0 + 32 * h + j) * 128 + row] = x[j];
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] = -x[j];
        st_row32(sm + DSP + 2 * TILE, row, 4 * h, x);   // -dR^T, over dS' atom 1
        // dQ = (S dO^T + K^T dP^T)^T
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (32 * h + j < nv && span_ok(err, spans.dq, dq + (row0 + 32 * h + j) * 128 + row, 4))
                dq[(row0 + 32 * h + j) * 128 + row] = y[j];
        // dT, stored transposed (fp32): dT^T[s][t] for this thread's row t = 16 q + lane
        if (lane < 16) {
            const int t = 16 * q + lane;
#pragma unroll
            for (int j = 0; j < 32; ++j) fdT[(32 * h + j) * LX + t] = z[j];
        }
    }
    {   // X^T (fp32): thread -> column c of X, rows 16 rb .. + 15; a warp reads 32 consecutive
        // columns of a row (one wavefront) and writes 16-byte pieces of 32 rows of X^T that are
        // LX = 4 (mod 32) words apart (conflict-free)
        const int c = tid & 63, rb = tid >> 6;
#pragma unroll
        for (int r = 16 * rb; r < 16 * rb + 16; r += 4)
            *reinterpret_cast<float4*>(fXT + c * LX + r) =
                make_float4(fX[r * LX + c], fX[(r + 1) * LX + c], fX[(r + 2) * LX + c], fX[(r + 3) * LX + c]);
    }
    handoff();
    // ---- 6. dK^T += S (-dR^T), while the CUDA cores go through T = X diag(alpha)
    if (warp == 0) {
        mma_ss(tm + C_DK, sb + SS, 2 * TILE, 32, 16, sb + DSP + 2 * TILE, TILE, 2048, TILE,
               idesc(128, K_MAJ, MN_MAJ), 8, true);
        commit();
    }
    // ---- 7. through T = X diag(alpha) and X = (I + A)^{-1}, fp32 on CUDA cores
    {   // dalpha_s = sum_t dT_ts X_ts;  dX^T = diag(alpha) dT^T, in place.  Row s = tid / 4,
        // a quarter of its 64 entries per thread (columns 8 u .. 8 u + 7 and 32 more, u = tid % 4:
        // the 16-byte pieces of the two rows that 8 lanes touch then fall in 8 different bank
        // groups), the four partial sums added by shuffles.
        const int srow = tid >> 2, u = tid & 3;
        const float a = al[srow];
        float sacc = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = 8 * u + 4 * (i & 1) + 32 * (i >> 1);
            float4 d4 = *reinterpret_cast<const float4*>(fdT + srow * LX + t);
            const float4 x4 = *reinterpret_cast<const float4*>(fXT + srow * LX + t);
            sacc = fmaf(d4.x, x4.x, fmaf(d4.y, x4.y, fmaf(d4.z, x4.z, fmaf(d4.w, x4.w, sacc))));
            d4.x *= a; d4.y *= a; d4.z *= a; d4.w *= a;
            *reinterpret_cast<float4*>(fdT + srow * LX + t) = d4;
        }
        sacc += __shfl_xor_sync(0xffffffffu, sacc, 1);
        sacc += __shfl_xor_sync(0xffffffffu, sacc, 2);
        if ((tid & 3) == 0) dal[srow] = sacc;
    }
    __syncthreads();
    const int g8 = lane >> 2, t4 = lane & 3, r0 = 16 * (warp & 3), c0 = 32 * (warp >> 2);
    {   // W = dX X^T:  W[r][c] = sum_m dX^T[m][r] X^T[m][c]
        float w[4][4];
        gemm_tn64_tc(fdT, fXT, w, warp, lane);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const int cc = c0 + 8 * nt + 2 * t4;
            *reinterpret_cast<float2*>(fW + (r0 + g8) * LX + cc) = make_float2(w[nt][0], w[nt][1]);
            *reinterpret_cast<float2*>(fW + (r0 + g8 + 8) * LX + cc) = make_float2(w[nt][2], w[nt][3]);
        }
    }
    __syncthreads();
    {   // dA = strict_tril(-X^T W) over dX^T:  dA[r][c] = -sum_m X[m][r] W[m][c];
        // dalpha_r += sum_{s<r} dA_rs G_rs (this warp's 32 columns, then the two halves)
        float w[4][4];
        gemm_tn64_tc(fX, fW, w, warp, lane);
        float p0 = 0.f, p1 = 0.f;
        const int ra = r0 + g8, rb = r0 + g8 + 8;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const int cc = c0 + 8 * nt + 2 * t4;
            const float a0 = cc < ra ? -w[nt][0] : 0.f, a1 = cc + 1 < ra ? -w[nt][1] : 0.f;
            const float b0 = cc < rb ? -w[nt][2] : 0.f, b1 = cc + 1 < rb ? -w[nt][3] : 0.f;
            *reinterpret_cast<float2*>(fdT + ra * LX + cc) = make_float2(a0, a1);
            *reinterpret_cast<float2*>(fdT + rb * LX + cc) = make_float2(b0, b1);
            fdA2[cc * LX + ra] = a0;          // the transpose, for dG^T below (a warp's 32 stores
            fdA2[(cc + 1) * LX + ra] = a1;    // of one instruction hit 32 different banks)
            fdA2[cc * LX + rb] = b0;
            fdA2[(cc + 1) * LX + rb] = b1;
            p0 = fmaf(a0, ld_tok(sm + DG, 0, ra, cc), fmaf(a1, ld_tok(sm + DG, 0, ra, cc + 1), p0));
            p1 = fmaf(b0, ld_tok(sm + DG, 0, rb, cc), fmaf(b1, ld_tok(sm + DG, 0, rb, cc + 1), p1));
        }
        // the four lanes of a row group hold its 32 columns: sum over them
        p0 += __shfl_xor_sync(0xffffffffu, p0, 1);
        p0 += __shfl_xor_sync(0xffffffffu, p0, 2);
        p1 += __shfl_xor_sync(0xffffffffu, p1, 1);
        p1 += __shfl_xor_sync(0xffffffffu, p1, 2);
        if (t4 == 0) {
            part[(warp >> 2) * 64 + ra] = p0;
            part[(warp >> 2) * 64 + rb] = p1;
        }
    }
    __syncthreads();
    if (tid < 64) dal[tid] += part[tid] + part[64 + tid];
    {   // dG + dG^T with dG = diag(alpha) dA (dA strictly lower, zero elsewhere), bf16 over G:
        // thread -> row r = tid / 4, columns 8 u .. 8 u + 7 and 8 u + 32 .. 8 u + 39 (u = tid % 4),
        // rows of dA and of dA^T read as 16-byte pieces in 8 different bank groups per 8 lanes
        const int r = tid >> 2, u = tid & 3;
        const float ar = al[r];
#pragma unroll
        for (int hlf = 0; hlf < 2; ++hlf) {
            const int sb0 = 8 * u + 32 * hlf;
            float x[8];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int s2 = sb0 + 4 * i;
                const float4 a4 = *reinterpret_cast<const float4*>(fdT + r * LX + s2);    // dA[r][s2 ..]
                const float4 b4 = *reinterpret_cast<const float4*>(fdA2 + r * LX + s2);   // dA[s2 ..][r]
                const float4 al4 = *reinterpret_cast<const float4*>(al + s2);
                x[4 * i] = fmaf(ar, a4.x, al4.x * b4.x);
                x[4 * i + 1] = fmaf(ar, a4.y, al4.y * b4.y);
                x[4 * i + 2] = fmaf(ar, a4.z, al4.z * b4.z);
                x[4 * i + 3] = fmaf(ar, a4.w, al4.w * b4.w);
            }
            uint4 w;
            w.x = pack2(x[0], x[1]);
            w.y = pack2(x[2], x[3]);
            w.z = pack2(x[4], x[5]);
            w.w = pack2(x[6], x[7]);
            *reinterpret_cast<uint4*>(sm + DG + sm100::sw128_off(r, u + 4 * hlf)) = w;
        }
    }
    if (tid < 64) {   // dbeta; the coefficient of k in dk's gate term
        float dadb, dadl;
        gate_derivatives(rule, bt[tid], lam[tid], al[tid], &dadb, &dadl);
        if (tid < nv && span_ok(err, spans.dbeta, dbeta + row0 + tid, 4)) dbeta[row0 + tid] = dal[tid] * dadb;
        lam[tid] = 2.f * dal[tid] * dadl;
    }
    wait_mma();           // dK^T += S (-dR^T) is done (the commits are waited on in order)
    handoff();
    // ---- 8. dK^T += K^T (dG + dG^T)
    if (warp == 0) {
        mma_ss(tm + C_DK, sb + KQ, 0, 2048, 2 * TILE, sb + DG, 0, 2048, TILE, idesc(128, MN_MAJ, MN_MAJ), 4, true);
        commit();
    }
    wait_mma();
    {   // dk[token][i] = dK^T[i][token] + coef[token] k[token][i]
        float x[32];
        tmem_ld32_wait(tm + lane_off + C_DK + 32 * h, x);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int s = 32 * h + j;
            if (s < nv && span_ok(err, spans.dk, dk + (row0 + s) * 128 + row, 4))
                dk[(row0 + s) * 128 + row] = x[j] + lam[s] * ld_tok(sm + KQ, 2 * TILE, s, row);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (*abort) {         // a wait ran out: record it, and let every issued MMA finish before
        if (tid == 0) atomicOr(err, kDevTimeout);   // the tensor memory is released
        if (warp == 0) {
            commit();
            if (lane == 0) {
                mbar_wait(bar + 1, mma_phase & 1, limit_ns);
                mbar_wait(bar, 0, limit_ns);        // and no copy may land after the block exits
            }
            __syncwarp();
        }
    }
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, C_COLS);
    }
}
// ============================================================================ reverse chain
namespace rc {
constexpr uint32_t TILE = 8192;
constexpr int kStages = 3;
constexpr int kThreads = 320;              // warps 0-7 convert, 8 copies (TMA), 9 issues the MMAs
constexpr uint32_t ST_Q = 0, ST_K = 2 * TILE, ST_T = 4 * TILE, ST_DO = 5 * TILE, STAGE = 6 * TILE;
constexpr uint32_t P = kStages * STAGE;    // P (bf16 [t][s])
constexpr uint32_t DSB = P + TILE;         // dS' (bf16, 128 rows i x 64 columns j)
constexpr uint32_t DD = DSB + 2 * TILE;    // dDelta (bf16 [s][j])
constexpr uint32_t NR = DD + TILE;         // -dR (bf16 [s][j])
constexpr uint32_t BAR = NR + TILE;        // mbarriers, see below
constexpr int NBAR = 16;
constexpr uint32_t MISC = BAR + NBAR * 8;  // TMEM base, abort flag
constexpr uint32_t SMEM_BYTES = MISC + 16 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory");
constexpr uint32_t C_DS = 0, C_P = 64, C_DD = 128, C_DR = 192, C_COLS = 256;
// mbarriers: stage full (TMA) and free (MMA commit) per stage; each product's commit and the
// converters' hand-off back (one arrival per converter warp); the first P~; the drain
enum : int {
    B_FULL = 0, B_FREE = 3, B_DD_FULL = 6, B_DD_READY, B_DR_FULL, B_DR_READY, B_DS_FULL, B_DS_READY, B_PRO,
    B_DRAIN
};
__host__ __device__ constexpr uint32_t bar_count(int i) {
    return (i == B_DD_READY || i == B_DR_READY || i == B_DS_READY) ? 8u : 1u;
}
}  // namespace rc

// One CTA (10 warps) per (stream, 64-column half of d_v) walks the chunks backwards with its
// half of dS in tensor memory.  Warp 8 keeps three chunks' Q, K, T and dO half in flight by
// TMA; warp 9 issues every MMA; warps 0-7 turn each accumulator into the next bf16 operand.
// The roles hand off through mbarriers only (every wait bounded), so an MMA issue that
// stalls on a full queue stalls no converter.  Step k (chunk c = nc - 1 - k):
//   issuer:     [dS'(c), P(c) ready]  store dS'(c) (TMA);  dDelta = P^T dO + K dS'  -> DD_FULL
//               [dDelta ready]        dR = T^T dDelta  -> DR_FULL;  dS += Q^T dO;  P~(c - 1)
//               [-dR ready]           dS += K^T (-dR)  -> DS_FULL, stage c free
//   converters: DD_FULL -> dDelta bf16;  DR_FULL -> -dR bf16;  DS_FULL -> dS'(c - 1) bf16 (or
//               dS0 after chunk 0) and P(c - 1) = tril_incl(P~) bf16  -> DS_READY
__global__ void __launch_bounds__(rc::kThreads, 1)
bwd_chain_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_t,
                 const __grid_constant__ CUtensorMap tm_dsp, const float* __restrict__ dST, float* __restrict__ dS0,
                 int T, uint32_t* __restrict__ err, unsigned long long limit_ns, BwdSpans spans) {
    using namespace rc;
    using namespace sm100;
    using tb::K_MAJ;
    using tb::MN_MAJ;
    using tb::idesc;
    using tb::mma_ss;
    using tb::st_row32;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + MISC);
    volatile int* abort = reinterpret_cast<volatile int*>(sm + MISC + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long bh = blockIdx.x >> 1;
    const int col0 = (blockIdx.x & 1) * 64;
    const int nc = (T + 63) / 64;
    const long tile0 = bh * nc;

    if (nc == 0) {        // no tokens: dS0 = dS_T
        if (dS0 && tid < 256) {
            const int q = (tid >> 5) & 3, h = tid >> 7, row = 32 * q + (tid & 31);
            const size_t srow = ((size_t)bh * 128 + row) * 128 + col0 + 32 * h;
            for (int j = 0; j < 32; ++j)
                if (span_ok(err, spans.ds0, dS0 + srow + j, 4))
                    dS0[srow + j] = dST && span_ok(err, spans.dst, dST + srow + j, 4) ? dST[srow + j] : 0.f;
        }
        return;
    }
    if (tid == 0) {
        for (int i = 0; i < NBAR; ++i) mbar_init(bar + i, bar_count(i));
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, C_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;
    // bounded wait; gives up early once another role has aborted
    auto wait = [&](int i, uint32_t parity) -> bool {
        if (*abort) return false;
        if (mbar_wait(bar + i, parity, limit_ns)) return true;
        *abort = 1;
        return false;
    };
    auto wwait = [&](int i, uint32_t parity) { return __all_sync(0xffffffffu, wait(i, parity)); };
    auto warp_arrive = [&](int i) {
        __syncwarp();
        if (lane == 0) mbar_arrive(bar + i);
    };
    auto stage = [&](int c) { return (uint32_t)(c % kStages); };
    auto use = [&](int c) { return (uint32_t)(((nc - 1 - c) / kStages) & 1); };   // phase of chunk c's stage

    if (warp == 8) {
        // ================================================================ TMA producer
        if (lane == 0) {
            int issued = 0;
            for (int c = nc - 1; c >= 0; --c, ++issued) {
                const uint32_t s = stage(c);
                if (issued >= kStages && !wait(B_FREE + s, use(c + kStages))) break;
                uint8_t* st = sm + s * STAGE;
                uint64_t* full = bar + B_FULL + s;
                mbar_arrive_expect_tx(full, STAGE);
                tma_load_3d(st + ST_Q, &tm_q, full, 0, c * 64, (int)bh);
                tma_load_3d(st + ST_Q + TILE, &tm_q, full, 64, c * 64, (int)bh);
                tma_load_3d(st + ST_K, &tm_k, full, 0, c * 64, (int)bh);
                tma_load_3d(st + ST_K + TILE, &tm_k, full, 64, c * 64, (int)bh);
                tma_load_2d(st + ST_T, &tm_t, full, 0, (int)((tile0 + c) * 64));
                tma_load_3d(st + ST_DO, &tm_do, full, col0, c * 64, (int)bh);
            }
            // no copy may land after the block exits
            for (int c = nc - issued; c < nc - issued + kStages && c < nc; ++c)
                mbar_wait(bar + B_FULL + stage(c), use(c), limit_ns);
        }
    } else if (warp == 9) {
        // ================================================================ MMA issuer (whole warp)
        bool ok = wwait(B_FULL + stage(nc - 1), use(nc - 1));
        if (ok) {
            tc_fence_after();
            const uint32_t st = sb + stage(nc - 1) * STAGE;
            mma_ss(tm + C_P, st + ST_Q, TILE, 32, 16, st + ST_K, TILE, 32, 16, idesc(64, K_MAJ, K_MAJ), 8, false);
            mma_commit_elect(bar + B_PRO);
        }
        for (int k = 0; k < nc && ok; ++k) {
            const int c = nc - 1 - k;
            const uint32_t st = sb + stage(c) * STAGE, ph = k & 1;
            if (!(ok = wwait(B_DS_READY, ph))) break;
            tc_fence_after();
            if (lane == 0) tma_store_2d(&tm_dsp, sm + DSB, col0, (int)((tile0 + c) * 128));   // dS' of chunk c
            __syncwarp();
            mma_ss(tm + C_DD, sb + P, 0, 2048, TILE, st + ST_DO, 0, 2048, TILE, idesc(64, MN_MAJ, MN_MAJ), 4, false);
            mma_ss(tm + C_DD, st + ST_K, TILE, 32, 16, sb + DSB, TILE, 2048, TILE, idesc(64, K_MAJ, MN_MAJ), 8, true);
            mma_commit_elect(bar + B_DD_FULL);
            if (!(ok = wwait(B_DD_READY, ph))) break;
            tc_fence_after();
            mma_ss(tm + C_DR, st + ST_T, 0, 2048, TILE, sb + DD, 0, 2048, TILE, idesc(64, MN_MAJ, MN_MAJ), 4, false);
            mma_commit_elect(bar + B_DR_FULL);
            // what does not need -dR: dS += Q^T dO, and the next chunk's P~
            mma_ss(tm + C_DS, st + ST_Q, 0, 2048, TILE, st + ST_DO, 0, 2048, TILE, idesc(128, MN_MAJ, MN_MAJ), 4, true);
            if (c > 0) {
                if (!(ok = wwait(B_FULL + stage(c - 1), use(c - 1)))) break;
                tc_fence_after();
                const uint32_t sp = sb + stage(c - 1) * STAGE;
                mma_ss(tm + C_P, sp + ST_Q, TILE, 32, 16, sp + ST_K, TILE, 32, 16, idesc(64, K_MAJ, K_MAJ), 8, false);
            }
            if (!(ok = wwait(B_DR_READY, ph))) break;
            if (lane == 0) tma_store_wait_read();   // dS' is rewritten once the dS update has landed
            __syncwarp();
            tc_fence_after();
            mma_ss(tm + C_DS, st + ST_K, 0, 2048, TILE, sb + NR, 0, 2048, TILE, idesc(128, MN_MAJ, MN_MAJ), 4, true);
            mma_commit_elect(bar + B_DS_FULL);
            mma_commit_elect(bar + B_FREE + stage(c));
        }
        mma_commit_elect(bar + B_DRAIN);
        if (lane == 0) {
            mbar_wait(bar + B_DRAIN, 0, limit_ns);
            tma_store_wait_all();
        }
        __syncwarp();
    } else {
        // ================================================================ converters (warps 0-7)
        const int q = warp & 3, h = warp >> 2;            // TMEM lane quarter, column half
        const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
        const int row = 32 * q + lane;                    // row of dS (d_k index)
        const int trow = 16 * q + lane;                   // row of an M = 64 product (lanes < 16)
        const size_t srow = ((size_t)bh * 128 + row) * 128 + col0 + 32 * h;   // this thread's 32 entries of dS
        auto emit_p = [&]() {   // P~ (M = 64) -> P = tril_incl, bf16 [t][s]
            float x[32];
            tmem_ld32_wait(tm + lane_off + C_P + 32 * h, x);
            if (lane < 16) {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (32 * h + j > trow) x[j] = 0.f;
                st_row32(sm + P, trow, 4 * h, x);
            }
        };
        auto hand_off = [&](int i) {
            fence_proxy_async_smem();
            tc_fence_before();
            warp_arrive(i);
        };
        bool ok = true;
        {   // the carried gradient starts as dS_T's half (or zero); P of the last chunk
            float x[32];
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                const float4 v = dST && span_ok(err, spans.dst, dST + srow + j, 16)
                                     ? *reinterpret_cast<const float4*>(dST + srow + j) : make_float4(0.f, 0.f, 0.f, 0.f);
                x[j] = v.x; x[j + 1] = v.y; x[j + 2] = v.z; x[j + 3] = v.w;
            }
            float lo[16], hi[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                lo[j] = x[j];
                hi[j] = x[16 + j];
            }
            tmem_st16(tm + lane_off + C_DS + 32 * h, lo);
            tmem_st16(tm + lane_off + C_DS + 32 * h + 16, hi);
            tmem_wait_st();
            st_row32(sm + DSB, row, 4 * h, x);
            ok = wwait(B_PRO, 0);
            tc_fence_after();
            emit_p();
            hand_off(B_DS_READY);
        }
        for (int k = 0; k < nc && ok; ++k) {
            const int c = nc - 1 - k;
            const uint32_t ph = k & 1;
            float x[32];
            if (!(ok = wwait(B_DD_FULL, ph))) break;
            tc_fence_after();
            tmem_ld32_wait(tm + lane_off + C_DD + 32 * h, x);
            if (lane < 16) st_row32(sm + DD, trow, 4 * h, x);
            hand_off(B_DD_READY);
            if (!(ok = wwait(B_DR_FULL, ph))) break;
            tc_fence_after();
            tmem_ld32_wait(tm + lane_off + C_DR + 32 * h, x);
#pragma unroll
            for (int j = 0; j < 32; ++j) x[j] = -x[j];
            if (lane < 16) st_row32(sm + NR, trow, 4 * h, x);
            hand_off(B_DR_READY);
            if (!(ok = wwait(B_DS_FULL, ph))) break;
            tc_fence_after();
            tmem_ld32_wait(tm + lane_off + C_DS + 32 * h, x);
            if (c > 0) {
                st_row32(sm + DSB, row, 4 * h, x);
                emit_p();
                hand_off(B_DS_READY);
            } else if (dS0) {
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    if (span_ok(err, spans.ds0, dS0 + srow + j, 16))
                        *reinterpret_cast<float4*>(dS0 + srow + j) = make_float4(x[j], x[j + 1], x[j + 2], x[j + 3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort) atomicOr(err, kDevTimeout);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, C_COLS);
    }
}

}  // namespace

constexpr unsigned long long kTileWaitNs = 2000000000ull;   // 2 s per wait

size_t bwd_chunk_workspace_bytes(long BH, int T) {
    const long ntiles = BH * ((T + kC - 1) / kC);
    return (size_t)ntiles * ((kC * kC + 2 * kD * kD) * sizeof(bf16) + kUtXBytes);   // T, X, S and dS' per tile
}

size_t bwd_saved_t_bytes(long BH, int T) { return (size_t)BH * ((T + kC - 1) / kC) * kC * kC * sizeof(bf16); }
size_t bwd_saved_x_bytes(long BH, int T) { return (size_t)BH * ((T + kC - 1) / kC) * kUtXBytes; }
size_t bwd_saved_state_bytes(long BH, int T) { return (size_t)BH * ((T + kC - 1) / kC) * kD * kD * sizeof(bf16); }

cudaError_t launch_bwd_chunk(const void* q, const void* k, const void* v, const void* beta, const float* S0,
                             const void* dO, const float* dST, float* dq, float* dk, float* dv, float* dbeta,
                             float* dS0, long BH, int T, int rule, uint32_t* err, void* scratch, cudaStream_t stream) {
    const int nchunks = (T + kC - 1) / kC;
    const long ntiles = BH * nchunks;
    bf16* Tt = static_cast<bf16*>(scratch);
    float* X = reinterpret_cast<float*>(Tt + (size_t)ntiles * kC * kC);
    bf16* states = reinterpret_cast<bf16*>(reinterpret_cast<char*>(X) + (size_t)ntiles * kUtXBytes);
    bf16* dSp = states + (size_t)ntiles * kD * kD;
    // 1. UT transforms (keeping X) and the forward chain, storing every chunk's entering state
    SegPlan plan;
    plan.states = states;
    plan.X = X;
    Seqs seqs{nullptr, nullptr, 0, 0, T, 0};
    cudaError_t e = launch_chunk_tc(q, k, v, beta, S0, nullptr, nullptr, seqs, BH, BH, T, ntiles, err, Tt, rule,
                                    stream, nullptr, plan);
    if (e != cudaSuccess) return e;
    // 2, 3. the reverse chain and every chunk's gradients
    return launch_bwd_chunk_saved(q, k, v, beta, dO, dST, dq, dk, dv, dbeta, dS0, BH, T, rule, err, Tt, X, states,
                                  dSp, stream);
}

cudaError_t launch_bwd_chunk_saved(const void* q, const void* k, const void* v, const void* beta, const void* dO,
                                   const float* dST, float* dq, float* dk, float* dv, float* dbeta, float* dS0,
                                   long BH, int T, int rule, uint32_t* err, const void* Tt, const float* X,
                                   const void* states, void* dSp, cudaStream_t stream) {
    const int nchunks = (T + kC - 1) / kC;
    const long ntiles = BH * nchunks;
    cudaError_t e;
    // 2. the reverse chain
    CUtensorMap mq, mk, mv, mdo, mt, ms, mdsp;
    if (!tma_map_tokens(&mq, q, kD, T, BH) || !tma_map_tokens(&mk, k, kD, T, BH) || !tma_map_tokens(&mv, v, kD, T, BH) ||
        !tma_map_tokens(&mdo, dO, kD, T, BH) || !tma_map_rows64(&mt, Tt, std::max<long>(1, ntiles) * kC) ||
        !tma_map_rows128(&ms, states, std::max<long>(1, ntiles) * kD) ||
        !tma_map_rows128(&mdsp, dSp, std::max<long>(1, ntiles) * kD))
        return cudaErrorInvalidValue;
    BwdSpans sp;
    const size_t tok = (size_t)BH * T, sbytes = (size_t)BH * kD * kD * 4;
    sp.beta = Span{beta, tok * 2};
    sp.dq = Span{dq, tok * kD * 4};
    sp.dk = Span{dk, tok * kD * 4};
    sp.dv = Span{dv, tok * kD * 4};
    sp.dbeta = Span{dbeta, tok * 4};
    sp.dst = Span{dST, sbytes};
    sp.ds0 = Span{dS0, sbytes};
    sp.x = Span{X, (size_t)ntiles * kUtXBytes};
    static std::atomic<uint64_t> smem_chain{0}, smem_tile{0};
    e = set_smem_limit_once(bwd_chain_kernel, (int)rc::SMEM_BYTES, smem_chain);
    if (e != cudaSuccess) return e;
    bwd_chain_kernel<<<(unsigned)(BH * 2), rc::kThreads, rc::SMEM_BYTES, stream>>>(mq, mk, mdo, mt, mdsp, dST, dS0, T, err,
                                                                          kTileWaitNs, sp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // 3. every chunk's gradients
    if (ntiles == 0) return cudaSuccess;
    e = set_smem_limit_once(bwd_tile_kernel, (int)tb::SMEM_BYTES, smem_tile);
    if (e != cudaSuccess) return e;
    bwd_tile_kernel<<<(unsigned)ntiles, 256, tb::SMEM_BYTES, stream>>>(
        mq, mk, mv, mdo, ms, mdsp, mt, X, (const bf16*)beta, dq, dk, dv, dbeta, T, rule, err, kTileWaitNs, sp);
    return cudaGetLastError();
}

}  // namespace efla