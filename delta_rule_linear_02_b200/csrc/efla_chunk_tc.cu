// efla_chunk_tc.cu -- chunkwise EFLA forward on the 5th-generation tensor cores (sm_100a).
//
// bf16 q, k, v, beta -> bf16 o, fp32 state.  One CTA owns one (b, h) stream and one
// 64-column slice of d_v (d_k = d_v = 128).  The fp32 state slice S (128 x 64) lives in
// tensor memory for the whole sequence as the accumulator of S += K^T Delta.
//
// Per 64-token chunk (Exact Flow Linear Attention, Section 3.3; row convention):
//   [G; P~] = [K; Q] K^T                    M=128 MMA   (G = K K^T, P~ = Q K^T)
//   alpha_r = gate(beta_r, G_rr)            Section 3.2 / 3.4 (lambda_r = ||k_r||^2 = G_rr)
//   T = (I + strictly-lower(diag(alpha) G))^{-1} diag(alpha)      fp32 on CUDA cores
//   [. ; W | U] = [P; T] [K | V]            M=128, N=192 MMA  (P = P~, causal incl. diagonal)
//   [QS; WS] = [Q; W] S                     M=128 MMA
//   Delta = U - WS                          fp32, then a bf16 operand
//   S += K^T Delta;  [O; .] = [QS; .] + [P; T] Delta               two M=128 MMAs
// Tokens past T are zero-filled by TMA (k = 0, beta = 0: alpha = 0, an exact no-op).
//
// Warp roles (16 warps).  Only S -> [Q;W]S -> Delta -> K^T Delta -> S is sequential;
// everything that does not depend on S runs one chunk ahead on other warps:
//   warp 0       TMA producer: K, Q, V tiles of chunk c into a 2-deep stage ring
//   warp 1       MMA issuer: one thread, issues whichever of the five MMAs is ready
//   warps 2-3    W/U converter: TMEM rows 64..127 of [W | U] -> bf16 W operand, fp32 U
//   warps 4-7    chain: Delta, the state's bf16 copy, O and the final state
//   warps 8-15   prep: alpha, the masked P operand and the UT solve for T
// Operands are staged by TMA (128-byte swizzle, no multicast) or written in the same
// swizzled layouts.  Every wait is bounded (2 s); a wait that runs out sets a CTA-wide
// abort flag, every role winds down, and the caller's workspace records the timeout.
// `dbg` (null in the library) receives CTA 0's chunk-0 intermediates for diagnosis:
// A [0,4096) alpha [4096,4160) T [4160,8256) W [8256,16448) U [16448,20544)
// WS [20544,24640) S after the chunk [24640,32832); and per chunk c < 64 the cycle at
// which each role passed its milestones, at [40000 + 16 c + k): k = 0..3 MMA issue of
// [G;P~], [W|U], [QS;WS], S-update; 4 GP read; 5 T ready; 6 W ready; 7 U ready;
// 8 Delta ready; 9 new S ready; 10 O stored; 11 TMA issued; 12 A written; 13 solve done.
#include <cudaTypedefs.h>

#include "efla_common.cuh"
#include "efla_kernels.h"
#include "sm100.cuh"

namespace efla {

namespace {
using namespace sm100;

constexpr int kThreads = 512;
constexpr int kD = 128;          // d_k = d_v
constexpr int LDX = 68;          // fp32 scratch row stride (16-byte aligned rows)

// ---- shared-memory map (bytes from a 1024-aligned base)
// stage s (x2): [K a0 | Q a0 | W a0 | K a1 | Q a1 | W a1 | V]: 7 tiles of 64 x 64 bf16
constexpr uint32_t TILE = 8192;
constexpr uint32_t ATOM_STRIDE = 3 * TILE;          // a0 -> a1 (one 64-column half of d_k)
constexpr uint32_t ST_K = 0, ST_Q = TILE, ST_W = 2 * TILE, ST_V = 6 * TILE;
constexpr uint32_t STAGE_BYTES = 7 * TILE;
constexpr uint32_t OFF_STAGE = 0;
constexpr uint32_t OFF_PT = OFF_STAGE + 2 * STAGE_BYTES;   // 2 x [P | T]
constexpr uint32_t OFF_DL = OFF_PT + 2 * 2 * TILE;         // Delta, MN-major 64 x 64
constexpr uint32_t OFF_SB = OFF_DL + TILE;                 // S bf16, MN-major 128 x 64
constexpr uint32_t OFF_AT = OFF_SB + 2 * TILE;             // A^T (upper) + merge scratch (lower)
constexpr uint32_t F32_TILE = 64 * LDX * 4;
constexpr uint32_t OFF_X = OFF_AT + F32_TILE;              // (I + A)^{-1}
constexpr uint32_t OFF_U = OFF_X + F32_TILE;               // U rows, fp32
constexpr uint32_t OFF_ALPHA = OFF_U + F32_TILE;
constexpr uint32_t OFF_BETA = OFF_ALPHA + 256;
constexpr uint32_t OFF_BAR = OFF_BETA + 256;
constexpr uint32_t NBAR = 24;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
constexpr uint32_t SMEM_USED = OFF_MISC + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;          // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared-memory map exceeds 227 KB");

// ---- mbarriers (all count 1)
enum : int {
    B_FULL = 0,        // [2] TMA landed stage s
    B_STAGE_FREE = 2,  // [2] last MMA reading stage s (and P/T buffer s) done
    B_GP_FULL = 4, B_GP_FREE, B_T_READY, B_WU_FULL, B_WU_FREE, B_W_READY, B_U_READY, B_U_FREE,
    B_Y_FULL = 12,     // [2]
    B_D_READY = 14, B_S_FULL,
    B_O_FULL = 16,     // [2]
    B_SB_READY = 18,
    B_Y_FREE = 19,     // [2]
    B_DRAIN = 21,      // [2] one per issuing thread
};

// ---- TMEM columns (fp32 accumulators, lanes 0..127)
constexpr uint32_t TM_S = 0, TM_Y = 64 /* x2 */, TM_GP = 192, TM_WU = 256, TM_COLS = 512;

constexpr uint32_t ID_GP = idesc_bf16(128, 64, false, false);
constexpr uint32_t ID_WU = idesc_bf16(128, 192, false, true);
constexpr uint32_t ID_Y = idesc_bf16(128, 64, false, true);
constexpr uint32_t ID_S = idesc_bf16(128, 64, true, true);

// ---- named barriers
constexpr int NB_CHAIN = 1, NB_DELTA = 2, NB_OUT = 3, NB_PREP = 4, NB_CONV = 5;

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

// 8 floats -> one 16-byte chunk of bf16 at a shared address
__device__ __forceinline__ void st_chunk(uint8_t* p, const float* v) {
    uint4 u;
    u.x = pack_bf16x2(v[0], v[1]);
    u.y = pack_bf16x2(v[2], v[3]);
    u.z = pack_bf16x2(v[4], v[5]);
    u.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4*>(p) = u;
}

struct Ctl {
    uint64_t* bar;
    volatile int* abort;
    unsigned long long limit;
    __device__ uint64_t* b(int i) const { return bar + i; }
    // bounded wait; gives up early once another role has aborted
    __device__ bool wait(int i, uint32_t parity) const {
        if (mbar_try_wait_sleep(bar + i, parity, 20000)) return true;
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait_sleep(bar + i, parity, 20000)) {
            if (*abort) return false;
            if (globaltimer_ns() - t0 > limit) {
                *abort = 1;
                return false;
            }
        }
        return true;
    }
};

// --------------------------------------------------------------------------- UT solve
// X = (I + A)^{-1} for the 64 x 64 strictly-lower A, by 256 threads (ptid), with
//   At[j * LDX + i] = A[i][j] (i > j)  -- only that part of At is read;
//   the merge products are kept in At's other triangle (At[r * LDX + c], r > c).
// X's strictly-upper 16 x 16 blocks are zero from the start of the kernel.
//   (1) 16 x 16 diagonal blocks by forward substitution, one thread per column (fp32);
//   (2) 32 x 32 merges X21 = -X22 (A21 X11);  (3) the 64 x 64 merge the same way.
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

// One warp: C(16 x 16) = sum over k-steps [k0, k1) of A(16 x 8) B(8 x 16).
//   A(r, k) = a_base[k * a_ks + r * a_rs]      B(k, n) = b_base[k * LDX + n]
// Output fragment: rows g, g + 8 (g = lane / 4), columns 8 nt + 2 t, + 1 (t = lane % 4).
__device__ __forceinline__ void warp_mm16x16(float (&c)[2][4], const float* __restrict__ a_base, int a_ks,
                                             int a_rs, const float* __restrict__ b_base, int k0, int k1,
                                             int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) c[nt][e] = 0.f;
    for (int ks = k0; ks < k1; ++ks) {
        const int k = 8 * ks + t;
        uint32_t a[4];
        a[0] = to_tf32(a_base[k * a_ks + g * a_rs]);
        a[1] = to_tf32(a_base[k * a_ks + (g + 8) * a_rs]);
        a[2] = to_tf32(a_base[(k + 4) * a_ks + g * a_rs]);
        a[3] = to_tf32(a_base[(k + 4) * a_ks + (g + 8) * a_rs]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            uint32_t b[2];
            b[0] = to_tf32(b_base[k * LDX + 8 * nt + g]);
            b[1] = to_tf32(b_base[(k + 4) * LDX + 8 * nt + g]);
            mma_tf32(c[nt], a, b);
        }
    }
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

__device__ __forceinline__ void ut_solve(float* __restrict__ At, float* __restrict__ X, int ptid) {
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
    bar_sync(NB_PREP, 256);
    float acc[2][4];
    if (pw < 2) {      // (2a) Y = A21 X11 for super-block pw (16 x 16 x 16; X11 lower: k >= n)
        const int r0 = 32 * pw + 16, c0 = 32 * pw;
        warp_mm16x16(acc, At + c0 * LDX + r0, LDX, 1, X + c0 * LDX + c0, 0, 2, lane);
        warp_st16x16(At + r0 * LDX + c0, acc, 1.f, lane);
    }
    bar_sync(NB_PREP, 256);
    if (pw < 2) {      // (2b) X21 = -X22 Y
        const int r0 = 32 * pw + 16, c0 = 32 * pw;
        warp_mm16x16(acc, X + r0 * LDX + r0, 1, LDX, At + r0 * LDX + c0, 0, 2, lane);
        warp_st16x16(X + r0 * LDX + c0, acc, -1.f, lane);
    }
    bar_sync(NB_PREP, 256);
    if (pw < 4) {      // (3a) Y = A21 X11 (32 x 32 x 32); tile (wr, wc), X11[k][n] = 0 for k < 16 wc
        const int wr = pw >> 1, wc = pw & 1;
        warp_mm16x16(acc, At + 32 + 16 * wr, LDX, 1, X + 16 * wc, 2 * wc, 4, lane);
        warp_st16x16(At + (32 + 16 * wr) * LDX + 16 * wc, acc, 1.f, lane);
    }
    bar_sync(NB_PREP, 256);
    if (pw < 4) {      // (3b) X21 = -X22 Y; X22[m][k] = 0 for k > 16 wr + 15
        const int wr = pw >> 1, wc = pw & 1;
        warp_mm16x16(acc, X + (32 + 16 * wr) * LDX + 32, 1, LDX, At + 32 * LDX + 16 * wc, 0, 2 * wr + 2, lane);
        warp_st16x16(X + (32 + 16 * wr) * LDX + 16 * wc, acc, -1.f, lane);
    }
    bar_sync(NB_PREP, 256);
}

__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __nv_bfloat16* __restrict__ beta,
                const float* __restrict__ S0, __nv_bfloat16* __restrict__ o, float* __restrict__ S_T,
                int T, uint32_t* __restrict__ err, unsigned long long limit_ns, float* __restrict__ dbg) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    float* At = reinterpret_cast<float*>(sm + OFF_AT);
    float* X = reinterpret_cast<float*>(sm + OFF_X);
    float* Us = reinterpret_cast<float*>(sm + OFF_U);
    float* al = reinterpret_cast<float*>(sm + OFF_ALPHA);
    float* bt = reinterpret_cast<float*>(sm + OFF_BETA);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
    Ctl ctl{reinterpret_cast<uint64_t*>(sm + OFF_BAR), reinterpret_cast<volatile int*>(sm + OFF_MISC + 4), limit_ns};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x >> 1;
    const int col0 = (blockIdx.x & 1) * 64;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;   // this warp's TMEM lanes
    const int nchunks = (T + 63) / 64;
    const size_t tok0 = (size_t)bh * T;
    const long long t_start = clock64();
#define EFLA_STAMP(c, k)                                                                  \
    do {                                                                                  \
        if (dbg && blockIdx.x == 0 && (c) < 64) dbg[40000 + 16 * (c) + (k)] = (float)(clock64() - t_start); \
    } while (0)

    if (tid == 0) {
        for (int i = 0; i < (int)NBAR; ++i) mbar_init(ctl.bar + i, 1);
        *ctl.abort = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, TM_COLS);
        tmem_relinquish();
    }
    // X's strictly-upper 16 x 16 blocks stay zero for the whole kernel
    for (int e = tid; e < 6 * 256; e += kThreads) {
        const int blk = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
        const int R = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
        const int C = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
        X[(16 * R + rr) * LDX + 16 * C + cc] = 0.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ================================================================ TMA producer + [G; P~] issuer
        if (lane == 0) {
            bool ok = true;
            for (int c = 0; c < nchunks && ok; ++c) {
                const int s = c & 1;
                if (c >= 2 && !(ok = ctl.wait(B_STAGE_FREE + s, ((c - 2) >> 1) & 1))) break;
                uint8_t* st = sm + OFF_STAGE + s * STAGE_BYTES;
                uint64_t* full = ctl.b(B_FULL + s);
                mbar_arrive_expect_tx(full, 5 * TILE);
                const int t0 = c * 64;
                tma_load_3d(st + ST_K, &tm_k, full, 0, t0, bh);
                tma_load_3d(st + ST_Q, &tm_q, full, 0, t0, bh);
                tma_load_3d(st + ATOM_STRIDE + ST_K, &tm_k, full, 64, t0, bh);
                tma_load_3d(st + ATOM_STRIDE + ST_Q, &tm_q, full, 64, t0, bh);
                tma_load_3d(st + ST_V, &tm_v, full, col0, t0, bh);
                EFLA_STAMP(c, 11);
                if (c + 2 < nchunks) {        // its stage frees only after chunk c: warm L2 now
                    const int t2 = t0 + 128;
                    tma_prefetch_l2_3d(&tm_k, 0, t2, bh);
                    tma_prefetch_l2_3d(&tm_q, 0, t2, bh);
                    tma_prefetch_l2_3d(&tm_k, 64, t2, bh);
                    tma_prefetch_l2_3d(&tm_q, 64, t2, bh);
                    tma_prefetch_l2_3d(&tm_v, col0, t2, bh);
                }
                // [G; P~] = [K; Q] K^T once the tiles landed and the prep warps released GP
                if (!(ok = ctl.wait(B_FULL + s, (c >> 1) & 1))) break;
                if (c > 0 && !(ok = ctl.wait(B_GP_FREE, (c - 1) & 1))) break;
                tc_fence_after();
                const uint32_t sa = sb + OFF_STAGE + s * STAGE_BYTES;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t aa = sa + (ks >> 2) * ATOM_STRIDE + ST_K + (ks & 3) * 32;
                    mma_bf16(tmem + TM_GP, sdesc_sw128(aa, 16, 1024), sdesc_sw128(aa, 16, 1024), ID_GP, ks > 0);
                }
                mma_commit(ctl.b(B_GP_FULL));
                EFLA_STAMP(c, 0);
            }
            // every copy and MMA this thread issued has landed before the CTA can exit
            mma_commit(ctl.b(B_DRAIN));
            mbar_wait(ctl.b(B_DRAIN), 0, limit_ns);
            for (int c = max(0, nchunks - 2); c < nchunks; ++c)
                mbar_wait(ctl.b(B_FULL + (c & 1)), (c >> 1) & 1, limit_ns);
        }
    } else if (warp == 1) {
        // ================================================================ chain + [W | U] issuer
        if (lane == 0) {
            auto issue_wu = [&](int c) {      // [. ; W | U] = [P; T] [K | V]
                tc_fence_after();
                const int s = c & 1;
                const uint32_t st = sb + OFF_STAGE + s * STAGE_BYTES;
                const uint32_t pt = sb + OFF_PT + s * 2 * TILE;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + TM_WU, sdesc_sw128(pt + ks * 32, 16, 1024),
                             sdesc_sw128(st + ST_K + ks * 2048, ATOM_STRIDE, 1024), ID_WU, ks > 0);
                mma_commit(ctl.b(B_WU_FULL));
                EFLA_STAMP(c, 1);
            };
            bool ok = ctl.wait(B_T_READY, 0);
            if (ok) issue_wu(0);
            int ic = 1;
            for (int c = 0; c < nchunks && ok; ++c) {
                const int s = c & 1;
                const uint32_t st = sb + OFF_STAGE + s * STAGE_BYTES;
                // [QS; WS] = [Q; W] S
                ok = ctl.wait(B_W_READY, c & 1) && ctl.wait(B_SB_READY, c & 1) &&
                     (c < 2 || ctl.wait(B_Y_FREE + s, ((c - 2) >> 1) & 1));
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t aa = st + (ks >> 2) * ATOM_STRIDE + ST_Q + (ks & 3) * 32;
                    mma_bf16(tmem + TM_Y + 64 * s, sdesc_sw128(aa, 16, 1024),
                             sdesc_sw128(sb + OFF_SB + ks * 2048, TILE, 1024), ID_Y, ks > 0);
                }
                mma_commit(ctl.b(B_Y_FULL + s));
                EFLA_STAMP(c, 2);
                // the next chunk's [W | U] goes right behind it when its T is already there
                if (ic < nchunks && mbar_test_wait(ctl.b(B_T_READY), ic & 1) &&
                    mbar_test_wait(ctl.b(B_WU_FREE), (ic - 1) & 1)) {
                    issue_wu(ic);
                    ++ic;
                }
                // S += K^T Delta, then [O; .] += [P; T] Delta
                if (!(ok = ctl.wait(B_D_READY, c & 1))) break;
                tc_fence_after();
                const uint32_t pt = sb + OFF_PT + s * 2 * TILE;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + TM_S, sdesc_sw128(st + ST_K + ks * 2048, ATOM_STRIDE, 1024),
                             sdesc_sw128(sb + OFF_DL + ks * 2048, TILE, 1024), ID_S, 1);
                mma_commit(ctl.b(B_S_FULL));
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + TM_Y + 64 * s, sdesc_sw128(pt + ks * 32, 16, 1024),
                             sdesc_sw128(sb + OFF_DL + ks * 2048, TILE, 1024), ID_Y, 1);
                mma_commit(ctl.b(B_O_FULL + s));
                mma_commit(ctl.b(B_STAGE_FREE + s));
                EFLA_STAMP(c, 3);
                if (ic == c + 1 && ic < nchunks) {
                    if (!(ok = ctl.wait(B_T_READY, ic & 1) && ctl.wait(B_WU_FREE, (ic - 1) & 1))) break;
                    issue_wu(ic);
                    ++ic;
                }
            }
            mma_commit(ctl.b(B_DRAIN + 1));
            mbar_wait(ctl.b(B_DRAIN + 1), 0, limit_ns);
        }
    } else if (warp < 4) {
        // ================================================================ W/U converter (TMEM lanes 64..127)
        const int r = tid - 64;                       // chunk row
        bool ok = true;
        for (int c = 0; c < nchunks && ok; ++c) {
            const int s = c & 1;
            ok = bar_and(NB_CONV, 64, ctl.wait(B_WU_FULL, c & 1));
            if (!ok) break;
            tc_fence_after();
            uint8_t* st = sm + OFF_STAGE + s * STAGE_BYTES;
#pragma unroll
            for (int q = 0; q < 8; ++q) {             // W row r -> bf16, K-major, two 64-column atoms
                float w16[16];
                tmem_ld16(tmem + lane_off + TM_WU + 16 * q, w16);
                tmem_wait_ld();
                uint8_t* dst = st + (q >> 2) * ATOM_STRIDE + ST_W;
                st_chunk(dst + sw128_off(r, (q & 3) * 2), w16);
                st_chunk(dst + sw128_off(r, (q & 3) * 2 + 1), w16 + 8);
                if (dbg && blockIdx.x == 0 && c == 0)
                    for (int j = 0; j < 16; ++j) dbg[8256 + r * 128 + 16 * q + j] = w16[j];
            }
            fence_proxy_async_smem();
            bar_sync(NB_CONV, 64);
            if (r == 0) {
                mbar_arrive(ctl.b(B_W_READY));
                EFLA_STAMP(c, 6);
            }
            ok = bar_and(NB_CONV, 64, c == 0 || ctl.wait(B_U_FREE, (c - 1) & 1));
            if (!ok) break;
#pragma unroll
            for (int q = 0; q < 4; ++q) {             // U row r stays fp32
                float u16[16];
                tmem_ld16(tmem + lane_off + TM_WU + 128 + 16 * q, u16);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; j += 4)
                    *reinterpret_cast<float4*>(Us + r * LDX + 16 * q + j) = make_float4(u16[j], u16[j + 1], u16[j + 2], u16[j + 3]);
                if (dbg && blockIdx.x == 0 && c == 0)
                    for (int j = 0; j < 16; ++j) dbg[16448 + r * 64 + 16 * q + j] = u16[j];
            }
            tc_fence_before();
            bar_sync(NB_CONV, 64);
            if (r == 0) {
                mbar_arrive(ctl.b(B_U_READY));
                mbar_arrive(ctl.b(B_WU_FREE));
                EFLA_STAMP(c, 7);
            }
        }
    } else if (warp < 8) {
        // ================================================================ chain (TMEM lanes 0..127)
        const int ct = tid - 128;                     // d_k row for S; rows of Y by quarter
        {   // initial state
            const float* src = S0 ? S0 + ((size_t)bh * kD + ct) * kD + col0 : nullptr;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float s16[16];
#pragma unroll
                for (int j = 0; j < 16; j += 4) {
                    float4 x = src ? *reinterpret_cast<const float4*>(src + 16 * q + j) : make_float4(0.f, 0.f, 0.f, 0.f);
                    s16[j] = x.x; s16[j + 1] = x.y; s16[j + 2] = x.z; s16[j + 3] = x.w;
                }
                tmem_st16(tmem + lane_off + TM_S + 16 * q, s16);
                st_chunk(sm + OFF_SB + sw128_off(ct, 2 * q), s16);
                st_chunk(sm + OFF_SB + sw128_off(ct, 2 * q + 1), s16 + 8);
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            bar_sync(NB_CHAIN, 128);
            if (ct == 0) mbar_arrive(ctl.b(B_SB_READY));
        }
        bool ok = true;
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            const uint32_t tY = tmem + lane_off + TM_Y + 64 * b;
            if (warp >= 6) {                          // Delta = U - WS (rows 64..127 of Y)
                const int r = ct - 64;
                bool w = ok && ctl.wait(B_Y_FULL + b, (c >> 1) & 1) && ctl.wait(B_U_READY, c & 1);
                w = bar_and(NB_DELTA, 64, w);
                if (w) {
                    tc_fence_after();
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float t16[16];
                        tmem_ld16(tY + 16 * q, t16);
                        tmem_wait_ld();
                        if (dbg && blockIdx.x == 0 && c == 0)
                            for (int j = 0; j < 16; ++j) dbg[20544 + r * 64 + 16 * q + j] = t16[j];
#pragma unroll
                        for (int j = 0; j < 16; j += 4) {
                            const float4 u = *reinterpret_cast<const float4*>(Us + r * LDX + 16 * q + j);
                            t16[j] = u.x - t16[j];
                            t16[j + 1] = u.y - t16[j + 1];
                            t16[j + 2] = u.z - t16[j + 2];
                            t16[j + 3] = u.w - t16[j + 3];
                        }
                        st_chunk(sm + OFF_DL + sw128_off(r, 2 * q), t16);
                        st_chunk(sm + OFF_DL + sw128_off(r, 2 * q + 1), t16 + 8);
                    }
                    fence_proxy_async_smem();
                    tc_fence_before();
                    bar_sync(NB_DELTA, 64);
                    if (r == 0) {
                        mbar_arrive(ctl.b(B_D_READY));
                        mbar_arrive(ctl.b(B_U_FREE));
                        EFLA_STAMP(c, 8);
                    }
                }
                ok = w;
            }
            // the new state: bf16 operand for the next chunk (and S_T after the last)
            ok = bar_and(NB_CHAIN, 128, ok && ctl.wait(B_S_FULL, c & 1));
            if (!ok) break;
            tc_fence_after();
            const bool last = (c == nchunks - 1);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float t16[16];
                tmem_ld16(tmem + lane_off + TM_S + 16 * q, t16);
                tmem_wait_ld();
                st_chunk(sm + OFF_SB + sw128_off(ct, 2 * q), t16);
                st_chunk(sm + OFF_SB + sw128_off(ct, 2 * q + 1), t16 + 8);
                if (dbg && blockIdx.x == 0 && c == 0)
                    for (int j = 0; j < 16; ++j) dbg[24640 + ct * 64 + 16 * q + j] = t16[j];
                if (last && S_T) {
                    float* dst = S_T + ((size_t)bh * kD + ct) * kD + col0 + 16 * q;
#pragma unroll
                    for (int j = 0; j < 16; j += 4)
                        *reinterpret_cast<float4*>(dst + j) = make_float4(t16[j], t16[j + 1], t16[j + 2], t16[j + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            bar_sync(NB_CHAIN, 128);
            if (ct == 0) {
                mbar_arrive(ctl.b(B_SB_READY));
                EFLA_STAMP(c, 9);
            }
            if (warp < 6) {                           // O rows (lanes 0..63 of Y)
                const int r = ct;
                bool w = bar_and(NB_OUT, 64, ctl.wait(B_O_FULL + b, (c >> 1) & 1));
                if (w) {
                    tc_fence_after();
                    const int t0 = c * 64;
                    const bool live = r < min(64, T - t0);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float t16[16];
                        tmem_ld16(tY + 16 * q, t16);
                        tmem_wait_ld();
                        if (live) {
                            uint4* dst = reinterpret_cast<uint4*>(o + (tok0 + t0 + r) * kD + col0 + 16 * q);
                            uint4 a, bb;
                            a.x = pack_bf16x2(t16[0], t16[1]); a.y = pack_bf16x2(t16[2], t16[3]);
                            a.z = pack_bf16x2(t16[4], t16[5]); a.w = pack_bf16x2(t16[6], t16[7]);
                            bb.x = pack_bf16x2(t16[8], t16[9]); bb.y = pack_bf16x2(t16[10], t16[11]);
                            bb.z = pack_bf16x2(t16[12], t16[13]); bb.w = pack_bf16x2(t16[14], t16[15]);
                            dst[0] = a;
                            dst[1] = bb;
                        }
                    }
                    tc_fence_before();
                    bar_sync(NB_OUT, 64);
                    if (r == 0) {
                        mbar_arrive(ctl.b(B_Y_FREE + b));
                        EFLA_STAMP(c, 10);
                    }
                }
                ok = w;
            }
        }
    } else {
        // ================================================================ prep (256 threads)
        const int ptid = tid - 256, pw = ptid >> 5;
        const int q = warp & 3;                       // TMEM lane quarter
        const int h = pw >> 2;                        // column half of the GP tile
        bool ok = true;
        float beta_next = (ptid < 64 && ptid < T) ? __bfloat162float(beta[tok0 + ptid]) : 0.f;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            if (ptid < 64) {                          // beta of this chunk; fetch the next one's
                bt[ptid] = beta_next;
                const int tn = (c + 1) * 64 + ptid;
                beta_next = (tn < T) ? __bfloat162float(beta[tok0 + tn]) : 0.f;
            }
            ok = bar_and(NB_PREP, 256, ok && ctl.wait(B_GP_FULL, c & 1));
            if (!ok) break;
            tc_fence_after();
            float g[32];
            {
                float t16[16];
                tmem_ld16(tmem + lane_off + TM_GP + 32 * h, t16);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) g[j] = t16[j];
                tmem_ld16(tmem + lane_off + TM_GP + 32 * h + 16, t16);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) g[16 + j] = t16[j];
            }
            const int r = 32 * (q & 1) + lane;        // row of G (q < 2) or of P~ (q >= 2)
            if (q < 2) {
                if ((q & 1) == h) {                   // this thread holds G[r][r]: lambda_r -> alpha_r
                    float lam = 0.f;
#pragma unroll
                    for (int j = 0; j < 32; ++j) lam = (j == lane) ? g[j] : lam;
                    al[r] = gate_alpha(bt[r], lam);
                }
            } else {                                  // P = P~ with the causal mask (diagonal kept)
                uint8_t* P = sm + OFF_PT + s * 2 * TILE;
#pragma unroll
                for (int j = 0; j < 32; ++j) g[j] = (32 * h + j <= r) ? g[j] : 0.f;
#pragma unroll
                for (int m = 0; m < 4; ++m) st_chunk(P + sw128_off(r, 4 * h + m), g + 8 * m);
            }
            tc_fence_before();
            bar_sync(NB_PREP, 256);                   // alpha visible, GP read
            if (ptid == 0) {
                mbar_arrive(ctl.b(B_GP_FREE));
                EFLA_STAMP(c, 4);
            }
            if (q < 2) {
                // A^T[r][i] = A[i][r] = alpha_i G[i][r] = alpha_i G[r][i] (G = K K^T is symmetric):
                // row r of A^T is this thread's G row scaled by alpha, written 4 floats at a time.
                // Entries with i <= r fall in the half the solve uses as scratch; they are not read.
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const float4 a = *reinterpret_cast<const float4*>(al + 32 * h + 4 * m);
                    *reinterpret_cast<float4*>(At + r * LDX + 32 * h + 4 * m) =
                        make_float4(a.x * g[4 * m], a.y * g[4 * m + 1], a.z * g[4 * m + 2], a.w * g[4 * m + 3]);
                }
            }
            bar_sync(NB_PREP, 256);
            if (ptid == 0) EFLA_STAMP(c, 12);
            if (dbg && blockIdx.x == 0 && c == 0) {
                for (int e = ptid; e < 4096; e += 256) {
                    const int i = e >> 6, j = e & 63;
                    dbg[e] = (j < i) ? At[j * LDX + i] : 0.f;
                }
                if (ptid < 64) dbg[4096 + ptid] = al[ptid];
            }
            ut_solve(At, X, ptid);
            if (ptid == 0) EFLA_STAMP(c, 13);
            {   // T = X diag(alpha) -> bf16 K-major rows of the T operand
                uint8_t* Tt = sm + OFF_PT + s * 2 * TILE + TILE;
                const int rr = ptid & 63;
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    const int jc = 2 * (ptid >> 6) + m;
                    float v8[8];
#pragma unroll
                    for (int e = 0; e < 8; e += 4) {
                        const float4 x = *reinterpret_cast<const float4*>(X + rr * LDX + 8 * jc + e);
                        const float4 a = *reinterpret_cast<const float4*>(al + 8 * jc + e);
                        v8[e] = x.x * a.x; v8[e + 1] = x.y * a.y; v8[e + 2] = x.z * a.z; v8[e + 3] = x.w * a.w;
                    }
                    st_chunk(Tt + sw128_off(rr, jc), v8);
                    if (dbg && blockIdx.x == 0 && c == 0)
                        for (int e = 0; e < 8; ++e) dbg[4160 + rr * 64 + 8 * jc + e] = v8[e];
                }
            }
            fence_proxy_async_smem();
            bar_sync(NB_PREP, 256);
            if (ptid == 0) {
                mbar_arrive(ctl.b(B_T_READY));
                EFLA_STAMP(c, 5);
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *ctl.abort) atomicOr(err, kDevTimeout);
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
#undef EFLA_STAMP
}

// A wait on an mbarrier that nothing arrives on: exercises the bounded wait and the
// device error word (the failure-detection path) without touching any data.
__global__ void wait_timeout_selftest_kernel(uint32_t* err, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    const bool ok = mbar_wait(&bar, 0, limit_ns);
    if (!ok && threadIdx.x == 0) atomicOr(err, kDevTimeout);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// [BH][T][D] bf16 viewed as a 3-D tensor, 64 x 64 boxes, 128-byte swizzle, zero fill past T.
bool make_map(CUtensorMap* map, const void* ptr, int D, int T, long BH) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)T * D * 2};
    cuuint32_t box[3] = {64, 64, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}
}  // namespace

constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s per wait

cudaError_t launch_chunk_tc(const void* q, const void* k, const void* v, const void* beta, const float* S0,
                            void* o, float* S_T, long BH, int T, uint32_t* err, cudaStream_t stream) {
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, kD, T, BH) || !make_map(&mk, k, kD, T, BH) || !make_map(&mv, v, kD, T, BH))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    chunk_tc_kernel<<<(unsigned)(BH * 2), kThreads, SMEM_BYTES, stream>>>(
        mq, mk, mv, (const __nv_bfloat16*)beta, S0, (__nv_bfloat16*)o, S_T, T, err, kWaitLimitNs, nullptr);
    return cudaGetLastError();
}

cudaError_t launch_wait_timeout_selftest(uint32_t* err, unsigned long long limit_ns, cudaStream_t stream) {
    wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(err, limit_ns);
    return cudaGetLastError();
}

}  // namespace efla
