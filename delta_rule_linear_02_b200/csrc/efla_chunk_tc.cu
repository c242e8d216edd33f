// efla_chunk_tc.cu -- chunkwise EFLA forward on the 5th-generation tensor cores (sm_100a).
//
// bf16 q, k, v, beta -> bf16 o, fp32 state.  One CTA owns one (b, h) stream and one
// 64-column slice of d_v (d_k = d_v = 128).  The fp32 state slice S (128 x 64) lives in
// tensor memory for the whole sequence as the accumulator of S += K^T Delta.  The UT
// transform T of every chunk comes precomputed from efla_ut.cu (bf16, via TMA).
//
// Per 64-token chunk (Exact Flow Linear Attention, Section 3.3; row convention):
//   [. ; P~] = [K; Q] K^T                   M=128 MMA  (P = P~ with the causal mask, diagonal kept)
//   [. ; W | U] = [P; T] [K | V]            M=128, N=192 MMA
//   [QS; WS] = [Q; W] S                     M=128 MMA
//   Delta = U - WS                          fp32, then a bf16 operand
//   S += K^T Delta;  [O; .] = [QS; .] + [P; T] Delta               two M=128 MMAs
// Tokens past T are zero-filled by TMA (k = 0, and T's rows/columns are zero there).
//
// Warp roles (12 warps).  Only S -> [Q;W]S -> Delta -> K^T Delta -> S is sequential;
// everything that does not depend on S runs a chunk ahead on other warps:
//   warp 0       one thread polls its barriers and issues whatever is ready: the TMA
//                copies (K, Q, V, T of chunk c into a 2-deep stage ring), [K;Q]K^T and
//                [P;T][K|V]
//   warp 1       chain MMA issue: [Q;W]S, K^T Delta, [P;T]Delta
//   warps 2-3    converter: TMEM rows 64..127 -> the masked P operand, the bf16 W operand
//                and fp32 U
//   warps 4-11   chain, two warps per TMEM lane quarter (one per 32-column half): Delta,
//                the state's bf16 copy, O and the final state
// Operands are staged by TMA (128-byte swizzle, no multicast) or written in the same
// swizzled layouts.  Every wait is bounded (2 s); a wait that runs out sets a CTA-wide
// abort flag, every role winds down, and the caller's workspace records the timeout.
// `dbg` (null in the library) receives CTA 0's chunk-0 intermediates for diagnosis:
// W [8256,16448) U [16448,20544) WS [20544,24640) S after the chunk [24640,32832); and
// per chunk c < 64 the cycle at which each role passed its milestones, at
// [40000 + 16 c + k): k = 0..3 MMA issue of [K;Q]K^T, [P;T][K|V], [Q;W]S, S-update;
// 4 P ready; 6 W ready; 7 U ready; 8 Delta ready; 9 new S ready; 10 O stored; 11 TMA.
#include <cudaTypedefs.h>

#include "efla_common.cuh"
#include "efla_kernels.h"
#include "efla_tma.cuh"
#include "sm100.cuh"

namespace efla {

namespace {
using namespace sm100;

constexpr int kThreads = 384;
constexpr int kD = 128;          // d_k = d_v
constexpr int LDU = 68;          // fp32 row stride of the U rows (16-byte aligned, conflict-free)

// ---- shared-memory map (bytes from a 1024-aligned base)
// stage s (x2): [K a0 | Q a0 | W a0 | K a1 | Q a1 | W a1 | V | P | T]: 9 tiles of 64 x 64 bf16
constexpr uint32_t TILE = 8192;
constexpr uint32_t ATOM_STRIDE = 3 * TILE;          // a0 -> a1 (one 64-column half of d_k)
constexpr uint32_t ST_K = 0, ST_Q = TILE, ST_W = 2 * TILE, ST_V = 6 * TILE, ST_P = 7 * TILE, ST_T = 8 * TILE;
constexpr uint32_t STAGE_BYTES = 9 * TILE;
constexpr uint32_t OFF_STAGE = 0;
constexpr uint32_t OFF_DL = OFF_STAGE + 2 * STAGE_BYTES;   // Delta, MN-major 64 x 64
constexpr uint32_t OFF_SB = OFF_DL + TILE;                 // S bf16, MN-major 128 x 64
constexpr uint32_t OFF_U = OFF_SB + 2 * TILE;              // U rows, fp32
constexpr uint32_t OFF_BAR = OFF_U + 64 * LDU * 4;
constexpr uint32_t NBAR = 24;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
constexpr uint32_t SMEM_USED = OFF_MISC + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;          // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared-memory map exceeds 227 KB");

// ---- mbarriers (all count 1)
enum : int {
    B_FULL = 0,        // [2] TMA landed stage s
    B_STAGE_FREE = 2,  // [2] last MMA reading stage s done
    B_GP_FULL = 4, B_GP_FREE, B_P_READY, B_WU_FULL, B_WU_FREE, B_W_READY, B_U_READY, B_U_FREE,
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
constexpr int NB_CHAIN = 1, NB_DELTA = 2, NB_OUT = 3, NB_CONV = 5;
constexpr int kChainThreads = 256;   // warps 4..11: two per TMEM lane quarter, one per column half

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

__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_t,
                const float* __restrict__ S0, __nv_bfloat16* __restrict__ o, float* __restrict__ S_T,
                int T, uint32_t* __restrict__ err, unsigned long long limit_ns, float* __restrict__ dbg) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    float* Us = reinterpret_cast<float*>(sm + OFF_U);
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
        tma_prefetch_desc(&tm_t);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ================================================================ TMA + [K;Q]K^T + [P;T][K|V]
        if (lane == 0) {
            int it = 0, ia = 0, ic = 0;       // next chunk to load / to issue [K;Q]K^T / [P;T][K|V] for
            unsigned idle = 0;
            uint64_t last = globaltimer_ns();
            while (ic < nchunks) {
                if (*ctl.abort) break;
                bool did = true;
                if (ic < ia && mbar_test_wait(ctl.b(B_P_READY), ic & 1) &&
                    (ic == 0 || mbar_test_wait(ctl.b(B_WU_FREE), (ic - 1) & 1))) {
                    // [. ; W | U] = [P; T] [K | V]
                    tc_fence_after();
                    const uint32_t st = sb + OFF_STAGE + (ic & 1) * STAGE_BYTES;
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16(tmem + TM_WU, sdesc_sw128(st + ST_P + ks * 32, 16, 1024),
                                 sdesc_sw128(st + ST_K + ks * 2048, ATOM_STRIDE, 1024), ID_WU, ks > 0);
                    mma_commit(ctl.b(B_WU_FULL));
                    EFLA_STAMP(ic, 1);
                    ++ic;
                } else if (ia < it && mbar_test_wait(ctl.b(B_FULL + (ia & 1)), (ia >> 1) & 1) &&
                           (ia == 0 || mbar_test_wait(ctl.b(B_GP_FREE), (ia - 1) & 1))) {
                    // [. ; P~] = [K; Q] K^T
                    tc_fence_after();
                    const uint32_t sa = sb + OFF_STAGE + (ia & 1) * STAGE_BYTES;
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t aa = sa + (ks >> 2) * ATOM_STRIDE + ST_K + (ks & 3) * 32;
                        mma_bf16(tmem + TM_GP, sdesc_sw128(aa, 16, 1024), sdesc_sw128(aa, 16, 1024), ID_GP, ks > 0);
                    }
                    mma_commit(ctl.b(B_GP_FULL));
                    EFLA_STAMP(ia, 0);
                    ++ia;
                } else if (it < nchunks && (it < 2 || mbar_test_wait(ctl.b(B_STAGE_FREE + (it & 1)), ((it - 2) >> 1) & 1))) {
                    const int s = it & 1;
                    uint8_t* st = sm + OFF_STAGE + s * STAGE_BYTES;
                    uint64_t* full = ctl.b(B_FULL + s);
                    mbar_arrive_expect_tx(full, 6 * TILE);
                    const int t0 = it * 64;
                    tma_load_3d(st + ST_K, &tm_k, full, 0, t0, bh);
                    tma_load_3d(st + ST_Q, &tm_q, full, 0, t0, bh);
                    tma_load_3d(st + ATOM_STRIDE + ST_K, &tm_k, full, 64, t0, bh);
                    tma_load_3d(st + ATOM_STRIDE + ST_Q, &tm_q, full, 64, t0, bh);
                    tma_load_3d(st + ST_V, &tm_v, full, col0, t0, bh);
                    tma_load_2d(st + ST_T, &tm_t, full, 0, (bh * nchunks + it) * 64);
                    EFLA_STAMP(it, 11);
                    if (it + 2 < nchunks) {   // its stage frees only after this chunk: warm L2 now
                        const int t2 = t0 + 128;
                        tma_prefetch_l2_3d(&tm_k, 0, t2, bh);
                        tma_prefetch_l2_3d(&tm_q, 0, t2, bh);
                        tma_prefetch_l2_3d(&tm_k, 64, t2, bh);
                        tma_prefetch_l2_3d(&tm_q, 64, t2, bh);
                        tma_prefetch_l2_3d(&tm_v, col0, t2, bh);
                        tma_prefetch_l2_2d(&tm_t, 0, (bh * nchunks + it + 2) * 64);
                    }
                    ++it;
                } else {
                    did = false;
                }
                if (did) {
                    idle = 0;
                } else if (++idle >= 512) {   // read the clock only now and then
                    idle = 0;
                    const uint64_t now = globaltimer_ns();
                    if (now - last > limit_ns) {
                        *ctl.abort = 1;
                        break;
                    }
                    continue;
                }
                if (did) last = globaltimer_ns();
            }
            // every copy and MMA this thread issued has landed before the CTA can exit
            mma_commit(ctl.b(B_DRAIN));
            mbar_wait(ctl.b(B_DRAIN), 0, limit_ns);
            for (int c = max(0, it - 2); c < it; ++c) mbar_wait(ctl.b(B_FULL + (c & 1)), (c >> 1) & 1, limit_ns);
        }
    } else if (warp == 1) {
        // ================================================================ chain issuer
        if (lane == 0) {
            bool ok = true;
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
                // S += K^T Delta, then [O; .] += [P; T] Delta
                if (!(ok = ctl.wait(B_D_READY, c & 1))) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + TM_S, sdesc_sw128(st + ST_K + ks * 2048, ATOM_STRIDE, 1024),
                             sdesc_sw128(sb + OFF_DL + ks * 2048, TILE, 1024), ID_S, 1);
                mma_commit(ctl.b(B_S_FULL));
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + TM_Y + 64 * s, sdesc_sw128(st + ST_P + ks * 32, 16, 1024),
                             sdesc_sw128(sb + OFF_DL + ks * 2048, TILE, 1024), ID_Y, 1);
                mma_commit(ctl.b(B_O_FULL + s));
                mma_commit(ctl.b(B_STAGE_FREE + s));
                EFLA_STAMP(c, 3);
            }
            mma_commit(ctl.b(B_DRAIN + 1));
            mbar_wait(ctl.b(B_DRAIN + 1), 0, limit_ns);
        }
    } else if (warp < 4) {
        // ================================================================ converter (TMEM lanes 64..127)
        const int r = tid - 64;                       // chunk row
        bool ok = true;
        for (int c = 0; c < nchunks && ok; ++c) {
            const int s = c & 1;
            uint8_t* st = sm + OFF_STAGE + s * STAGE_BYTES;
            // P = P~ with the causal mask (diagonal kept) -> bf16 K-major rows
            ok = bar_and(NB_CONV, 64, ctl.wait(B_GP_FULL, c & 1));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int qd = 0; qd < 4; ++qd) {
                float t16[16];
                tmem_ld16(tmem + lane_off + TM_GP + 16 * qd, t16);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) t16[j] = (16 * qd + j <= r) ? t16[j] : 0.f;
                st_chunk(st + ST_P + sw128_off(r, 2 * qd), t16);
                st_chunk(st + ST_P + sw128_off(r, 2 * qd + 1), t16 + 8);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            bar_sync(NB_CONV, 64);
            if (r == 0) {
                mbar_arrive(ctl.b(B_GP_FREE));
                mbar_arrive(ctl.b(B_P_READY));
                EFLA_STAMP(c, 4);
            }
            // W row r -> bf16, K-major, two 64-column atoms
            ok = bar_and(NB_CONV, 64, ctl.wait(B_WU_FULL, c & 1));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int qd = 0; qd < 8; ++qd) {
                float w16[16];
                tmem_ld16(tmem + lane_off + TM_WU + 16 * qd, w16);
                tmem_wait_ld();
                uint8_t* dst = st + (qd >> 2) * ATOM_STRIDE + ST_W;
                st_chunk(dst + sw128_off(r, (qd & 3) * 2), w16);
                st_chunk(dst + sw128_off(r, (qd & 3) * 2 + 1), w16 + 8);
                if (dbg && blockIdx.x == 0 && c == 0)
                    for (int j = 0; j < 16; ++j) dbg[8256 + r * 128 + 16 * qd + j] = w16[j];
            }
            fence_proxy_async_smem();
            bar_sync(NB_CONV, 64);
            if (r == 0) {
                mbar_arrive(ctl.b(B_W_READY));
                EFLA_STAMP(c, 6);
            }
            // U row r stays fp32 (after the chain has read the previous chunk's)
            ok = bar_and(NB_CONV, 64, c == 0 || ctl.wait(B_U_FREE, (c - 1) & 1));
            if (!ok) break;
#pragma unroll
            for (int qd = 0; qd < 4; ++qd) {
                float u16[16];
                tmem_ld16(tmem + lane_off + TM_WU + 128 + 16 * qd, u16);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; j += 4)
                    *reinterpret_cast<float4*>(Us + r * LDU + 16 * qd + j) = make_float4(u16[j], u16[j + 1], u16[j + 2], u16[j + 3]);
                if (dbg && blockIdx.x == 0 && c == 0)
                    for (int j = 0; j < 16; ++j) dbg[16448 + r * 64 + 16 * qd + j] = u16[j];
            }
            tc_fence_before();
            bar_sync(NB_CONV, 64);
            if (r == 0) {
                mbar_arrive(ctl.b(B_U_READY));
                mbar_arrive(ctl.b(B_WU_FREE));
                EFLA_STAMP(c, 7);
            }
        }
    } else {
        // ================================================================ chain (TMEM lanes 0..127)
        const int q = warp & 3;                       // TMEM lane quarter
        const int ch = (warp - 4) >> 2;               // column half: 32 of this CTA's 64 columns
        const int ct = 32 * q + lane;                 // d_k row for S; rows of Y by quarter
        const int cc = 32 * ch;                       // first column of this thread's half
        {   // initial state
            const float* src = S0 ? S0 + ((size_t)bh * kD + ct) * kD + col0 + cc : nullptr;
#pragma unroll
            for (int qd = 0; qd < 2; ++qd) {
                float s16[16];
#pragma unroll
                for (int j = 0; j < 16; j += 4) {
                    float4 x = src ? *reinterpret_cast<const float4*>(src + 16 * qd + j) : make_float4(0.f, 0.f, 0.f, 0.f);
                    s16[j] = x.x; s16[j + 1] = x.y; s16[j + 2] = x.z; s16[j + 3] = x.w;
                }
                tmem_st16(tmem + lane_off + TM_S + cc + 16 * qd, s16);
                st_chunk(sm + OFF_SB + sw128_off(ct, 4 * ch + 2 * qd), s16);
                st_chunk(sm + OFF_SB + sw128_off(ct, 4 * ch + 2 * qd + 1), s16 + 8);
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            bar_sync(NB_CHAIN, kChainThreads);
            if (warp == 4 && lane == 0) mbar_arrive(ctl.b(B_SB_READY));
        }
        bool ok = true;
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            const uint32_t tY = tmem + lane_off + TM_Y + 64 * b + cc;
            if (q >= 2) {                             // Delta = U - WS (rows 64..127 of Y)
                const int r = ct - 64;
                bool w = ok && ctl.wait(B_Y_FULL + b, (c >> 1) & 1) && ctl.wait(B_U_READY, c & 1);
                w = bar_and(NB_DELTA, 128, w);
                if (w) {
                    tc_fence_after();
#pragma unroll
                    for (int qd = 0; qd < 2; ++qd) {
                        float t16[16];
                        tmem_ld16(tY + 16 * qd, t16);
                        tmem_wait_ld();
                        if (dbg && blockIdx.x == 0 && c == 0)
                            for (int j = 0; j < 16; ++j) dbg[20544 + r * 64 + cc + 16 * qd + j] = t16[j];
#pragma unroll
                        for (int j = 0; j < 16; j += 4) {
                            const float4 u = *reinterpret_cast<const float4*>(Us + r * LDU + cc + 16 * qd + j);
                            t16[j] = u.x - t16[j];
                            t16[j + 1] = u.y - t16[j + 1];
                            t16[j + 2] = u.z - t16[j + 2];
                            t16[j + 3] = u.w - t16[j + 3];
                        }
                        st_chunk(sm + OFF_DL + sw128_off(r, 4 * ch + 2 * qd), t16);
                        st_chunk(sm + OFF_DL + sw128_off(r, 4 * ch + 2 * qd + 1), t16 + 8);
                    }
                    fence_proxy_async_smem();
                    tc_fence_before();
                    bar_sync(NB_DELTA, 128);
                    if (warp == 6 && lane == 0) {
                        mbar_arrive(ctl.b(B_D_READY));
                        mbar_arrive(ctl.b(B_U_FREE));
                        EFLA_STAMP(c, 8);
                    }
                }
                ok = w;
            }
            // the new state: bf16 operand for the next chunk (and S_T after the last)
            ok = bar_and(NB_CHAIN, kChainThreads, ok && ctl.wait(B_S_FULL, c & 1));
            if (!ok) break;
            tc_fence_after();
            const bool last = (c == nchunks - 1);
#pragma unroll
            for (int qd = 0; qd < 2; ++qd) {
                float t16[16];
                tmem_ld16(tmem + lane_off + TM_S + cc + 16 * qd, t16);
                tmem_wait_ld();
                st_chunk(sm + OFF_SB + sw128_off(ct, 4 * ch + 2 * qd), t16);
                st_chunk(sm + OFF_SB + sw128_off(ct, 4 * ch + 2 * qd + 1), t16 + 8);
                if (dbg && blockIdx.x == 0 && c == 0)
                    for (int j = 0; j < 16; ++j) dbg[24640 + ct * 64 + cc + 16 * qd + j] = t16[j];
                if (last && S_T) {
                    float* dst = S_T + ((size_t)bh * kD + ct) * kD + col0 + cc + 16 * qd;
#pragma unroll
                    for (int j = 0; j < 16; j += 4)
                        *reinterpret_cast<float4*>(dst + j) = make_float4(t16[j], t16[j + 1], t16[j + 2], t16[j + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            bar_sync(NB_CHAIN, kChainThreads);
            if (warp == 4 && lane == 0) {
                mbar_arrive(ctl.b(B_SB_READY));
                EFLA_STAMP(c, 9);
            }
            if (q < 2) {                              // O rows (lanes 0..63 of Y)
                const int r = ct;
                bool w = bar_and(NB_OUT, 128, ctl.wait(B_O_FULL + b, (c >> 1) & 1));
                if (w) {
                    tc_fence_after();
                    const int t0 = c * 64;
                    const bool live = r < min(64, T - t0);
#pragma unroll
                    for (int qd = 0; qd < 2; ++qd) {
                        float t16[16];
                        tmem_ld16(tY + 16 * qd, t16);
                        tmem_wait_ld();
                        if (live) {
                            uint4* dst = reinterpret_cast<uint4*>(o + (tok0 + t0 + r) * kD + col0 + cc + 16 * qd);
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
                    bar_sync(NB_OUT, 128);
                    if (warp == 4 && lane == 0) {
                        mbar_arrive(ctl.b(B_Y_FREE + b));
                        EFLA_STAMP(c, 10);
                    }
                }
                ok = w;
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
}  // namespace

constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s per wait

size_t chunk_tc_workspace_bytes(long BH, int T) {
    const long nchunks = (T + 63) / 64;
    return (size_t)BH * nchunks * 64 * 64 * 2;     // the bf16 T of every chunk
}

cudaError_t launch_chunk_tc(const void* q, const void* k, const void* v, const void* beta, const float* S0,
                            void* o, float* S_T, long BH, int T, uint32_t* err, void* scratch,
                            cudaStream_t stream) {
    const int nchunks = (T + 63) / 64;
    cudaError_t e = launch_ut(k, beta, scratch, BH, T, err, kWaitLimitNs, stream);
    if (e != cudaSuccess) return e;
    CUtensorMap mq, mk, mv, mt;
    if (!tma_map_tokens(&mq, q, kD, T, BH) || !tma_map_tokens(&mk, k, kD, T, BH) ||
        !tma_map_tokens(&mv, v, kD, T, BH) || !tma_map_rows64(&mt, scratch, BH * nchunks * 64))
        return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    chunk_tc_kernel<<<(unsigned)(BH * 2), kThreads, SMEM_BYTES, stream>>>(mq, mk, mv, mt, S0, (__nv_bfloat16*)o,
                                                                          S_T, T, err, kWaitLimitNs, nullptr);
    return cudaGetLastError();
}

cudaError_t launch_wait_timeout_selftest(uint32_t* err, unsigned long long limit_ns, cudaStream_t stream) {
    wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(err, limit_ns);
    return cudaGetLastError();
}

}  // namespace efla
