// efla_chunk_tc.cu -- chunkwise EFLA forward on the 5th-generation tensor cores (sm_100a).
//
// bf16 q, k, v, beta -> bf16 o, fp32 state.  One CTA owns one (b, h) stream and one
// 64-column slice of d_v (d_k = d_v = 128).  The fp32 state slice S (128 x 64) lives in
// tensor memory for the whole sequence as the accumulator of S += K^T Delta.  The UT
// transform T of every chunk comes precomputed from efla_ut.cu (bf16, via TMA).
//
// Per 64-token chunk (Exact Flow Linear Attention, Section 3.3; row convention):
//   [W | U] = T [K | V]                      (M=64, N=192)
//   X = [W; Q] S                             (M=128: rows 0-63 W S, rows 64-127 Q S)
//   Delta = U - W S                          fp32, then a bf16 operand
//   S += K^T Delta                           (M=128)
//   P~ = Q K^T, P = P~ masked causally (diagonal kept)               (M=64)
//   X += [Delta'; P] Delta                   (M=128: rows 64-127 become O = Q S + P Delta;
//                                             rows 0-63, W S already consumed, take junk)
// Tokens past T are zero-filled by TMA (k = 0, and T's rows/columns are zero there).
// Stacking W over Q makes Q S free: an M=128 MMA issues as fast as an M=64 one.
//
// One warp issues every MMA, in a fixed order per chunk c:
//   [W;Q] S(c), [W|U](c+1), K^T Delta(c) (after Delta), P Delta(c), Q K^T(c+1)
// so that the state chain ([W;Q] S, K^T Delta) never queues behind work that could wait;
// the others fill the in-order tensor pipe while the chain's epilogues run.  Issue is by
// a converged warp with elect.sync (warp-uniform control flow keeps the descriptors in
// uniform registers; a one-lane issuer in a data-dependent loop issues far slower).
// What bounds a chunk step here is shared memory: an N = 64 MMA reads about 6 KB of
// operands in the ~47 cycles it takes, close to the SM's shared-memory bandwidth, and
// while it runs the CUDA-core epilogues' shared loads and stores (and every mbarrier
// probe) wait several times longer than on an idle pipe.  A chunk moves about 256 KB
// through shared memory (TMA writes, MMA operand reads, epilogue writes).
//
// Shared memory: two TMA rings, so each load has a chunk period or more of lead time.
//   KVT ring (3 deep): [K a0 | K a1 | V | T] of chunk c (K, V half, T: 4 x 8 KiB)
//   WQ ring (2 deep):  [W a0 | Q a0 | W a1 | Q a1] of chunk c (Q by TMA, W by the converter),
//                      so that [W; Q] is one 128-row K-major operand per 64-column atom
//   Delta (MN-major) directly followed by P (K-major): the 128-row operand [Delta'; P]
//   S bf16 (MN-major 128 x 64), U fp32 rows.
//
// Warp roles (14 warps):
//   warp 0       TMA producer (no multicast), L2 prefetch ahead
//   warp 1       MMA issuer
//   warps 2-5    converter, one per TMEM lane quarter (the M=64 products keep row r in
//                lane (r%16) + 32(r/16)): W -> bf16 operand, U -> fp32 rows, P~ -> P
//   warps 6-13   chain, two per lane quarter (32-column halves).  Quarters 0-1 form Delta
//                from X rows 0-63; quarters 2-3 store O from X rows 64-127 (so O of chunk
//                c overlaps Delta of chunk c+1); all eight rebuild the bf16 S and S_T.
// Every wait is bounded (2 s); a wait that runs out sets a CTA-wide abort flag, every
// role winds down, and the caller's workspace records the timeout.
// `dbg` (null in the library) receives CTA 0's chunk-0 intermediates for diagnosis:
// W [8256,16448) U [16448,20544) WS [20544,24640) S after the chunk [24640,32832); and
// per chunk c < 64 the cycle at which each role passed its milestones, at
// [40000 + 16 c + k): k = 0 QK^T, 1 [W|U], 2 [W;Q]S, 3 K^T Delta issued; 4 P ready;
// 6 W ready; 7 U ready; 8 Delta ready; 9 new S ready; 10 O stored; 11 TMA issued.
#include <cudaTypedefs.h>

#include "efla_common.cuh"
#include "efla_kernels.h"
#include "efla_tma.cuh"
#include "sm100.cuh"

namespace efla {

namespace {
using namespace sm100;

constexpr int kThreads = 448;
constexpr int kD = 128;          // d_k = d_v
constexpr int LDU = 68;          // fp32 row stride of the U rows (16-byte aligned, conflict-free)
constexpr int kKvtStages = 3, kWqStages = 2;

// ---- shared-memory map (bytes from a 1024-aligned base); tiles are 64 x 64 bf16, SW128
constexpr uint32_t TILE = 8192;
constexpr uint32_t KVT_K = 0, KVT_V = 2 * TILE, KVT_T = 3 * TILE, KVT_BYTES = 4 * TILE;
constexpr uint32_t WQ_W = 0, WQ_Q = TILE, WQ_ATOM = 2 * TILE, WQ_BYTES = 4 * TILE;
constexpr uint32_t OFF_KVT = 0;
constexpr uint32_t OFF_WQ = OFF_KVT + kKvtStages * KVT_BYTES;
constexpr uint32_t OFF_DL = OFF_WQ + kWqStages * WQ_BYTES;     // Delta, MN-major 64 x 64
constexpr uint32_t OFF_P = OFF_DL + TILE;                      // P, K-major 64 x 64 (follows Delta)
constexpr uint32_t OFF_SB = OFF_P + TILE;                      // S bf16, MN-major 128 x 64
constexpr uint32_t OFF_U = OFF_SB + 2 * TILE;                  // U rows, fp32
constexpr uint32_t OFF_BAR = OFF_U + 64 * LDU * 4;
constexpr uint32_t NBAR = 32;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
constexpr uint32_t SMEM_USED = OFF_MISC + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;          // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared-memory map exceeds 227 KB");

// ---- mbarriers (all count 1)
enum : int {
    B_KVT_FULL = 0,     // [3] TMA landed K, V, T of a stage
    B_KVT_FREE = 3,     // [3] the last MMA reading that stage is done
    B_WQ_FULL = 6,      // [2] TMA landed Q of a stage
    B_WQ_FREE = 8,      // [2] [W;Q] S of that stage is done
    B_GP_FULL = 10, B_GP_FREE, B_P_READY, B_WU_FULL, B_WU_FREE, B_W_READY, B_U_READY, B_U_FREE,
    B_XS_FULL = 18,     // [2] [W;Q] S landed in X[b]
    B_D_READY = 20, B_S_FULL, B_SB_READY,
    B_O_FULL = 23,      // [2] O complete in X[b]
    B_X_FREE = 25,      // [2] O of X[b] stored
    B_DRAIN = 27,
};

// ---- TMEM columns (fp32 accumulators)
constexpr uint32_t TM_S = 0;          // M=128: S (d_k x 64)
constexpr uint32_t TM_X = 64;         // M=128, x2: [W;Q] S, then + [Delta'; P] Delta
constexpr uint32_t TM_GP = 192;       // M=64:  Q K^T
constexpr uint32_t TM_WU = 256;       // M=64, N=192: [W | U]
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t ID_QK = idesc_bf16(64, 64, false, false);
constexpr uint32_t ID_WU = idesc_bf16(64, 192, false, true);
constexpr uint32_t ID_X = idesc_bf16(128, 64, false, true);     // [W;Q] S and [Delta'; P] Delta
constexpr uint32_t ID_S = idesc_bf16(128, 64, true, true);      // K^T Delta

// ---- named barriers
constexpr int NB_CONV = 1, NB_DELTA = 2, NB_OUT = 3, NB_CHAIN = 4;
constexpr int kConvThreads = 128, kHalfChain = 128, kChainThreads = 256;

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
    // bounded wait; gives up early once another role has aborted.  A phase that has
    // already completed is seen by one non-blocking probe.
    __device__ bool wait(int i, uint32_t parity) const {
        if (mbar_test_wait(bar + i, parity)) return true;
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

// One accumulator tile: nk tcgen05.mma of K = 16, issued by a converged warp.  Operand
// k-step ks starts at base + (ks / 4) * atom + (ks % 4) * step (a K-major operand walks
// 32 bytes within a 64-column swizzle atom and jumps `atom` bytes between atoms; an
// MN-major operand walks 16 rows = 2048 bytes, atom = 8192).
__device__ __forceinline__ void mma_group(uint32_t d, uint32_t a, uint32_t a_atom, uint32_t a_step, uint32_t a_lbo,
                                          uint32_t b, uint32_t b_atom, uint32_t b_step, uint32_t b_lbo,
                                          uint32_t idesc, int nk, uint32_t acc) {
#pragma unroll
    for (int ks = 0; ks < nk; ++ks) {
        mma_bf16_elect(d, sdesc_sw128(a + (ks >> 2) * a_atom + (ks & 3) * a_step, a_lbo, 1024),
                       sdesc_sw128(b + (ks >> 2) * b_atom + (ks & 3) * b_step, b_lbo, 1024), idesc, (acc | ks) != 0);
    }
}

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
    const int q = warp & 3;                                                  // TMEM lane quarter
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const int bh = blockIdx.x >> 1;
    const int col0 = (blockIdx.x & 1) * 64;
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
    auto kvt = [&](int c) { return OFF_KVT + (uint32_t)(c % kKvtStages) * KVT_BYTES; };   // byte offsets
    auto wq = [&](int c) { return OFF_WQ + (uint32_t)(c % kWqStages) * WQ_BYTES; };

    if (warp == 0) {
        // ================================================================ TMA producer
        if (lane == 0) {
            bool ok = true;
            int kvt_issued = 0, wq_issued = 0;
            for (int c = 0; c < nchunks && ok; ++c) {
                const int t0 = c * 64;
                {   // K, V, T of chunk c
                    const int s = c % kKvtStages;
                    if (c >= kKvtStages && !(ok = ctl.wait(B_KVT_FREE + s, ((c - kKvtStages) / kKvtStages) & 1))) break;
                    uint8_t* st = sm + kvt(c);
                    uint64_t* full = ctl.b(B_KVT_FULL + s);
                    mbar_arrive_expect_tx(full, 4 * TILE);
                    tma_load_3d(st + KVT_K, &tm_k, full, 0, t0, bh);
                    tma_load_3d(st + KVT_K + TILE, &tm_k, full, 64, t0, bh);
                    tma_load_3d(st + KVT_V, &tm_v, full, col0, t0, bh);
                    tma_load_2d(st + KVT_T, &tm_t, full, 0, (bh * nchunks + c) * 64);
                    kvt_issued = c + 1;
                }
                {   // Q of chunk c
                    const int s = c % kWqStages;
                    if (c >= kWqStages && !(ok = ctl.wait(B_WQ_FREE + s, ((c - kWqStages) / kWqStages) & 1))) break;
                    uint8_t* st = sm + wq(c);
                    uint64_t* full = ctl.b(B_WQ_FULL + s);
                    mbar_arrive_expect_tx(full, 2 * TILE);
                    tma_load_3d(st + WQ_Q, &tm_q, full, 0, t0, bh);
                    tma_load_3d(st + WQ_Q + WQ_ATOM, &tm_q, full, 64, t0, bh);
                    wq_issued = c + 1;
                }
                EFLA_STAMP(c, 11);
                if (c + 3 < nchunks) {      // warm L2 for the chunk three ahead
                    const int t3 = t0 + 192;
                    tma_prefetch_l2_3d(&tm_k, 0, t3, bh);
                    tma_prefetch_l2_3d(&tm_k, 64, t3, bh);
                    tma_prefetch_l2_3d(&tm_v, col0, t3, bh);
                    tma_prefetch_l2_3d(&tm_q, 0, t3, bh);
                    tma_prefetch_l2_3d(&tm_q, 64, t3, bh);
                    tma_prefetch_l2_2d(&tm_t, 0, (bh * nchunks + c + 3) * 64);
                }
            }
            // no copy may land after exit
            for (int c = max(0, kvt_issued - kKvtStages); c < kvt_issued; ++c)
                mbar_wait(ctl.b(B_KVT_FULL + c % kKvtStages), (c / kKvtStages) & 1, limit_ns);
            for (int c = max(0, wq_issued - kWqStages); c < wq_issued; ++c)
                mbar_wait(ctl.b(B_WQ_FULL + c % kWqStages), (c / kWqStages) & 1, limit_ns);
        }
    } else if (warp == 1) {
        // ================================================================ MMA issuer (whole warp)
        // Warp-uniform control flow: every lane polls the barrier and the warp votes;
        // elect.sync inside each MMA and commit picks the issuing lane.
        auto wait = [&](int i, uint32_t parity) { return __all_sync(0xffffffffu, ctl.wait(i, parity)); };
        auto issue_qk = [&](int c) {      // P~ = Q K^T (M = 64)
            tc_fence_after();
            mma_group(tmem + TM_GP, sb + wq(c) + WQ_Q, WQ_ATOM, 32, 16, sb + kvt(c) + KVT_K, TILE, 32, 16, ID_QK, 8, 0);
            mma_commit_elect(ctl.b(B_GP_FULL));
            EFLA_STAMP(c, 0);
        };
        auto issue_wu = [&](int c) {      // [W | U] = T [K | V] (M = 64, N = 192)
            tc_fence_after();
            const uint32_t st = sb + kvt(c);
            mma_group(tmem + TM_WU, st + KVT_T, TILE, 32, 16, st + KVT_K, 4 * 2048, 2048, TILE, ID_WU, 4, 0);
            mma_commit_elect(ctl.b(B_WU_FULL));
            EFLA_STAMP(c, 1);
        };
        bool ok = wait(B_KVT_FULL, 0) && wait(B_WQ_FULL, 0);
        if (ok) {
            issue_qk(0);
            issue_wu(0);
        }
        for (int c = 0; c < nchunks && ok; ++c) {
            const int b = c & 1;
            const uint32_t kv = sb + kvt(c), x = tmem + TM_X + 64 * b;
            // X = [W; Q] S (state chain)
            if (!(ok = wait(B_W_READY, c & 1) && wait(B_SB_READY, c & 1) &&
                       (c < 2 || wait(B_X_FREE + b, ((c - 2) >> 1) & 1)))) break;
            tc_fence_after();
            mma_group(x, sb + wq(c) + WQ_W, WQ_ATOM, 32, 16, sb + OFF_SB, 4 * 2048, 2048, TILE, ID_X, 8, 0);
            mma_commit_elect(ctl.b(B_XS_FULL + b));
            mma_commit_elect(ctl.b(B_WQ_FREE + c % kWqStages));
            EFLA_STAMP(c, 2);
            // the next chunk's [W | U] fills the pipe while Delta is formed
            if (c + 1 < nchunks) {
                if (!(ok = wait(B_KVT_FULL + (c + 1) % kKvtStages, ((c + 1) / kKvtStages) & 1) &&
                           wait(B_WU_FREE, c & 1))) break;
                issue_wu(c + 1);
            }
            // S += K^T Delta (state chain)
            if (!(ok = wait(B_D_READY, c & 1))) break;
            tc_fence_after();
            mma_group(tmem + TM_S, kv + KVT_K, 4 * 2048, 2048, TILE, sb + OFF_DL, 4 * 2048, 2048, TILE, ID_S, 4, 1);
            mma_commit_elect(ctl.b(B_S_FULL));
            mma_commit_elect(ctl.b(B_KVT_FREE + c % kKvtStages));
            EFLA_STAMP(c, 3);
            // X += [Delta'; P] Delta: rows 64-127 become O = Q S + P Delta
            if (!(ok = wait(B_P_READY, c & 1))) break;
            tc_fence_after();
            mma_group(x, sb + OFF_DL, TILE, 32, 16, sb + OFF_DL, 4 * 2048, 2048, TILE, ID_X, 4, 1);
            mma_commit_elect(ctl.b(B_O_FULL + b));
            // the next chunk's Q K^T
            if (c + 1 < nchunks) {
                if (!(ok = wait(B_WQ_FULL + (c + 1) % kWqStages, ((c + 1) / kWqStages) & 1) &&
                           wait(B_GP_FREE, c & 1))) break;
                issue_qk(c + 1);
            }
        }
        mma_commit_elect(ctl.b(B_DRAIN));
        if (lane == 0) mbar_wait(ctl.b(B_DRAIN), 0, limit_ns);
        __syncwarp();
    } else if (warp < 6) {
        // ================================================================ converter (one warp per lane quarter)
        const int r = 16 * q + lane;                  // chunk row held by lanes 0..15
        const bool act = lane < 16;
        bool ok = true;
        for (int c = 0; c < nchunks && ok; ++c) {
            // W row r -> bf16, K-major, into the [W; Q] operand of chunk c
            ok = bar_and(NB_CONV, kConvThreads, ctl.wait(B_WU_FULL, c & 1));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float w[64];
                tmem_ld64_wait(tmem + lane_off + TM_WU + 64 * h, w);
                if (act) {
                    uint8_t* dst = sm + wq(c) + WQ_W + h * WQ_ATOM;
#pragma unroll
                    for (int j = 0; j < 8; ++j) st_chunk(dst + sw128_off(r, j), w + 8 * j);
                    if (dbg && blockIdx.x == 0 && c == 0)
                        for (int j = 0; j < 64; ++j) dbg[8256 + r * 128 + 64 * h + j] = w[j];
                }
            }
            fence_proxy_async_smem();
            bar_sync(NB_CONV, kConvThreads);
            if (warp == 2 && lane == 0) {
                mbar_arrive(ctl.b(B_W_READY));
                EFLA_STAMP(c, 6);
            }
            // U row r stays fp32 (after the chain has read the previous chunk's)
            ok = bar_and(NB_CONV, kConvThreads, c == 0 || ctl.wait(B_U_FREE, (c - 1) & 1));
            if (!ok) break;
            {
                float u[64];
                tmem_ld64_wait(tmem + lane_off + TM_WU + 128, u);
                if (act) {
#pragma unroll
                    for (int j = 0; j < 64; j += 4)
                        *reinterpret_cast<float4*>(Us + r * LDU + j) = make_float4(u[j], u[j + 1], u[j + 2], u[j + 3]);
                    if (dbg && blockIdx.x == 0 && c == 0)
                        for (int j = 0; j < 64; ++j) dbg[16448 + r * 64 + j] = u[j];
                }
            }
            tc_fence_before();
            bar_sync(NB_CONV, kConvThreads);
            if (warp == 2 && lane == 0) {
                mbar_arrive(ctl.b(B_U_READY));
                mbar_arrive(ctl.b(B_WU_FREE));
                EFLA_STAMP(c, 7);
            }
            // P = P~ with the causal mask (diagonal kept) -> bf16 K-major rows
            ok = bar_and(NB_CONV, kConvThreads, ctl.wait(B_GP_FULL, c & 1));
            if (!ok) break;
            tc_fence_after();
            {
                float t[64];
                tmem_ld64_wait(tmem + lane_off + TM_GP, t);
                if (act) {
#pragma unroll
                    for (int j = 0; j < 64; ++j) t[j] = (j <= r) ? t[j] : 0.f;
#pragma unroll
                    for (int j = 0; j < 8; ++j) st_chunk(sm + OFF_P + sw128_off(r, j), t + 8 * j);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            bar_sync(NB_CONV, kConvThreads);
            if (warp == 2 && lane == 0) {
                mbar_arrive(ctl.b(B_GP_FREE));
                mbar_arrive(ctl.b(B_P_READY));
                EFLA_STAMP(c, 4);
            }
        }
    } else {
        // ================================================================ chain (two warps per lane quarter)
        // Quarters 0-1 (X rows 0-63, W S) form Delta; quarters 2-3 (X rows 64-127) store O.
        // The groups meet at the S epilogue; a group that gives up still reaches the next
        // S-epilogue barrier with ok = false, so both groups stop together.
        const int ch = (warp - 6) >> 2;               // column half: 32 of this CTA's 64 columns
        const int cc = 32 * ch;
        const int ct = 32 * q + lane;                 // d_k row of S, and row of X
        const bool delta_group = q < 2;
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
            if (warp == 6 && lane == 0) mbar_arrive(ctl.b(B_SB_READY));
        }
        bool ok = true;
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            const uint32_t x = tmem + lane_off + TM_X + 64 * b + cc;
            if (delta_group && ok) {
                // Delta = U - W S (X rows 0-63)
                ok = bar_and(NB_DELTA, kHalfChain, ctl.wait(B_XS_FULL + b, (c >> 1) & 1) && ctl.wait(B_U_READY, c & 1));
                if (ok) {
                    tc_fence_after();
                    float t[32];
                    tmem_ld32_wait(x, t);
                    if (dbg && blockIdx.x == 0 && c == 0)
                        for (int j = 0; j < 32; ++j) dbg[20544 + ct * 64 + cc + j] = t[j];
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        const float4 u = *reinterpret_cast<const float4*>(Us + ct * LDU + cc + j);
                        t[j] = u.x - t[j];
                        t[j + 1] = u.y - t[j + 1];
                        t[j + 2] = u.z - t[j + 2];
                        t[j + 3] = u.w - t[j + 3];
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) st_chunk(sm + OFF_DL + sw128_off(ct, 4 * ch + j), t + 8 * j);
                    fence_proxy_async_smem();
                    tc_fence_before();
                    bar_sync(NB_DELTA, kHalfChain);
                    if (warp == 8 && lane == 0) {
                        mbar_arrive(ctl.b(B_D_READY));
                        mbar_arrive(ctl.b(B_U_FREE));
                        EFLA_STAMP(c, 8);
                    }
                }
            }
            // the new state: bf16 operand for the next chunk (and S_T after the last)
            ok = bar_and(NB_CHAIN, kChainThreads, ok && ctl.wait(B_S_FULL, c & 1));
            if (!ok) break;
            tc_fence_after();
            {
                float t[32];
                tmem_ld32_wait(tmem + lane_off + TM_S + cc, t);
#pragma unroll
                for (int j = 0; j < 4; ++j) st_chunk(sm + OFF_SB + sw128_off(ct, 4 * ch + j), t + 8 * j);
                if (dbg && blockIdx.x == 0 && c == 0)
                    for (int j = 0; j < 32; ++j) dbg[24640 + ct * 64 + cc + j] = t[j];
                if (c == nchunks - 1 && S_T) {
                    float* dst = S_T + ((size_t)bh * kD + ct) * kD + col0 + cc;
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4*>(dst + j) = make_float4(t[j], t[j + 1], t[j + 2], t[j + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            bar_sync(NB_CHAIN, kChainThreads);
            if (warp == 6 && lane == 0) {
                mbar_arrive(ctl.b(B_SB_READY));
                EFLA_STAMP(c, 9);
            }
            if (!delta_group) {
                // O = Q S + P Delta (X rows 64-127) -> bf16 global
                ok = bar_and(NB_OUT, kHalfChain, ctl.wait(B_O_FULL + b, (c >> 1) & 1));
                if (ok) {
                    tc_fence_after();
                    const int r = ct - 64, t0 = c * 64;
                    float t[32];
                    tmem_ld32_wait(x, t);
                    if (r < min(64, T - t0)) {
                        uint4* dst = reinterpret_cast<uint4*>(o + (tok0 + t0 + r) * kD + col0 + cc);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            uint4 y;
                            y.x = pack_bf16x2(t[8 * j], t[8 * j + 1]);
                            y.y = pack_bf16x2(t[8 * j + 2], t[8 * j + 3]);
                            y.z = pack_bf16x2(t[8 * j + 4], t[8 * j + 5]);
                            y.w = pack_bf16x2(t[8 * j + 6], t[8 * j + 7]);
                            dst[j] = y;
                        }
                    }
                    tc_fence_before();
                    bar_sync(NB_OUT, kHalfChain);
                    if (warp == 6 && lane == 0) {
                        mbar_arrive(ctl.b(B_X_FREE + b));
                        EFLA_STAMP(c, 10);
                    }
                }
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
