// efla_chunk_tc.cu -- chunkwise EFLA forward on the 5th-generation tensor cores (sm_100a).
//
// bf16 q, k, v, beta -> bf16 o, fp32 state.  One CTA owns one (b, h) stream and one
// 64-column slice of d_v (d_k = d_v = 128).  The fp32 state slice S (128 x 64) lives in
// tensor memory for the whole sequence as the accumulator of S += K^T Delta.  The UT
// transform T of every chunk comes precomputed from efla_ut.cu (bf16, via TMA).
//
// Per 64-token chunk (Exact Flow Linear Attention, Section 3.3; row convention), all
// products M = 128 (row m of a result in TMEM lane m):
//   [W | U] = [T; *] [K | V]                 (N=192; rows 64-127 unused)
//   X = [W; Q] S                             (rows 0-63 W S, rows 64-127 Q S)
//   Delta = U - W S                          fp32, then a bf16 operand
//   S += K^T Delta
//   P~ = [W; Q] K^T                          (rows 64-127 Q K^T), P = P~ masked causally,
//                                             diagonal kept
//   X += [*; P] Delta                        (rows 64-127 become O = Q S + P Delta)
// Tokens past T are zero-filled by TMA (k = 0, and T's rows/columns are zero there).
//
// The A operands [W; Q] and [*; P] live in tensor memory (bf16, K-major: TMEM column j of
// lane m holds elements 2j and 2j + 1 of row m): an N = 64 MMA with A in tensor memory
// runs at the tensor core's math rate (~33 cycles), one with both operands in shared
// memory at the shared-memory bandwidth (~49 cycles).  W goes from its fp32 accumulator
// to the A operand without touching shared memory, P likewise, Q is copied in once, and
// U is read by the Delta warps straight from its accumulator.  Shared memory then holds
// only the TMA tiles (K, V, T, Q), Delta and the bf16 copy of S.
//
// A chunk step is bound by latency, not by a unit's throughput: its MMAs take ~1,240
// tensor-pipe cycles, and the rest of a step is the hand-offs of the chain
// [W;Q] S -> Delta -> K^T Delta -> bf16 S -> the next [W;Q] S between roles.
//
// One warp issues every MMA, in a fixed order per chunk c:
//   [W;Q] S(c), Q K^T(c), K^T Delta(c) (after Delta), P Delta(c), [W|U](c+2)
// so that only Q K^T(c) is ahead of K^T Delta(c) in the in-order pipe, and [W|U] fills the
// state-rebuild window two chunks ahead (the Delta warps take U(c+1) into registers right
// after forming Delta(c), which frees its accumulator early).
// Issue is by a converged warp with elect.sync (warp-uniform control flow keeps the
// descriptors in uniform registers; a one-lane issuer in a data-dependent loop issues
// several times slower).
//
// Warp roles (14 warps):
//   warp 0       TMA producer (no multicast), L2 prefetch ahead
//   warp 1       MMA issuer
//   warps 4-5    W: fp32 accumulator rows 0-63 -> bf16 A operand rows 0-63
//   warps 2-3    Q rows -> A operand rows 64-127; P~ rows 64-127 -> masked bf16 P; O
//                (X rows 64-127) -> global, X released as soon as O is in registers
//   warps 6-13   chain, two per lane quarter (32-column halves).  Quarters 0-1 form Delta
//                (U taken from its accumulator as soon as it lands); all eight rebuild the
//                bf16 S and S_T.
// A hand-off between roles is an mbarrier that counts warps: each warp of a role waits on
// its own (every lane polls, the warp votes) and arrives once after its own fences, so no
// hand-off passes a named barrier.
// Every wait is bounded (2 s); a wait that runs out sets a CTA-wide abort flag, every
// role winds down, and the caller's workspace records the timeout.
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
constexpr int kKvtStages = 3, kQStages = 2;

// ---- shared-memory map (bytes from a 1024-aligned base); tiles are 64 x 64 bf16, SW128
constexpr uint32_t TILE = 8192;
constexpr uint32_t Q_BYTES = 2 * TILE;                         // [Q a0 | Q a1]
// A stage holds K (two tiles), the V half and T; the gated flow adds T_U and the chunk's
// cumulative log-decay (64 fp32, log2 units).  Gated Delta has a second, decay-scaled copy.
template <bool G>
struct Lay {
    static constexpr uint32_t KVT_K = 0, KVT_V = 2 * TILE, KVT_T = 3 * TILE, KVT_TU = 4 * TILE, KVT_GL = 5 * TILE;
    static constexpr uint32_t KVT_BYTES = G ? 5 * TILE + 1024 : 4 * TILE;
    static constexpr uint32_t KVT_TX = G ? 5 * TILE + 256 : 4 * TILE;    // transaction bytes per stage
    static constexpr uint32_t OFF_KVT = 0;
    static constexpr uint32_t OFF_Q = OFF_KVT + kKvtStages * KVT_BYTES;
    static constexpr uint32_t OFF_DL = OFF_Q + kQStages * Q_BYTES;       // Delta, MN-major 64 x 64
    static constexpr uint32_t OFF_DL2 = G ? OFF_DL + TILE : OFF_DL;     // gated: Delta scaled by Gam_last / Gam_r
    static constexpr uint32_t OFF_SB = OFF_DL2 + TILE;                  // S bf16, MN-major 128 x 64
    static constexpr uint32_t OFF_BAR = OFF_SB + 2 * TILE;
    static constexpr uint32_t OFF_MISC = OFF_BAR + 32 * 8;
    static constexpr uint32_t SMEM_USED = OFF_MISC + 16;
    static constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;           // + alignment slack
    static_assert(SMEM_BYTES <= 232448, "shared-memory map exceeds 227 KB");
    // A [T; *] operand reads the 8 KiB after its T as (unused) rows 64-127: that stays inside
    // the map for every stage (the last stage is followed by the Q ring).
    static_assert(OFF_KVT + (kKvtStages - 1) * KVT_BYTES + (G ? KVT_TU : KVT_T) + 2 * TILE <= OFF_BAR,
                  "[T; *] reads past the map");
};
constexpr uint32_t NBAR = 32;

// ---- mbarriers (count 1 unless noted)
enum : int {
    B_KVT_FULL = 0,     // [3] TMA landed K, V, T of a stage
    B_KVT_FREE = 3,     // [3] the last MMA reading that stage is done
    B_Q_FULL = 6,       // [2] TMA landed Q of a stage
    B_Q_FREE = 8,       // [2] Q of that stage copied into tensor memory
    B_GP_FULL = 10,     // Q K^T landed
    B_GP_FREE,          // P~ read
    B_P_READY,          // P in the A operand
    B_WU_FULL,          // [W | U] landed
    B_WU_FREE,          // W and U both taken
    B_W_READY,          // W in the A operand
    B_Q_READY,          // Q in the A operand
    B_XS_FULL,          // [W;Q] S landed
    B_D_READY,          // Delta in shared memory
    B_S_FULL,           // K^T Delta landed
    B_SB_READY,         // bf16 S in shared memory
    B_O_FULL,           // P Delta landed (O complete)
    B_X_FREE,           // O stored
    B_DRAIN,
};

// arrivals per phase: one per arriving warp (W: warps 4-5; Q/P: warps 2-3; Delta: the four
// chain warps of quarters 0-1; S: all eight chain warps); TMA and MMA commits arrive once
__host__ __device__ constexpr uint32_t bar_count(int i) {
    return i == B_WU_FREE                                                   ? 6u
         : i == B_W_READY || i == B_Q_READY || i == B_GP_FREE || i == B_P_READY || i == B_X_FREE ||
                   i == B_Q_FREE || i == B_Q_FREE + 1                       ? 2u
         : i == B_D_READY                                                   ? 4u
         : i == B_SB_READY                                                  ? 8u
                                                                            : 1u;
}

// ---- TMEM columns
constexpr uint32_t TM_S = 0;          // fp32 S (d_k x 64)
constexpr uint32_t TM_X = 64;         // fp32 [W;Q] S, then + [*;P] Delta
constexpr uint32_t TM_WU = 128;       // fp32 [W | U] (192 columns)
constexpr uint32_t TM_GP = 320;       // fp32 [W;Q] K^T
constexpr uint32_t TM_AWQ = 384;      // bf16 A operand [W; Q]: 128 rows x 128 (64 columns)
constexpr uint32_t TM_AP = 448;       // bf16 A operand [*; P]: rows 64-127 x 64 (32 columns)
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t ID_N64 = idesc_bf16(128, 64, false, true);     // [W;Q] S, [*;P] Delta
constexpr uint32_t ID_WU = idesc_bf16(128, 192, false, true);     // [T;*] [K | V]
constexpr uint32_t ID_GP = idesc_bf16(128, 64, false, false);     // [W;Q] K^T
constexpr uint32_t ID_S = idesc_bf16(128, 64, true, true);        // K^T Delta
constexpr uint32_t ID_W = idesc_bf16(128, 128, false, true);      // gated: [T_W;*] K


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
    // already completed is seen by one inlined non-blocking probe; the sleeping, timed
    // part is one out-of-line copy, which keeps the role loops small in the
    // instruction cache.
    __device__ __forceinline__ bool wait(int i, uint32_t parity) const {
        if (mbar_test_wait(bar + i, parity)) return true;
        return wait_slow(i, parity);
    }
    __device__ __noinline__ bool wait_slow(int i, uint32_t parity) const {
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
    // whole-warp forms: every lane polls, the warp votes (warp-uniform control flow)
    __device__ __forceinline__ bool wwait(int i, uint32_t parity) const {
        return __all_sync(0xffffffffu, wait(i, parity));
    }
    // one arrival per warp once the whole warp got here (after its own fences)
    __device__ __forceinline__ void warp_arrive(int i, int lane) const {
        __syncwarp();
        if (lane == 0) mbar_arrive(bar + i);
    }
};

// nk k-steps of K = 16 with A and B in shared memory.  Operand k-step ks starts at
// base + (ks / 4) * atom + (ks % 4) * step (a K-major operand walks 32 bytes within a
// 64-column swizzle atom and jumps `atom` bytes between atoms; an MN-major operand walks
// 16 rows = 2048 bytes, atom = 8192).  A descriptor's start field is address / 16, so a
// k-step adds its byte offset / 16 (shared addresses stay below 256 KiB).
__device__ __forceinline__ void mma_ss(uint32_t d, uint32_t a, uint32_t a_atom, uint32_t a_step, uint32_t a_lbo,
                                       uint32_t b, uint32_t b_atom, uint32_t b_step, uint32_t b_lbo, uint32_t idesc,
                                       int nk, uint32_t acc) {
    const uint64_t da = sdesc_sw128(a, a_lbo, 1024), db = sdesc_sw128(b, b_lbo, 1024);
#pragma unroll
    for (int ks = 0; ks < nk; ++ks)
        mma_bf16_elect(d, da + (((ks >> 2) * a_atom + (ks & 3) * a_step) >> 4),
                       db + (((ks >> 2) * b_atom + (ks & 3) * b_step) >> 4), idesc, (acc | ks) != 0);
}
// nk k-steps with A in tensor memory (8 columns per k-step) and B in shared memory.
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint32_t b, uint32_t b_atom, uint32_t b_step,
                                       uint32_t b_lbo, uint32_t idesc, int nk, uint32_t acc) {
    const uint64_t db = sdesc_sw128(b, b_lbo, 1024);
#pragma unroll
    for (int ks = 0; ks < nk; ++ks)
        mma_bf16_ts_elect(d, a_tmem + 8 * ks, db + (((ks >> 2) * b_atom + (ks & 3) * b_step) >> 4), idesc,
                          (acc | ks) != 0);
}

// kSeg: the segmented scan's roles (G > 1) and the chunk states kept for the backward are
// compiled in; the plain forward runs the instantiation without them (a smaller kernel).
template <bool kGated, bool kSeg>
__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_t,
                const __grid_constant__ CUtensorMap tm_st,
                const float* __restrict__ S0, __nv_bfloat16* __restrict__ o, float* __restrict__ S_T,
                Seqs seqs, int Tdim, uint32_t* __restrict__ err, unsigned long long limit_ns,
                const float* __restrict__ gl_all, long ntiles, SegPlan seg, ChainSpans spans) {
    using L = Lay<kGated>;
    constexpr uint32_t KVT_K = L::KVT_K, KVT_V = L::KVT_V, KVT_T = L::KVT_T, KVT_BYTES = L::KVT_BYTES;
    constexpr uint32_t OFF_KVT = L::OFF_KVT, OFF_Q = L::OFF_Q, OFF_DL = L::OFF_DL, OFF_SB = L::OFF_SB;
    constexpr uint32_t OFF_BAR = L::OFF_BAR, OFF_MISC = L::OFF_MISC;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
    Ctl ctl{reinterpret_cast<uint64_t*>(sm + OFF_BAR), reinterpret_cast<volatile int*>(sm + OFF_MISC + 4), limit_ns};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3;                                                  // TMEM lane quarter
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    // This CTA's recurrence: a stream's 64-column half of d_v, or with a segmented scan one
    // segment of it (see SegPlan): its tokens, entering state, final state and outputs.
    long sidx;
    StreamJob jb;
    int col0;
    const float* s0p;             // entering state (128 x 128, row stride 128) or null (zero)
    bool s0_identity = false;     // transition product: the entering state is I
    float* stp;                   // final state (128 x 128) or null
    __nv_bfloat16* op = o;        // outputs [.., Tdim, 128]
    bool vzero = false;           // transition product: V = 0
    if (!kSeg || seg.G <= 1) {
        sidx = blockIdx.x >> 1;
        jb = seqs.job(sidx);
        col0 = (blockIdx.x & 1) * 64;
        s0p = S0 ? S0 + (size_t)sidx * kD * kD : nullptr;
        stp = S_T ? S_T + (size_t)sidx * kD * kD : nullptr;
    } else {
        const int per = 2 + 4 * (seg.G - 1);
        sidx = blockIdx.x / per;
        const int kk = (int)(blockIdx.x % per);
        const int g = kk < 2 ? 0 : 1 + (kk - 2) / 4;
        const int role = kk < 2 ? kk : (kk - 2) % 4;          // 0, 1: the state's halves; 2, 3: transition
        jb = seqs.job(sidx);
        const int first = g * seg.seg_chunks * 64;
        const int last = g == seg.G - 1 ? jb.len : min(jb.len, first + seg.seg_chunks * 64);
        jb.y0 += first;
        jb.len = max(0, last - first);
        jb.tile0 += (long)g * seg.seg_chunks;
        col0 = (role & 1) * 64;
        const size_t slot = ((size_t)sidx * seg.G + g) * kD * kD;
        if (role < 2) {
            s0p = g == 0 && S0 ? S0 + (size_t)sidx * kD * kD : nullptr;
            stp = seg.Sloc + slot;
        } else {
            s0p = nullptr;
            s0_identity = true;
            stp = seg.Phi + slot;
            op = seg.R;
            vzero = true;
        }
    }
    const int T = jb.len, zc = jb.z, y0 = jb.y0;
    const int nchunks = (T + 63) / 64;
    const size_t tok0 = (size_t)zc * Tdim + y0;
    // the extents this CTA's pointers must stay inside (checked builds)
    const Span op_span = op == o ? spans.o : spans.r;
    const bool st_in_phi = seg.Phi && stp >= seg.Phi && stp < seg.Phi + spans.phi.bytes / sizeof(float);
    const Span st_span = (!kSeg || seg.G <= 1) ? spans.st : (st_in_phi ? spans.phi : spans.sloc);
    const Span s0_span = spans.s0;
    if (nchunks == 0) {   // an empty sequence: the state passes through (nothing else runs)
        if (stp) {
            for (int e = tid; e < kD * 64; e += kThreads) {
                const int i = e >> 6, j = e & 63;
                const size_t at = (size_t)i * kD + col0 + j;
                float x = s0_identity ? (i == col0 + j ? 1.f : 0.f) : 0.f;
                if (!s0_identity && s0p && span_ok(err, s0_span, s0p + at, 4)) x = s0p[at];
                if (span_ok(err, st_span, stp + at, 4)) stp[at] = x;
            }
        }
        return;
    }
    if (vzero) {   // the transition product's V tiles stay zero (never loaded)
        for (int e = tid; e < kKvtStages * (int)(TILE / 16); e += kThreads) {
            const int stg = e / (int)(TILE / 16), off = e % (int)(TILE / 16);
            reinterpret_cast<uint4*>(sm + OFF_KVT + stg * KVT_BYTES + KVT_V)[off] = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
    }

    if (tid == 0) {
        for (int i = 0; i < (int)NBAR; ++i) mbar_init(ctl.bar + i, bar_count(i));
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
    auto qst = [&](int c) { return OFF_Q + (uint32_t)(c % kQStages) * Q_BYTES; };

    if (warp == 0) {
        // ================================================================ TMA producer
        if (lane == 0) {
            bool ok = true;
            int kvt_issued = 0, q_issued = 0;
            for (int c = 0; c < nchunks && ok; ++c) {
                const int t0 = c * 64;
                {   // K, V, T of chunk c
                    const int s = c % kKvtStages;
                    if (c >= kKvtStages && !(ok = ctl.wait(B_KVT_FREE + s, ((c - kKvtStages) / kKvtStages) & 1))) break;
                    uint8_t* st = sm + kvt(c);
                    uint64_t* full = ctl.b(B_KVT_FULL + s);
                    mbar_arrive_expect_tx(full, L::KVT_TX - (vzero ? TILE : 0));
                    tma_load_3d(st + KVT_K, &tm_k, full, 0, y0 + t0, zc);
                    tma_load_3d(st + KVT_K + TILE, &tm_k, full, 64, y0 + t0, zc);
                    if (!vzero) tma_load_3d(st + KVT_V, &tm_v, full, col0, y0 + t0, zc);
                    if (EFLA_CHECKED && (jb.tile0 + c + 1) * 64 > spans.t_rows) atomicOr(err, kDevBounds);
                    tma_load_2d(st + KVT_T, &tm_t, full, 0, (int)((jb.tile0 + c) * 64));
                    if constexpr (kGated) {
                        tma_load_2d(st + L::KVT_TU, &tm_t, full, 0, (int)((ntiles + jb.tile0 + c) * 64));
                        const float* src = gl_all + (jb.tile0 + c) * 64;
                        if (!span_ok(err, spans.gl, src, 256)) src = gl_all;   // keep the transaction count
                        bulk_load(st + L::KVT_GL, src, 256, full);
                    }
                    kvt_issued = c + 1;
                }
                {   // Q of chunk c
                    const int s = c % kQStages;
                    if (c >= kQStages && !(ok = ctl.wait(B_Q_FREE + s, ((c - kQStages) / kQStages) & 1))) break;
                    uint8_t* st = sm + qst(c);
                    uint64_t* full = ctl.b(B_Q_FULL + s);
                    mbar_arrive_expect_tx(full, 2 * TILE);
                    tma_load_3d(st, &tm_q, full, 0, y0 + t0, zc);
                    tma_load_3d(st + TILE, &tm_q, full, 64, y0 + t0, zc);
                    q_issued = c + 1;
                }
                if (c + 3 < nchunks) {      // warm L2 for the chunk three ahead
                    const int t3 = y0 + t0 + 192;
                    tma_prefetch_l2_3d(&tm_k, 0, t3, zc);
                    tma_prefetch_l2_3d(&tm_k, 64, t3, zc);
                    if (!vzero) tma_prefetch_l2_3d(&tm_v, col0, t3, zc);
                    tma_prefetch_l2_3d(&tm_q, 0, t3, zc);
                    tma_prefetch_l2_3d(&tm_q, 64, t3, zc);
                    tma_prefetch_l2_2d(&tm_t, 0, (int)((jb.tile0 + c + 3) * 64));
                }
            }
            // no copy may land after exit
            for (int c = max(0, kvt_issued - kKvtStages); c < kvt_issued; ++c)
                mbar_wait(ctl.b(B_KVT_FULL + c % kKvtStages), (c / kKvtStages) & 1, limit_ns);
            for (int c = max(0, q_issued - kQStages); c < q_issued; ++c)
                mbar_wait(ctl.b(B_Q_FULL + c % kQStages), (c / kQStages) & 1, limit_ns);
        }
    } else if (warp == 1) {
        // ================================================================ MMA issuer (whole warp)
        // Warp-uniform control flow: every lane polls the barrier and the warp votes;
        // elect.sync inside each MMA and commit picks the issuing lane.
        auto wait = [&](int i, uint32_t parity) { return __all_sync(0xffffffffu, ctl.wait(i, parity)); };
        auto issue_qk = [&](int c, int k0, int k1) {      // [W;Q] K^T, k-steps [k0, k1): rows 64-127 are Q K^T
            tc_fence_after();
            const uint64_t db = sdesc_sw128(sb + kvt(c) + KVT_K, 16, 1024);
            for (int ks = k0; ks < k1; ++ks)
                mma_bf16_ts_elect(tmem + TM_GP, tmem + TM_AWQ + 8 * ks, db + (((ks >> 2) * TILE + (ks & 3) * 32) >> 4),
                                  ID_GP, ks > 0);
            if (k1 == 8) {
                mma_commit_elect(ctl.b(B_GP_FULL));
            }
        };
        auto issue_wu = [&](int c) {      // [W | U] = [T; *] [K | V]   (gated: [T_W;*] K | [T_U;*] V)
            tc_fence_after();
            const uint32_t st = sb + kvt(c);
            if constexpr (kGated) {
                mma_ss(tmem + TM_WU, st + KVT_T, TILE, 32, 16, st + KVT_K, 4 * 2048, 2048, TILE, ID_W, 4, 0);
                mma_ss(tmem + TM_WU + 128, st + L::KVT_TU, TILE, 32, 16, st + KVT_V, 4 * 2048, 2048, TILE, ID_N64, 4, 0);
            } else {
                mma_ss(tmem + TM_WU, st + KVT_T, TILE, 32, 16, st + KVT_K, 4 * 2048, 2048, TILE, ID_WU, 4, 0);
            }
            mma_commit_elect(ctl.b(B_WU_FULL));
        };
        bool ok = wait(B_KVT_FULL, 0);
        if (ok) issue_wu(0);
        if (ok && nchunks > 1) {
            ok = wait(B_KVT_FULL + 1, 0) && wait(B_WU_FREE, 0);
            if (ok) issue_wu(1);
        }
        for (int c = 0; c < nchunks && ok; ++c) {
            // X = [W; Q] S (state chain)
            if (!(ok = wait(B_W_READY, c & 1) && wait(B_Q_READY, c & 1) && wait(B_SB_READY, c & 1) &&
                       (c == 0 || wait(B_X_FREE, (c - 1) & 1))))
                break;
            tc_fence_after();
            mma_ts(tmem + TM_X, tmem + TM_AWQ, sb + OFF_SB, 4 * 2048, 2048, TILE, ID_N64, 8, 0);
            mma_commit_elect(ctl.b(B_XS_FULL));
            if (kSeg && seg.states && lane == 0) {   // chunk c's entering state, for the backward: one TMA store
                const long srow = (jb.tile0 + c) * kD;
                if (span_ok(err, spans.states, seg.states + (srow + kD) * kD - 1, 2))
                    tma_store_2d(&tm_st, sm + OFF_SB, col0, (int)srow);
            }
            __syncwarp();
            // this chunk's Q K^T (its Q has been in place since the last chunk) runs while
            // Delta is formed
            if (!(ok = c == 0 || wait(B_GP_FREE, (c - 1) & 1))) break;
            issue_qk(c, 0, 8);
            // S += K^T Delta (state chain)
            if (!(ok = wait(B_D_READY, c & 1))) break;
            if (kSeg && seg.states && lane == 0) tma_store_wait_read();   // the bf16 S is rewritten after this product
            __syncwarp();
            tc_fence_after();
            mma_ss(tmem + TM_S, sb + kvt(c) + KVT_K, 4 * 2048, 2048, TILE, sb + L::OFF_DL2, 4 * 2048, 2048, TILE,
                   ID_S, 4, 1);
            mma_commit_elect(ctl.b(B_S_FULL));
            // gated: the P warps still read the stage's log-decays until P is ready
            if constexpr (!kGated) mma_commit_elect(ctl.b(B_KVT_FREE + c % kKvtStages));
            // X += [*; P] Delta: rows 64-127 become O = Q S + P Delta
            if (!(ok = wait(B_P_READY, c & 1))) break;
            tc_fence_after();
            mma_ts(tmem + TM_X, tmem + TM_AP, sb + OFF_DL, 4 * 2048, 2048, TILE, ID_N64, 4, 1);
            mma_commit_elect(ctl.b(B_O_FULL));
            if constexpr (kGated) mma_commit_elect(ctl.b(B_KVT_FREE + c % kKvtStages));
            if (c + 2 < nchunks) {   // [W|U] two chunks ahead, in this chunk's state-rebuild window
                if (!(ok = wait(B_KVT_FULL + (c + 2) % kKvtStages, ((c + 2) / kKvtStages) & 1) &&
                           wait(B_WU_FREE, (c + 1) & 1))) break;
                issue_wu(c + 2);
            }
        }
        mma_commit_elect(ctl.b(B_DRAIN));
        if (lane == 0) {
            mbar_wait(ctl.b(B_DRAIN), 0, limit_ns);
            if (kSeg && seg.states) tma_store_wait_all();
        }
        __syncwarp();
    } else if (warp == 4 || warp == 5) {
        // ================================================================ W -> A operand (quarters 0-1)
        bool ok = true;
        for (int c = 0; c < nchunks && ok; ++c) {
            // [W | U](c) landed, and [W;Q] S(c-1) no longer reads the A operand
            ok = ctl.wwait(B_WU_FULL, c & 1) && (c == 0 || ctl.wwait(B_XS_FULL, (c - 1) & 1));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float w[64];
                uint32_t pk[32];
                tmem_ld64_wait(tmem + lane_off + TM_WU + 64 * h, w);
#pragma unroll
                for (int j = 0; j < 32; ++j) pk[j] = pack_bf16x2(w[2 * j], w[2 * j + 1]);
                tmem_st32(tmem + lane_off + TM_AWQ + 32 * h, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            ctl.warp_arrive(B_WU_FREE, lane);
            ctl.warp_arrive(B_W_READY, lane);
        }
    } else if (warp < 4) {
        // ================================================================ Q and P -> A operands (quarters 2-3)
        const int r = 32 * (q - 2) + lane;            // chunk row of this lane (TMEM lane 64 + r)
        auto copy_q = [&](int c) {                    // Q row r (SW128 tile, two atoms) -> A rows 64-127
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t pk[32];
                const uint8_t* src = sm + qst(c) + h * TILE;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint4 x = *reinterpret_cast<const uint4*>(src + sw128_off(r, j));
                    pk[4 * j] = x.x; pk[4 * j + 1] = x.y; pk[4 * j + 2] = x.z; pk[4 * j + 3] = x.w;
                }
                tmem_st32(tmem + lane_off + TM_AWQ + 32 * h, pk);
            }
            ctl.warp_arrive(B_Q_FREE + c % kQStages, lane);
            tmem_wait_st();
            tc_fence_before();
            ctl.warp_arrive(B_Q_READY, lane);
        };
        // O(c) = X rows 64-127 once P Delta(c) has landed: taken into registers, X released
        // at once for [W;Q] S(c+1), then stored to global as bf16 (rows past T skipped)
        auto store_o = [&](int c) {
            if (!ctl.wwait(B_O_FULL, c & 1)) return false;
            tc_fence_after();
            float t[64];
            tmem_ld64_wait(tmem + lane_off + TM_X, t);
            tc_fence_before();
            ctl.warp_arrive(B_X_FREE, lane);
            const int t0 = c * 64;
            if (op && r < min(64, T - t0) && span_ok(err, op_span, op + (tok0 + t0 + r) * kD + col0, 128)) {
                uint4* dst = reinterpret_cast<uint4*>(op + (tok0 + t0 + r) * kD + col0);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint4 y;
                    y.x = pack_bf16x2(t[8 * j], t[8 * j + 1]);
                    y.y = pack_bf16x2(t[8 * j + 2], t[8 * j + 3]);
                    y.z = pack_bf16x2(t[8 * j + 4], t[8 * j + 5]);
                    y.w = pack_bf16x2(t[8 * j + 6], t[8 * j + 7]);
                    dst[j] = y;
                }
            }
            return true;
        };
        if (q == 2) {       // bf16 P columns 32-63 of chunk rows 0-31: zero for good
            const float z[16] = {};
            tmem_st16(tmem + lane_off + TM_AP + 16, z);
            tmem_wait_st();
            tc_fence_before();
        }
        bool ok = ctl.wwait(B_Q_FULL, 0);
        if (ok) copy_q(0);
        for (int c = 0; c < nchunks && ok; ++c) {
            if (c > 0 && !(ok = store_o(c - 1))) break;
            // P = Q K^T masked causally (diagonal kept) -> A rows 64-127 (P Delta(c-1) is done).
            // Chunk rows 0-31 have no entry past column 31 (those bf16 columns were zeroed
            // once, above); rows 32-63 keep columns 0-31 whole.  Each warp masks 32 columns.
            if (!(ok = ctl.wwait(B_GP_FULL, c & 1))) break;
            tc_fence_after();
            if constexpr (kGated) {
                // P~[r][s] = (Q K^T)[r][s] Gam_r / Gam_s (s <= r), and the Q S rows of X scaled by
                // Gam_r before P Delta accumulates onto them: O = diag(Gam) Q S + P~ Delta
                const float* glc = reinterpret_cast<const float*>(sm + kvt(c) + L::KVT_GL);
                const float glr = glc[r];
                if (q == 2) {
                    float t[32], pk[16];
                    tmem_ld32_wait(tmem + lane_off + TM_GP, t);
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        pk[j] = __uint_as_float(pack_bf16x2(2 * j <= lane ? t[2 * j] * exp2f(glr - glc[2 * j]) : 0.f,
                                                            2 * j + 1 <= lane ? t[2 * j + 1] * exp2f(glr - glc[2 * j + 1]) : 0.f));
                    tmem_st16(tmem + lane_off + TM_AP, pk);
                } else {
                    float t[64];
                    uint32_t pk[32];
                    tmem_ld64_wait(tmem + lane_off + TM_GP, t);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        pk[j] = pack_bf16x2(t[2 * j] * exp2f(glr - glc[2 * j]), t[2 * j + 1] * exp2f(glr - glc[2 * j + 1]));
                        pk[16 + j] = pack_bf16x2(2 * j <= lane ? t[32 + 2 * j] * exp2f(glr - glc[32 + 2 * j]) : 0.f,
                                                 2 * j + 1 <= lane ? t[33 + 2 * j] * exp2f(glr - glc[33 + 2 * j]) : 0.f);
                    }
                    tmem_st32(tmem + lane_off + TM_AP, pk);
                }
                {
                    const float gm = exp2f(glr);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float x[32];
                        tmem_ld32_wait(tmem + lane_off + TM_X + 32 * h, x);
                        float y0[16], y1[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            y0[j] = x[j] * gm;
                            y1[j] = x[16 + j] * gm;
                        }
                        tmem_st16(tmem + lane_off + TM_X + 32 * h, y0);
                        tmem_st16(tmem + lane_off + TM_X + 32 * h + 16, y1);
                    }
                }
            } else if (q == 2) {
                float t[32], pk[16];
                tmem_ld32_wait(tmem + lane_off + TM_GP, t);
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    pk[j] = __uint_as_float(
                        pack_bf16x2(2 * j <= lane ? t[2 * j] : 0.f, 2 * j + 1 <= lane ? t[2 * j + 1] : 0.f));
                tmem_st16(tmem + lane_off + TM_AP, pk);
            } else {
                float t[64];
                uint32_t pk[32];
                tmem_ld64_wait(tmem + lane_off + TM_GP, t);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    pk[j] = pack_bf16x2(t[2 * j], t[2 * j + 1]);
                    pk[16 + j] = pack_bf16x2(2 * j <= lane ? t[32 + 2 * j] : 0.f, 2 * j + 1 <= lane ? t[33 + 2 * j] : 0.f);
                }
                tmem_st32(tmem + lane_off + TM_AP, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            ctl.warp_arrive(B_GP_FREE, lane);
            ctl.warp_arrive(B_P_READY, lane);
            // Q(c+1) -> A rows 64-127, once [W;Q] S(c) no longer reads them
            if (c + 1 < nchunks) {
                ok = ctl.wwait(B_Q_FULL + (c + 1) % kQStages, ((c + 1) / kQStages) & 1) && ctl.wwait(B_XS_FULL, c & 1);
                if (!ok) break;
                copy_q(c + 1);
            }
        }
        if (ok) store_o(nchunks - 1);
    } else {
        // ================================================================ chain (two warps per lane quarter)
        // Quarters 0-1 (X rows 0-63, W S) form Delta; all eight rebuild the bf16 S.  Each warp
        // waits and arrives on its own (the barriers count warps): no group barrier in a
        // hand-off.
        const int ch = (warp - 6) >> 2;               // column half: 32 of this CTA's 64 columns
        const int cc = 32 * ch;
        const int ct = 32 * q + lane;                 // d_k row of S, and row of X / [W | U]
        const bool delta_group = q < 2;
        // gated: the accumulator carries Gam_last(c) S_c into the write of chunk c
        auto decay_of = [&](int c) -> float {
            if constexpr (kGated) {
                if (!ctl.wwait(B_KVT_FULL + c % kKvtStages, (c / kKvtStages) & 1)) return 1.f;
                return exp2f(reinterpret_cast<const float*>(sm + kvt(c) + L::KVT_GL)[63]);
            }
            return 1.f;
        };
        {   // initial state
            const float* src = s0p ? s0p + (size_t)ct * kD + col0 + cc : nullptr;
            const float dec0 = decay_of(0);
#pragma unroll
            for (int qd = 0; qd < 2; ++qd) {
                float s16[16];
#pragma unroll
                for (int j = 0; j < 16; j += 4) {
                    float4 x = src && span_ok(err, s0_span, src + 16 * qd + j, 16)
                                   ? *reinterpret_cast<const float4*>(src + 16 * qd + j) : make_float4(0.f, 0.f, 0.f, 0.f);
                    if (s0_identity) {
                        const int c0 = col0 + cc + 16 * qd + j;    // this row's 1 sits in column ct
                        x = make_float4(ct == c0 ? 1.f : 0.f, ct == c0 + 1 ? 1.f : 0.f, ct == c0 + 2 ? 1.f : 0.f,
                                        ct == c0 + 3 ? 1.f : 0.f);
                    }
                    s16[j] = x.x; s16[j + 1] = x.y; s16[j + 2] = x.z; s16[j + 3] = x.w;
                }
                if (smem_ok(err, OFF_SB + sw128_off(ct, 4 * ch + 2 * qd + 1), 16, OFF_SB + 2 * TILE)) {
                    st_chunk(sm + OFF_SB + sw128_off(ct, 4 * ch + 2 * qd), s16);
                    st_chunk(sm + OFF_SB + sw128_off(ct, 4 * ch + 2 * qd + 1), s16 + 8);
                }
                if constexpr (kGated) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) s16[j] *= dec0;
                }
                tmem_st16(tmem + lane_off + TM_S + cc + 16 * qd, s16);
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            ctl.warp_arrive(B_SB_READY, lane);
        }
        bool ok = true;
        float u[32];
        auto take_u = [&](int cu) {
            if (!ctl.wwait(B_WU_FULL, cu & 1)) return false;
            tc_fence_after();
            tmem_ld32_wait(tmem + lane_off + TM_WU + 128 + cc, u);
            tc_fence_before();
            ctl.warp_arrive(B_WU_FREE, lane);
            return true;
        };
        if (delta_group) ok = take_u(0);
        for (int c = 0; c < nchunks && ok; ++c) {
            if (delta_group) {
                // Delta = U - W S (X rows 0-63)
                if (!(ok = ctl.wwait(B_XS_FULL, c & 1))) break;
                tc_fence_after();
                float t[32];
                tmem_ld32_wait(tmem + lane_off + TM_X + cc, t);
#pragma unroll
                for (int j = 0; j < 32; ++j) t[j] = u[j] - t[j];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (smem_ok(err, OFF_DL + sw128_off(ct, 4 * ch + j), 16, OFF_DL + TILE))
                        st_chunk(sm + OFF_DL + sw128_off(ct, 4 * ch + j), t + 8 * j);
                if constexpr (kGated) {   // the state's copy: row r scaled by Gam_last / Gam_r
                    const float* glc = reinterpret_cast<const float*>(sm + kvt(c) + L::KVT_GL);
                    const float sc = exp2f(glc[63] - glc[ct]);
#pragma unroll
                    for (int j = 0; j < 32; ++j) t[j] *= sc;
#pragma unroll
                    for (int j = 0; j < 4; ++j) st_chunk(sm + L::OFF_DL2 + sw128_off(ct, 4 * ch + j), t + 8 * j);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                ctl.warp_arrive(B_D_READY, lane);
                if (c + 1 < nchunks && !(ok = take_u(c + 1))) break;   // U(c+1) before [W|U](c+2)
            }
            // the new state: bf16 operand for the next chunk (and S_T after the last)
            if (!(ok = ctl.wwait(B_S_FULL, c & 1))) break;
            tc_fence_after();
            {
                float t[32];
                tmem_ld32_wait(tmem + lane_off + TM_S + cc, t);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (smem_ok(err, OFF_SB + sw128_off(ct, 4 * ch + j), 16, OFF_SB + 2 * TILE))
                        st_chunk(sm + OFF_SB + sw128_off(ct, 4 * ch + j), t + 8 * j);
                if (c == nchunks - 1 && stp && span_ok(err, st_span, stp + (size_t)ct * kD + col0 + cc, 128)) {
                    float* dst = stp + (size_t)ct * kD + col0 + cc;
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4*>(dst + j) = make_float4(t[j], t[j + 1], t[j + 2], t[j + 3]);
                }
                if constexpr (kGated) {
                    if (c + 1 < nchunks) {
                        const float dec = decay_of(c + 1);
                        float y0[16], y1[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            y0[j] = t[j] * dec;
                            y1[j] = t[16 + j] * dec;
                        }
                        tmem_st16(tmem + lane_off + TM_S + cc, y0);
                        tmem_st16(tmem + lane_off + TM_S + cc + 16, y1);
                        tmem_wait_st();
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            ctl.warp_arrive(B_SB_READY, lane);
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *ctl.abort) atomicOr(err, kDevTimeout);
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
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

size_t chunk_tc_gated_workspace_bytes(long BH, int T) {
    const long ntiles = BH * ((T + 63) / 64);
    return (size_t)ntiles * (2 * 64 * 64 * 2 + 64 * 4);   // T_W, T_U (bf16) and G log2(e) (fp32) per tile
}

cudaError_t launch_chunk_tc(const void* q, const void* k, const void* v, const void* beta, const float* S0,
                            void* o, float* S_T, const Seqs& seqs, long nstreams, long Z, int Tdim, long ntiles,
                            uint32_t* err, void* scratch, int rule, cudaStream_t stream, const float* g,
                            const SegPlan& seg) {
    cudaError_t e = launch_ut(k, beta, scratch, seqs, Z, Tdim, ntiles, err, kWaitLimitNs, rule, stream, g, seg.X);
    if (e != cudaSuccess) return e;
    const long ctas = seg.G > 1 ? nstreams * (2 + 4 * (seg.G - 1)) : nstreams * 2;
    ChainSpans sp;
    const size_t obytes = (size_t)Z * Tdim * kD * 2, sbytes = (size_t)nstreams * kD * kD * 4;
    sp.o = Span{o, obytes};
    sp.r = Span{seg.R, obytes};
    sp.s0 = Span{S0, sbytes};
    sp.st = Span{S_T, sbytes};
    sp.sloc = Span{seg.Sloc, sbytes * std::max(1, seg.G)};
    sp.phi = Span{seg.Phi, sbytes * std::max(1, seg.G)};
    sp.states = Span{seg.states, (size_t)ntiles * kD * kD * 2};
    sp.gl = Span{g ? static_cast<const char*>(scratch) + ntiles * 8192 * 2 : nullptr, (size_t)ntiles * 256};
    sp.t_rows = (g ? 2 : 1) * ntiles * 64;
    CUtensorMap mq, mk, mv, mt, mst;
    if (!tma_map_tokens(&mq, q, kD, Tdim, Z) || !tma_map_tokens(&mk, k, kD, Tdim, Z) ||
        !tma_map_tokens(&mv, v, kD, Tdim, Z) || !tma_map_rows64(&mt, scratch, std::max<long>(1, (g ? 2 : 1) * ntiles) * 64) ||
        !(seg.states ? tma_map_rows128(&mst, seg.states, std::max<long>(1, ntiles) * kD) : (mst = mt, true)))
        return cudaErrorInvalidValue;
    const float* gl = g ? reinterpret_cast<const float*>(static_cast<const char*>(scratch) + ntiles * 8192 * 2)
                        : nullptr;
    const bool full = seg.G > 1 || seg.states;
    if (g) {
        static std::atomic<uint64_t> smem_set_g{0}, smem_set_gs{0};
        e = full ? set_smem_limit_once(chunk_tc_kernel<true, true>, (int)Lay<true>::SMEM_BYTES, smem_set_gs)
                 : set_smem_limit_once(chunk_tc_kernel<true, false>, (int)Lay<true>::SMEM_BYTES, smem_set_g);
        if (e != cudaSuccess) return e;
        if (full)
            chunk_tc_kernel<true, true><<<(unsigned)ctas, kThreads, Lay<true>::SMEM_BYTES, stream>>>(
                mq, mk, mv, mt, mst, S0, (__nv_bfloat16*)o, S_T, seqs, Tdim, err, kWaitLimitNs, gl, ntiles, seg, sp);
        else
            chunk_tc_kernel<true, false><<<(unsigned)ctas, kThreads, Lay<true>::SMEM_BYTES, stream>>>(
                mq, mk, mv, mt, mst, S0, (__nv_bfloat16*)o, S_T, seqs, Tdim, err, kWaitLimitNs, gl, ntiles, seg, sp);
        return cudaGetLastError();
    }
    static std::atomic<uint64_t> smem_set{0}, smem_set_s{0};
    e = full ? set_smem_limit_once(chunk_tc_kernel<false, true>, (int)Lay<false>::SMEM_BYTES, smem_set_s)
             : set_smem_limit_once(chunk_tc_kernel<false, false>, (int)Lay<false>::SMEM_BYTES, smem_set);
    if (e != cudaSuccess) return e;
    if (full)
        chunk_tc_kernel<false, true><<<(unsigned)ctas, kThreads, Lay<false>::SMEM_BYTES, stream>>>(
            mq, mk, mv, mt, mst, S0, (__nv_bfloat16*)o, S_T, seqs, Tdim, err, kWaitLimitNs, nullptr, ntiles, seg, sp);
    else
        chunk_tc_kernel<false, false><<<(unsigned)ctas, kThreads, Lay<false>::SMEM_BYTES, stream>>>(
            mq, mk, mv, mt, mst, S0, (__nv_bfloat16*)o, S_T, seqs, Tdim, err, kWaitLimitNs, nullptr, ntiles, seg, sp);
    return cudaGetLastError();
}

cudaError_t launch_wait_timeout_selftest(uint32_t* err, unsigned long long limit_ns, cudaStream_t stream) {
    wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(err, limit_ns);
    return cudaGetLastError();
}

}  // namespace efla
