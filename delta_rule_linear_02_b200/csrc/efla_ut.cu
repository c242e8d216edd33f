// efla_ut.cu -- the UT transform of every 64-token chunk of every stream (bf16, d_k = 128).
//
// Exact Flow Linear Attention, Section 3.3: inside a chunk the rank-1 writes satisfy
// (I + A) Delta = diag(alpha) (V - K S) with A = strictly-lower(diag(alpha) K K^T), so
// Delta = T (V - K S) with T = (I + A)^{-1} diag(alpha).  T depends on K and beta only,
// not on the state, so it is computed here for all chunks at once, in parallel, and the
// chain kernel (efla_chunk_tc.cu) reads it back as a bf16 operand.
//
// Per tile (stream bh, chunk c):
//   G = K K^T                                   tcgen05 MMA, M = 64 (bf16 in, fp32 in TMEM;
//                                                row r in lane (r % 16) + 32 (r / 16))
//   lambda_r = G_rr, alpha_r = gate(beta_r, lambda_r)   (Section 3.2 / 3.4; beta_r itself
//                                                under the Euler rule, Section 2)
//   A^T rows = alpha (.) G rows                 (G is symmetric)
//   X = (I + A)^{-1}                            efla_ut_tf32.cuh (fp32 + TF32 merges)
//   T = X diag(alpha) -> bf16, row-major 64 x 64, at Tout + 4096 * (bh * nchunks + c)
// Tokens past T are zero-filled by TMA (k = 0, beta = 0: alpha = 0, their rows and
// columns of T are zero).
//
// Gated flow (Section 3.4, Gated EFLA; per-token log-decay g): with the cumulative
// log-decay G_r = g_0 + ... + g_r of the tile and Gam_r = e^{G_r},
//   A[r][s] = alpha_r (Gam_r / Gam_s) G[r][s]  (s < r),  X = (I + A)^{-1},
// and two transforms are stored, T_W = X diag(alpha Gam) (at Tout, as above) and
// T_U = X diag(abar) (ntiles tiles further on), plus G_r log2(e) of every row (fp32, 64 per
// tile, after both transform regions) for the chain kernel's decay factors.
//
// A persistent grid of six CTAs per SM walks the tiles; the CTAs on an SM overlap each
// other's latency.  The K tile is dead once G has been formed, so A^T is written over it:
// a CTA holds one fp32 64 x 68 tile for K / A^T and one for X (36 KB), and the next K tile
// is loaded while the T of the current one is stored.  Warp 0 (whole-warp control flow,
// elect.sync) issues the TMA copies and the MMA; warps 1-4 compute the gate, the solve and
// the bf16 store.  Every wait is bounded.
#include "efla_common.cuh"
#include "efla_kernels.h"
#include "efla_tma.cuh"
#include "efla_ut_tf32.cuh"
#include "sm100.cuh"

namespace efla {

namespace {
using namespace sm100;
using ut::LDX;

constexpr int kThreads = 160;
constexpr int kCtasPerSm = 6;
constexpr uint32_t TILE = 8192;
constexpr uint32_t F32_TILE = 64 * LDX * 4;            // 17,408 bytes (a multiple of 1024)
constexpr uint32_t OFF_K = 0;                          // [K a0 | K a1], then A^T over it
constexpr uint32_t OFF_AT = OFF_K;
constexpr uint32_t OFF_X = OFF_AT + F32_TILE;
static_assert(2 * TILE <= F32_TILE && F32_TILE % 1024 == 0, "K / A^T region");
constexpr uint32_t OFF_ALPHA = OFF_X + F32_TILE;
constexpr uint32_t OFF_BETA = OFF_ALPHA + 256;
constexpr uint32_t OFF_BAR = OFF_BETA + 256;
constexpr uint32_t NBAR = 8;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
constexpr uint32_t SMEM_USED = OFF_MISC + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;
static_assert(kCtasPerSm * SMEM_BYTES <= 232448, "UT kernel: shared memory for the target occupancy");
// gated flow only: raw log-decay, its cumulative sum (log2 units), abar, alpha * Gam
constexpr uint32_t OFF_GRAW = SMEM_USED;
constexpr uint32_t OFF_GL = OFF_GRAW + 256;
constexpr uint32_t OFF_ABAR = OFF_GL + 256;
constexpr uint32_t OFF_MW = OFF_ABAR + 256;
constexpr uint32_t SMEM_BYTES_G = OFF_MW + 256 + 1024;
static_assert(kCtasPerSm * (SMEM_BYTES_G + 1024) <= 233472, "gated UT kernel: shared memory per SM");

enum : int { B_FULL = 0, B_GP_FULL = 1, B_GP_FREE = 2, B_AT_FREE = 3, B_DRAIN = 4 };
constexpr uint32_t TM_COLS = 64;
constexpr uint32_t ID_G = idesc_bf16(64, 64, false, false);
constexpr int NB_W = 1;                                // named barrier of the 128 worker threads

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort,
                                             unsigned long long limit) {
    if (mbar_try_wait_sleep(bar, parity, 20000)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_sleep(bar, parity, 20000)) {
        if (*abort) return false;
        if (globaltimer_ns() - t0 > limit) {
            *abort = 1;
            return false;
        }
    }
    return true;
}

template <bool kGated>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
ut_kernel(const __grid_constant__ CUtensorMap tm_k, const __nv_bfloat16* __restrict__ beta,
          __nv_bfloat16* __restrict__ Tout, Seqs seqs, int Tdim, long ntiles, uint32_t* __restrict__ err,
          unsigned long long limit_ns, int rule, const float* __restrict__ gdec, Span t_span, Span b_span,
          Span g_span, float* __restrict__ Xout, Span x_span) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    float* At = reinterpret_cast<float*>(sm + OFF_AT);
    float* X = reinterpret_cast<float*>(sm + OFF_X);
    float* al = reinterpret_cast<float*>(sm + OFF_ALPHA);
    float* bt = reinterpret_cast<float*>(sm + OFF_BETA);
    float* graw = reinterpret_cast<float*>(sm + OFF_GRAW);    // gated flow only
    float* gl = reinterpret_cast<float*>(sm + OFF_GL);
    float* abar = reinterpret_cast<float*>(sm + OFF_ABAR);
    float* mw = reinterpret_cast<float*>(sm + OFF_MW);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
    volatile int* abort = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long first = blockIdx.x, step = gridDim.x;
    const int ntile = first < ntiles ? (int)((ntiles - first + step - 1) / step) : 0;

    if (tid == 0) {
        for (int i = 0; i < (int)NBAR; ++i) mbar_init(bar + i, 1);
        *abort = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_k);
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
        // ------------------------------------------------------------ TMA + MMA issue (whole warp)
        // Warp-uniform control flow (every lane polls, the warp votes); lane 0 issues the
        // TMA copies, elect.sync the MMAs and commits.
        auto wait = [&](uint64_t* b, uint32_t parity) {
            return __all_sync(0xffffffffu, wait_bounded(b, parity, abort, limit_ns));
        };
        auto load = [&](int j) {
            if (lane == 0) {
                const long tile = first + (long)j * step;
                int c;
                const StreamJob jb = seqs.tile(tile, &c);
                mbar_arrive_expect_tx(bar + B_FULL, 2 * TILE);
                tma_load_3d(sm + OFF_K, &tm_k, bar + B_FULL, 0, jb.y0 + c * 64, jb.z);
                tma_load_3d(sm + OFF_K + TILE, &tm_k, bar + B_FULL, 64, jb.y0 + c * 64, jb.z);
            }
            __syncwarp();
        };
        if (ntile > 0) load(0);
        bool ok = true;
        for (int j = 0; j < ntile && ok; ++j) {
            ok = wait(bar + B_FULL, j & 1) && (j == 0 || wait(bar + B_GP_FREE, (j - 1) & 1));
            if (!ok) break;
            tc_fence_after();
            const uint64_t d0 = sdesc_sw128(sb + OFF_K, 16, 1024);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t d = d0 + (((ks >> 2) * TILE + (ks & 3) * 32) >> 4);
                mma_bf16_elect(tmem, d, d, ID_G, ks > 0);
            }
            mma_commit_elect(bar + B_GP_FULL);
            if (j + 1 < ntile) {  // the region is free once the solve no longer reads A^T
                if (!(ok = wait(bar + B_AT_FREE, j & 1))) break;
                load(j + 1);
            }
        }
        mma_commit_elect(bar + B_DRAIN);
        if (lane == 0) mbar_wait(bar + B_DRAIN, 0, limit_ns);
        __syncwarp();
    } else {
        // ------------------------------------------------------------ workers (128 threads)
        const int wt = tid - 32;
        const int q = warp & 3;                       // TMEM lane quarter of this warp
        const int r = 16 * q + lane;                  // G row held by lanes 0-15 of each quarter
        const bool grow = lane < 16;
        const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
        auto beta_of = [&](int j) -> float {
            if (j >= ntile || wt >= 64) return 0.f;
            const long tile = first + (long)j * step;
            int c;
            const StreamJob jb = seqs.tile(tile, &c);
            const int t = c * 64 + wt;
            const __nv_bfloat16* p = beta + (long)jb.z * Tdim + jb.y0 + t;
            return t < jb.len && span_ok(err, b_span, p, 2) ? __bfloat162float(*p) : 0.f;
        };
        auto g_of = [&](int j) -> float {
            if (j >= ntile || wt >= 64) return 0.f;
            const long tile = first + (long)j * step;
            int c;
            const StreamJob jb = seqs.tile(tile, &c);
            const int t = c * 64 + wt;
            const float* p = gdec + (long)jb.z * Tdim + jb.y0 + t;
            return t < jb.len && span_ok(err, g_span, p, 4) ? *p : 0.f;
        };
        float beta_next = beta_of(0);
        float g_next = 0.f;
        if constexpr (kGated) g_next = g_of(0);
        bool ok = true;
        for (int j = 0; j < ntile; ++j) {
            if (wt < 64) {
                bt[wt] = beta_next;
                beta_next = beta_of(j + 1);
                if constexpr (kGated) {
                    graw[wt] = g_next;
                    g_next = g_of(j + 1);
                }
            }
            if constexpr (kGated) {   // cumulative log-decay (log2 units) by worker warp 0, a shuffle scan
                bar_sync(NB_W, 128);
                if (wt < 32) {
                    const float a0 = graw[2 * wt], a1 = graw[2 * wt + 1];
                    float run = a0 + a1;
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        const float y = __shfl_up_sync(0xffffffffu, run, off);
                        if (wt >= off) run += y;
                    }
                    float before = __shfl_up_sync(0xffffffffu, run, 1);
                    if (wt == 0) before = 0.f;
                    constexpr float kLog2e = 1.4426950408889634f;
                    gl[2 * wt] = (before + a0) * kLog2e;
                    gl[2 * wt + 1] = ((before + a0) + a1) * kLog2e;
                }
            }
            ok = bar_and(NB_W, 128, ok && wait_bounded(bar + B_GP_FULL, j & 1, abort, limit_ns));
            if (!ok) break;
            tc_fence_after();
            {   // lambda_r = G_rr from the 32-column half that holds column r (warp-uniform)
                float g[32];
                tmem_ld32_wait(tmem + lane_off + 32 * (q >> 1), g);
                if (grow) {
                    // a masked sum, not a select chain: it keeps g in registers (the compiler
                    // turns a select chain over g into an indexed local-memory load)
                    const int d = r - 32 * (q >> 1);
                    float lam = 0.f;
#pragma unroll
                    for (int e = 0; e < 32; ++e) lam = fmaf(g[e], e == d ? 1.f : 0.f, lam);
                    const float a = rule_alpha(rule, bt[r], lam);
                    al[r] = a;
                    if constexpr (kGated) {
                        abar[r] = rule_write_gate(rule, bt[r], lam, graw[r]);
                        mw[r] = a * exp2f(gl[r]);
                    }
                }
            }
            bar_sync(NB_W, 128);                     // alpha visible
            // A^T[r][i] = A[i][r] = alpha_i G[i][r] = alpha_i G[r][i]; only i > r is read.
            // The K tile under A^T was read by the finished G MMA.
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float g[32];
                tmem_ld32_wait(tmem + lane_off + 32 * h, g);
                if (grow) {
                    if constexpr (kGated) {
                        // A^T[r][i] = alpha_i (Gam_i / Gam_r) G[r][i]; only i > r is read, where the
                        // ratio is <= 1 for decays
                        const float glr = gl[r];
#pragma unroll
                        for (int m = 0; m < 8; ++m) {
                            const float4 a = *reinterpret_cast<const float4*>(al + 32 * h + 4 * m);
                            const float4 l = *reinterpret_cast<const float4*>(gl + 32 * h + 4 * m);
                            *reinterpret_cast<float4*>(At + r * LDX + 32 * h + 4 * m) =
                                make_float4(a.x * exp2f(l.x - glr) * g[4 * m], a.y * exp2f(l.y - glr) * g[4 * m + 1],
                                            a.z * exp2f(l.z - glr) * g[4 * m + 2], a.w * exp2f(l.w - glr) * g[4 * m + 3]);
                        }
                    } else {
#pragma unroll
                        for (int m = 0; m < 8; ++m) {
                            const float4 a = *reinterpret_cast<const float4*>(al + 32 * h + 4 * m);
                            *reinterpret_cast<float4*>(At + r * LDX + 32 * h + 4 * m) =
                                make_float4(a.x * g[4 * m], a.y * g[4 * m + 1], a.z * g[4 * m + 2], a.w * g[4 * m + 3]);
                        }
                    }
                }
            }
            tc_fence_before();
            if (Xout && wt == 0) tma_store_wait_read();   // the last tile's X has been copied out
            bar_sync(NB_W, 128);                     // G read, A^T written
            if (wt == 0) mbar_arrive(bar + B_GP_FREE);
            ut::ut_solve<NB_W, 128>(At, X, wt);
            // A^T is dead: the next K tile may land over it (the async-proxy TMA write is
            // ordered after this tile's generic writes there)
            fence_proxy_async_smem();
            bar_sync(NB_W, 128);
            if (wt == 0) mbar_arrive(bar + B_AT_FREE);
            if (Xout && wt == 0) {   // X itself, for the backward: one bulk copy of the padded tile
                float* dst = Xout + (first + (long)j * step) * 64 * LDX;
                if (span_ok(err, x_span, dst, F32_TILE)) bulk_store(dst, X, F32_TILE);
            }
            {   // T = X diag(alpha) -> bf16, 64 bytes per thread (a warp reads 32 consecutive
                // rows of one column half: conflict-free with the 68-float row stride).
                // Gated: T_W = X diag(alpha Gam), T_U = X diag(abar), and the row's G log2(e).
                const long tile = first + (long)j * step;
                const int rr = wt & 63, h = wt >> 6;
                auto store = [&](const float* mult, long tile_at) {
                    uint4* dst = reinterpret_cast<uint4*>(Tout + (tile_at * 64 + rr) * 64 + 32 * h);
                    if (!span_ok(err, t_span, dst, 64)) return;
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const float4 x0 = *reinterpret_cast<const float4*>(X + rr * LDX + 32 * h + 8 * m);
                        const float4 x1 = *reinterpret_cast<const float4*>(X + rr * LDX + 32 * h + 8 * m + 4);
                        const float4 a0 = *reinterpret_cast<const float4*>(mult + 32 * h + 8 * m);
                        const float4 a1 = *reinterpret_cast<const float4*>(mult + 32 * h + 8 * m + 4);
                        uint4 u;
                        u.x = pack_bf16x2(x0.x * a0.x, x0.y * a0.y);
                        u.y = pack_bf16x2(x0.z * a0.z, x0.w * a0.w);
                        u.z = pack_bf16x2(x1.x * a1.x, x1.y * a1.y);
                        u.w = pack_bf16x2(x1.z * a1.z, x1.w * a1.w);
                        dst[m] = u;
                    }
                };
                if constexpr (kGated) {
                    store(mw, tile);
                    store(abar, ntiles + tile);
                    float* gdst = reinterpret_cast<float*>(Tout + 2 * ntiles * 4096) + tile * 64 + wt;
                    if (wt < 64 && span_ok(err, t_span, gdst, 4)) *gdst = gl[wt];
                } else {
                    store(al, tile);
                }
            }
        }
    }

    if (Xout && tid == 32) tma_store_wait_all();
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort) atomicOr(err, kDevTimeout);
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

int sm_count() {
    static int n[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!n[dev] && cudaDeviceGetAttribute(&n[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n[dev] = 148;
    return n[dev];
}
}  // namespace

cudaError_t launch_ut(const void* k, const void* beta, void* Tout, const Seqs& seqs, long Z, int Tdim,
                      long ntiles, uint32_t* err, unsigned long long limit_ns, int rule, cudaStream_t stream,
                      const float* g, float* Xout) {
    if (ntiles == 0) return cudaSuccess;
    CUtensorMap mk;
    if (!tma_map_tokens(&mk, k, 128, Tdim, Z)) return cudaErrorInvalidValue;
    const long grid = std::min<long>(ntiles, (long)sm_count() * kCtasPerSm);
    const Span t_span{Tout, (size_t)ntiles * (g ? 2 * 8192 + 256 : 8192)};
    const Span b_span{beta, (size_t)Z * Tdim * 2}, g_span{g, (size_t)Z * Tdim * 4};
    const Span x_span{Xout, (size_t)ntiles * F32_TILE};
    cudaError_t e;
    if (g) {
        static std::atomic<uint64_t> smem_set_g{0};
        e = set_smem_limit_once(ut_kernel<true>, (int)SMEM_BYTES_G, smem_set_g);
        if (e != cudaSuccess) return e;
        ut_kernel<true><<<(unsigned)grid, kThreads, SMEM_BYTES_G, stream>>>(
            mk, (const __nv_bfloat16*)beta, (__nv_bfloat16*)Tout, seqs, Tdim, ntiles, err, limit_ns, rule, g, t_span,
            b_span, g_span, nullptr, x_span);
    } else {
        static std::atomic<uint64_t> smem_set{0};
        e = set_smem_limit_once(ut_kernel<false>, (int)SMEM_BYTES, smem_set);
        if (e != cudaSuccess) return e;
        ut_kernel<false><<<(unsigned)grid, kThreads, SMEM_BYTES, stream>>>(
            mk, (const __nv_bfloat16*)beta, (__nv_bfloat16*)Tout, seqs, Tdim, ntiles, err, limit_ns, rule, nullptr,
            t_span, b_span, g_span, Xout, x_span);
    }
    return cudaGetLastError();
}

}  // namespace efla
