// efla_kernels.h -- internal launchers (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <cuda_bf16.h>

#include "efla_common.cuh"

namespace efla {

cudaError_t launch_gate(const void* k, const void* beta, float* alpha, long n, int dk, bool bf16,
                        cudaStream_t stream);

// rule: kRuleExact (the exact-flow gate) or kRuleEuler (alpha = beta, the delta rule).
// g: per-token log-decay (float32, one per stream and token) for the gated flow, or null.
cudaError_t launch_decode(const void* q, const void* k, const void* v, const void* beta, float* S,
                          void* o, long NH, int D, bool bf16, int rule, cudaStream_t stream,
                          const float* g = nullptr);

cudaError_t launch_chunk_simt(const void* q, const void* k, const void* v, const void* beta,
                              const float* S0, void* o, float* S_T, const Seqs& seqs, long nstreams, int Tdim,
                              int D, bool bf16, int rule, cudaStream_t stream, const float* g = nullptr);

// bf16, d_k = d_v = 128: the UT kernel (efla_ut.cu) writes every chunk's T into `scratch`
// (chunk_tc_workspace_bytes bytes, 16-byte aligned), then the chain kernel runs.
size_t chunk_tc_workspace_bytes(long BH, int T);
// the gated flow (g != null): two transforms and the cumulative log-decay per chunk
size_t chunk_tc_gated_workspace_bytes(long BH, int T);
// Segmented scan of long streams (d = 128, bf16).  With G > 1 every stream is split into G
// segments of seg_chunks chunks (the last takes the rest).  The chain launch then runs per
// stream 2 CTAs for segment 0 (from S0, exact outputs, final state into Sloc[.][0]) and 4 per
// later segment g: 2 from a zero state (outputs O_loc into o, final state into Sloc[.][g]) and
// 2 for the segment's transition product (V = 0 from S = I: final state Phi[.][g], outputs
// R into R).  The chunk map S -> (I - K^T W) S + K^T U is affine, so the true entering state
// of segment g is S_in(g) = Phi[g-1] S_in(g-1) + Sloc[g-1] and its outputs O_loc + R S_in(g).
struct SegPlan {
    __nv_bfloat16* states = nullptr;   // if set: the entering state of every chunk, bf16 [tiles][128][128]
    float* X = nullptr;                // if set: X = (I + A)^{-1} of every chunk, fp32 [tiles][64][68] (ungated)
    int G = 1;                     // 1: no segmentation
    int seg_chunks = 0;
    float* Sloc = nullptr;         // [nstreams][G][128][128]
    float* Phi = nullptr;          // [nstreams][G][128][128]
    __nv_bfloat16* R = nullptr;    // [Z][Tdim][128] (rows of segments >= 1)
};

// The extents of every buffer the chain kernel addresses directly (checked builds test each
// access against them; see efla_common.cuh).
struct ChainSpans {
    Span o, r, s0, st, sloc, phi, states, gl;
    long t_rows = 0;               // rows of the tensor map over the UT transforms
};

// nstreams recurrences described by `seqs` over tensors [Z][Tdim][d]; ntiles UT tiles
cudaError_t launch_chunk_tc(const void* q, const void* k, const void* v, const void* beta, const float* S0,
                            void* o, float* S_T, const Seqs& seqs, long nstreams, long Z, int Tdim, long ntiles,
                            uint32_t* err, void* scratch, int rule, cudaStream_t stream, const float* g = nullptr,
                            const SegPlan& seg = SegPlan());
// the segmented scan's combine (S_in of every segment, S_T) and output correction o += R S_in
// (SinT: bf16 [nstreams][G][128][128], S_in of every segment transposed, written by the combine)
cudaError_t launch_seg_combine(const SegPlan& seg, const float* S0, float* S_T, void* SinT, long nstreams,
                               cudaStream_t stream);
cudaError_t launch_seg_correct(const SegPlan& seg, const void* SinT, __nv_bfloat16* o, long nstreams, int T,
                               cudaStream_t stream);
// g != null: the gated flow's transforms (two per tile plus the cumulative log-decay, see
// efla_ut.cu) into Tout, which then holds chunk_tc_gated_workspace_bytes.
// tiles: ntiles of `seqs` (dense: BH * ceil(T / 64); packed: H * tileoff[N]); tensors [Z][Tdim][d]
cudaError_t launch_ut(const void* k, const void* beta, void* Tout, const Seqs& seqs, long Z, int Tdim,
                      long ntiles, uint32_t* err, unsigned long long limit_ns, int rule, cudaStream_t stream,
                      const float* g = nullptr, float* Xout = nullptr);
// bytes of one chunk's X as launch_ut writes it (fp32 64 x 64, rows padded to 68 floats)
constexpr size_t kUtXBytes = 64 * 68 * 4;

// reverse-mode pass (efla_bwd.cu): fp32 gradients; workspace of bwd_workspace_bytes
size_t bwd_workspace_bytes(long BH, int T, int D);
cudaError_t launch_bwd(const void* q, const void* k, const void* v, const void* beta, const float* S0,
                       const void* dO, const float* dST, float* dq, float* dk, float* dv, float* dbeta, float* dS0,
                       long BH, int T, int D, bool bf16, int rule, void* workspace, cudaStream_t stream);

// packed batches: tileoff[n] = sum over m < n of ceil((cu[m+1] - cu[m]) / 64), n = 0..N
cudaError_t launch_seq_prep(const int* cu, int* tileoff, int N, cudaStream_t stream);

// the backward through the chunkwise form (bf16, d = 128): UT transforms, the forward chain
// storing each chunk's entering state, the reverse chain (dS' per chunk), per-chunk gradients.
// scratch: bwd_chunk_workspace_bytes bytes (16-byte aligned); err: the device error word.
size_t bwd_chunk_workspace_bytes(long BH, int T);
cudaError_t launch_bwd_chunk(const void* q, const void* k, const void* v, const void* beta, const float* S0,
                             const void* dO, const float* dST, float* dq, float* dk, float* dv, float* dbeta,
                             float* dS0, long BH, int T, int rule, uint32_t* err, void* scratch, cudaStream_t stream);
// the same from saved residuals (training): T of every chunk (Tt, ntiles x 64 x 64 bf16), its
// X = (I + A)^{-1} (fp32, kUtXBytes each) and every chunk's entering state (states, ntiles x
// 128 x 128 bf16) as the forward left them; dSp: the per-chunk dS' scratch (bf16 128 x 128)
cudaError_t launch_bwd_chunk_saved(const void* q, const void* k, const void* v, const void* beta, const void* dO,
                                   const float* dST, float* dq, float* dk, float* dv, float* dbeta, float* dS0,
                                   long BH, int T, int rule, uint32_t* err, const void* Tt, const float* X,
                                   const void* states, void* dSp, cudaStream_t stream);
// bytes of T (bf16), of X (fp32, launch_ut's padded tiles) and of the entering states (bf16)
// kept for the backward (d = 128)
size_t bwd_saved_t_bytes(long BH, int T);
size_t bwd_saved_x_bytes(long BH, int T);
size_t bwd_saved_state_bytes(long BH, int T);

cudaError_t launch_wait_timeout_selftest(uint32_t* err, unsigned long long limit_ns, cudaStream_t stream);

}  // namespace efla
