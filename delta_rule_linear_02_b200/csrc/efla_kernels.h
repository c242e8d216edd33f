// efla_kernels.h -- internal launchers (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

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
// nstreams recurrences described by `seqs` over tensors [Z][Tdim][d]; ntiles UT tiles
cudaError_t launch_chunk_tc(const void* q, const void* k, const void* v, const void* beta, const float* S0,
                            void* o, float* S_T, const Seqs& seqs, long nstreams, long Z, int Tdim, long ntiles,
                            uint32_t* err, void* scratch, int rule, cudaStream_t stream, const float* g = nullptr);
// g != null: the gated flow's transforms (two per tile plus the cumulative log-decay, see
// efla_ut.cu) into Tout, which then holds chunk_tc_gated_workspace_bytes.
// tiles: ntiles of `seqs` (dense: BH * ceil(T / 64); packed: H * tileoff[N]); tensors [Z][Tdim][d]
cudaError_t launch_ut(const void* k, const void* beta, void* Tout, const Seqs& seqs, long Z, int Tdim,
                      long ntiles, uint32_t* err, unsigned long long limit_ns, int rule, cudaStream_t stream,
                      const float* g = nullptr);

// reverse-mode pass (efla_bwd.cu): fp32 gradients; workspace of bwd_workspace_bytes
size_t bwd_workspace_bytes(long BH, int T, int D);
cudaError_t launch_bwd(const void* q, const void* k, const void* v, const void* beta, const float* S0,
                       const void* dO, const float* dST, float* dq, float* dk, float* dv, float* dbeta, float* dS0,
                       long BH, int T, int D, bool bf16, int rule, void* workspace, cudaStream_t stream);

// packed batches: tileoff[n] = sum over m < n of ceil((cu[m+1] - cu[m]) / 64), n = 0..N
cudaError_t launch_seq_prep(const int* cu, int* tileoff, int N, cudaStream_t stream);

cudaError_t launch_wait_timeout_selftest(uint32_t* err, unsigned long long limit_ns, cudaStream_t stream);

}  // namespace efla
