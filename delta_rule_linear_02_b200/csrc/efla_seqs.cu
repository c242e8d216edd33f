// efla_seqs.cu -- chunk offsets of a packed variable-length batch.
//
// Exact Flow Linear Attention, Section 3.3 chunks each sequence on its own: sequence n's
// chunks start at its first token.  The UT kernel numbers the chunks of all sequences of a
// head consecutively, so it needs the prefix sums of the per-sequence chunk counts.
#include "efla_common.cuh"
#include "efla_kernels.h"

namespace efla {

namespace {
constexpr int kThreads = 1024;

// One CTA: each thread sums the chunk counts of a contiguous run of sequences, a shared-memory
// scan over the threads' sums gives each run's offset, then every run writes its prefix sums.
__global__ void __launch_bounds__(kThreads) seq_prep_kernel(const int* __restrict__ cu, int* __restrict__ tileoff,
                                                            int N) {
    __shared__ int part[kThreads];
    const int t = threadIdx.x;
    const int per = (N + kThreads - 1) / kThreads;
    const int n0 = min(N, t * per), n1 = min(N, n0 + per);
    int sum = 0;
    for (int n = n0; n < n1; ++n) sum += (cu[n + 1] - cu[n] + 63) / 64;
    part[t] = sum;
    __syncthreads();
    for (int off = 1; off < kThreads; off <<= 1) {   // inclusive scan (Hillis-Steele)
        const int y = t >= off ? part[t - off] : 0;
        __syncthreads();
        part[t] += y;
        __syncthreads();
    }
    int run = part[t] - sum;                         // exclusive offset of this run
    for (int n = n0; n < n1; ++n) {
        tileoff[n] = run;
        run += (cu[n + 1] - cu[n] + 63) / 64;
    }
    if (t == kThreads - 1) tileoff[N] = part[t];
}
}  // namespace

cudaError_t launch_seq_prep(const int* cu, int* tileoff, int N, cudaStream_t stream) {
    seq_prep_kernel<<<1, kThreads, 0, stream>>>(cu, tileoff, N);
    return cudaGetLastError();
}

}  // namespace efla
