// efla_api.cu -- the C ABI declared in include/efla.h: argument checks, then launches.
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <atomic>

#include "../../include/efla.h"
#include "efla_common.cuh"
#include "efla_kernels.h"

namespace {

constexpr size_t kWorkspaceHeader = 256;   // device error word + reserved

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
    return a0 < b0 + nb && b0 < a0 + na;
}

size_t elem_size(int dtype) { return dtype == EFLA_DTYPE_BF16 ? 2 : 4; }

int from_cuda(cudaError_t e) { return e == cudaSuccess ? EFLA_OK : EFLA_ERR_CUDA; }

}  // namespace

extern "C" {

const char* efla_status_string(int status) {
    switch (status) {
        case EFLA_OK: return "EFLA_OK";
        case EFLA_ERR_INVALID_ARG: return "EFLA_ERR_INVALID_ARG";
        case EFLA_ERR_UNSUPPORTED: return "EFLA_ERR_UNSUPPORTED";
        case EFLA_ERR_CUDA: return "EFLA_ERR_CUDA";
        case EFLA_ERR_TIMEOUT: return "EFLA_ERR_TIMEOUT";
        case EFLA_ERR_BOUNDS: return "EFLA_ERR_BOUNDS";
        default: return "EFLA_ERR_UNKNOWN";
    }
}

int efla_gate(const void* k, const void* beta, float* alpha, long n, int d_k, int dtype,
              efla_stream_t stream) {
    if (dtype != EFLA_DTYPE_F32 && dtype != EFLA_DTYPE_BF16) return EFLA_ERR_UNSUPPORTED;
    if (n < 0 || d_k < 1 || d_k > 4096) return EFLA_ERR_INVALID_ARG;
    if ((d_k * elem_size(dtype)) % 16 != 0) return EFLA_ERR_UNSUPPORTED;
    if (n == 0) return EFLA_OK;
    if (!k || !beta || !alpha || !aligned16(k) || !aligned16(beta) || !aligned16(alpha))
        return EFLA_ERR_INVALID_ARG;
    return from_cuda(efla::launch_gate(k, beta, alpha, n, d_k, dtype == EFLA_DTYPE_BF16,
                                       (cudaStream_t)stream));
}

static int check_chunk_shape(int B, int H, int T, int d_k, int d_v, int chunk, int dtype) {
    if (B < 0 || H < 0 || T < 0 || d_k <= 0 || d_v <= 0 || chunk <= 0) return EFLA_ERR_INVALID_ARG;
    if (dtype != EFLA_DTYPE_F32 && dtype != EFLA_DTYPE_BF16) return EFLA_ERR_UNSUPPORTED;
    if (d_k != d_v || (d_k != 64 && d_k != 128) || chunk != 64) return EFLA_ERR_UNSUPPORTED;
    if ((long long)B * H * 2 >= (1ll << 31)) return EFLA_ERR_UNSUPPORTED;
    return EFLA_OK;
}

size_t efla_chunk_fwd_workspace_bytes(int B, int H, int T, int d_k, int d_v, int chunk, int dtype) {
    if (check_chunk_shape(B, H, T, d_k, d_v, chunk, dtype) != EFLA_OK) return 0;
    if (dtype == EFLA_DTYPE_BF16 && d_k == 128)   // + the per-chunk UT transforms
        return kWorkspaceHeader + efla::chunk_tc_workspace_bytes((long)B * H, T);
    return kWorkspaceHeader;
}

size_t efla_chunk_fwd_gated_workspace_bytes(int B, int H, int T, int d_k, int d_v, int chunk, int dtype) {
    if (check_chunk_shape(B, H, T, d_k, d_v, chunk, dtype) != EFLA_OK) return 0;
    if (dtype == EFLA_DTYPE_BF16 && d_k == 128)   // + two transforms and the log-decays per chunk
        return kWorkspaceHeader + efla::chunk_tc_gated_workspace_bytes((long)B * H, T);
    return kWorkspaceHeader;
}

// The forward with or without the gated flow's log-decay g (null: ungated).
static int chunk_fwd_impl(const void* q, const void* k, const void* v, const void* beta, const float* g,
                          const float* S0, void* o, float* S_T, int B, int H, int T, int d_k, int d_v,
                          int chunk, int dtype, int rule, void* workspace, size_t workspace_bytes,
                          efla_stream_t stream, bool save = false) {
    int st = check_chunk_shape(B, H, T, d_k, d_v, chunk, dtype);
    if (st != EFLA_OK) return st;
    if (rule != EFLA_RULE_EXACT && rule != EFLA_RULE_EULER) return EFLA_ERR_INVALID_ARG;
    if (save && (g || dtype != EFLA_DTYPE_BF16 || d_k != 128)) return EFLA_ERR_UNSUPPORTED;
    const size_t need = save ? efla_train_saved_bytes(B, H, T, d_k, d_v, chunk, dtype)
                      : g    ? efla_chunk_fwd_gated_workspace_bytes(B, H, T, d_k, d_v, chunk, dtype)
                             : efla_chunk_fwd_workspace_bytes(B, H, T, d_k, d_v, chunk, dtype);
    if (!workspace || !aligned16(workspace) || workspace_bytes < need) return EFLA_ERR_INVALID_ARG;
    const long BH = (long)B * H;
    if (BH == 0) return EFLA_OK;
    const size_t es = elem_size(dtype);
    const size_t nqk = (size_t)BH * T * d_k * es, nv = (size_t)BH * T * d_v * es;
    const size_t nb = (size_t)BH * T * es, ns = (size_t)BH * d_k * d_v * sizeof(float);
    if ((S0 && !aligned16(S0)) || (S_T && !aligned16(S_T))) return EFLA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    if (T == 0) {   // empty sequence: the state passes through unchanged
        if (!S_T || S_T == S0) return EFLA_OK;
        return from_cuda(S0 ? cudaMemcpyAsync(S_T, S0, ns, cudaMemcpyDeviceToDevice, s)
                            : cudaMemsetAsync(S_T, 0, ns, s));
    }
    if (!q || !k || !v || !beta || !o) return EFLA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(beta) || !aligned16(o))
        return EFLA_ERR_INVALID_ARG;
    const size_t ng = g ? (size_t)BH * T * sizeof(float) : 0;
    if (g && !aligned16(g)) return EFLA_ERR_INVALID_ARG;
    if (overlaps(o, nv, q, nqk) || overlaps(o, nv, k, nqk) || overlaps(o, nv, v, nv) ||
        overlaps(o, nv, beta, nb) || overlaps(o, nv, S0, ns) || overlaps(o, nv, S_T, ns) ||
        overlaps(o, nv, g, ng) || overlaps(o, nv, workspace, workspace_bytes))
        return EFLA_ERR_INVALID_ARG;
    if (S_T && S_T != S0 &&
        (overlaps(S_T, ns, q, nqk) || overlaps(S_T, ns, k, nqk) || overlaps(S_T, ns, v, nv) ||
         overlaps(S_T, ns, beta, nb) || overlaps(S_T, ns, S0, ns) || overlaps(S_T, ns, g, ng)))
        return EFLA_ERR_INVALID_ARG;
    // the kernels write the workspace (error word, UT transforms) while the inputs are
    // still being read, and S_T last: neither may share bytes with it
    if (overlaps(workspace, workspace_bytes, q, nqk) || overlaps(workspace, workspace_bytes, k, nqk) ||
        overlaps(workspace, workspace_bytes, v, nv) || overlaps(workspace, workspace_bytes, beta, nb) ||
        overlaps(workspace, workspace_bytes, S0, ns) || overlaps(workspace, workspace_bytes, S_T, ns) ||
        overlaps(workspace, workspace_bytes, g, ng))
        return EFLA_ERR_INVALID_ARG;
    efla::Seqs seqs{nullptr, nullptr, 0, 0, T, 0};
    if (dtype == EFLA_DTYPE_BF16 && d_k == 128) {
        char* scratch = static_cast<char*>(workspace) + kWorkspaceHeader;
        efla::SegPlan plan;   // training: every chunk's entering state after the transforms
        if (save) {
            plan.X = reinterpret_cast<float*>(scratch + efla::bwd_saved_t_bytes(BH, T));
            plan.states = reinterpret_cast<__nv_bfloat16*>(scratch + efla::bwd_saved_t_bytes(BH, T) +
                                                           efla::bwd_saved_x_bytes(BH, T));
        }
        return from_cuda(efla::launch_chunk_tc(q, k, v, beta, S0, o, S_T, seqs, BH, BH, T, BH * ((T + 63) / 64),
                                               static_cast<uint32_t*>(workspace), scratch, rule, s, g, plan));
    }
    return from_cuda(efla::launch_chunk_simt(q, k, v, beta, S0, o, S_T, seqs, BH, T, d_k,
                                             dtype == EFLA_DTYPE_BF16, rule, s, g));
}

// ---------------------------------------------------------------- segmented scan of long streams
static int device_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 148;
    return n;
}

// Segments per stream: the request, or (0) the most whose chain CTAs still fit one wave
// (B*H*(4G - 2) <= SMs), each segment at least 8 chunks long.
static int seg_count(long BH, int T, int segments) {
    const int nchunks = (T + 63) / 64;
    int G = segments;
    if (G <= 0) {
        G = 1;
        while (BH * (4L * (G + 1) - 2) <= device_sms()) ++G;
    }
    G = std::min(G, std::max(1, nchunks / 8));
    return std::max(1, G);
}

static size_t seg_workspace(long BH, int T, int G, bool gated) {
    const size_t tiles = gated ? efla::chunk_tc_gated_workspace_bytes(BH, T) : efla::chunk_tc_workspace_bytes(BH, T);
    const size_t mats = (size_t)BH * G * 128 * 128 * sizeof(float);
    return kWorkspaceHeader + tiles + 3 * mats + (size_t)BH * T * 128 * 2;
}

size_t efla_chunk_fwd_segmented_workspace_bytes(int B, int H, int T, int d_k, int d_v, int chunk, int dtype, int gated,
                                                int segments) {
    if (check_chunk_shape(B, H, T, d_k, d_v, chunk, dtype) != EFLA_OK || segments < 0) return 0;
    const long BH = (long)B * H;
    if (!(dtype == EFLA_DTYPE_BF16 && d_k == 128) || BH == 0 || seg_count(BH, T, segments) == 1)
        return gated ? efla_chunk_fwd_gated_workspace_bytes(B, H, T, d_k, d_v, chunk, dtype)
                     : efla_chunk_fwd_workspace_bytes(B, H, T, d_k, d_v, chunk, dtype);
    return seg_workspace(BH, T, seg_count(BH, T, segments), gated);
}

int efla_chunk_fwd_segmented(const void* q, const void* k, const void* v, const void* beta, const float* g,
                             const float* S0, void* o, float* S_T, int B, int H, int T, int d_k, int d_v, int chunk,
                             int dtype, int rule, int segments, void* workspace, size_t workspace_bytes,
                             efla_stream_t stream) {
    int st = check_chunk_shape(B, H, T, d_k, d_v, chunk, dtype);
    if (st != EFLA_OK) return st;
    if (segments < 0) return EFLA_ERR_INVALID_ARG;
    const long BH = (long)B * H;
    const int G = BH > 0 ? seg_count(BH, T, segments) : 1;
    if (!(dtype == EFLA_DTYPE_BF16 && d_k == 128) || BH == 0 || T == 0 || G == 1)
        return chunk_fwd_impl(q, k, v, beta, g, S0, o, S_T, B, H, T, d_k, d_v, chunk, dtype, rule, workspace,
                              workspace_bytes, stream);
    // the argument checks of the plain forward (nothing is launched by them)
    if (rule != EFLA_RULE_EXACT && rule != EFLA_RULE_EULER) return EFLA_ERR_INVALID_ARG;
    const size_t need = seg_workspace(BH, T, G, g != nullptr);
    if (!workspace || !aligned16(workspace) || workspace_bytes < need) return EFLA_ERR_INVALID_ARG;
    if (!q || !k || !v || !beta || !o) return EFLA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(beta) || !aligned16(o) ||
        (S0 && !aligned16(S0)) || (S_T && !aligned16(S_T)) || (g && !aligned16(g)))
        return EFLA_ERR_INVALID_ARG;
    const size_t nx = (size_t)BH * T * d_k * 2, nb = (size_t)BH * T * 2, ns = (size_t)BH * d_k * d_v * 4;
    const size_t ng = g ? (size_t)BH * T * 4 : 0;
    const void* ins[6] = {q, k, v, beta, S0, g};
    const size_t inn[6] = {nx, nx, nx, nb, ns, ng};
    for (int j = 0; j < 6; ++j)
        if (overlaps(o, nx, ins[j], inn[j]) || overlaps(workspace, workspace_bytes, ins[j], inn[j]) ||
            (S_T != S0 && overlaps(S_T, ns, ins[j], inn[j])))
            return EFLA_ERR_INVALID_ARG;
    if (overlaps(o, nx, S_T, ns) || overlaps(o, nx, workspace, workspace_bytes) ||
        overlaps(S_T, ns, workspace, workspace_bytes))
        return EFLA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    char* ws = static_cast<char*>(workspace);
    char* scratch = ws + kWorkspaceHeader;
    const size_t tiles = g ? efla::chunk_tc_gated_workspace_bytes(BH, T) : efla::chunk_tc_workspace_bytes(BH, T);
    const size_t mats = (size_t)BH * G * 128 * 128 * sizeof(float);
    efla::SegPlan plan;
    plan.G = G;
    plan.seg_chunks = ((T + 63) / 64 + G - 1) / G;
    plan.Sloc = reinterpret_cast<float*>(scratch + tiles);
    plan.Phi = reinterpret_cast<float*>(scratch + tiles + mats);
    float* Sin = reinterpret_cast<float*>(scratch + tiles + 2 * mats);
    plan.R = reinterpret_cast<__nv_bfloat16*>(scratch + tiles + 3 * mats);
    efla::Seqs seqs{nullptr, nullptr, 0, 0, T, 0};
    cudaError_t e = efla::launch_chunk_tc(q, k, v, beta, S0, o, S_T, seqs, BH, BH, T, BH * ((T + 63) / 64),
                                          static_cast<uint32_t*>(workspace), scratch, rule, s, g, plan);
    if (e == cudaSuccess) e = efla::launch_seg_combine(plan, S0, S_T, Sin, BH, s);
    if (e == cudaSuccess) e = efla::launch_seg_correct(plan, Sin, static_cast<__nv_bfloat16*>(o), BH, T, s);
    return from_cuda(e);
}

// ---------------------------------------------------------------- packed variable-length batches
// Workspace: [header 256 B][cu: N+1 int32][tileoff: N+1 int32][pad to 256 B][UT tiles].
static size_t varlen_meta_bytes(int N) { return (((size_t)2 * (N + 1) * sizeof(int)) + 255) & ~(size_t)255; }

// Checks the host offsets; returns the chunks per head (sum of ceil(len / 64)) or -1.
static long varlen_chunks(const int* cu, int N) {
    if (!cu || N < 0 || cu[0] != 0) return -1;
    long chunks = 0;
    for (int n = 0; n < N; ++n) {
        if (cu[n + 1] < cu[n]) return -1;
        chunks += (cu[n + 1] - cu[n] + 63) / 64;
    }
    return chunks;
}

size_t efla_chunk_fwd_varlen_workspace_bytes(const int* cu_seqlens, int N, int H, int d_k, int d_v, int chunk,
                                             int dtype, int gated) {
    if (check_chunk_shape(1, H, 0, d_k, d_v, chunk, dtype) != EFLA_OK || N < 1) return 0;
    const long chunks = varlen_chunks(cu_seqlens, N);
    if (chunks < 0 || (long long)N * H * 2 >= (1ll << 31)) return 0;
    size_t tiles = 0;
    if (dtype == EFLA_DTYPE_BF16 && d_k == 128) {
        const long ntiles = chunks * H;
        tiles = gated ? (size_t)ntiles * (2 * 8192 + 256) : (size_t)ntiles * 8192;
    }
    return kWorkspaceHeader + varlen_meta_bytes(N) + tiles;
}

int efla_chunk_fwd_varlen(const void* q, const void* k, const void* v, const void* beta, const float* g,
                          const int* cu_seqlens, const float* S0, void* o, float* S_T, int N, int H, int d_k,
                          int d_v, int chunk, int dtype, int rule, void* workspace, size_t workspace_bytes,
                          efla_stream_t stream) {
    int st = check_chunk_shape(1, H, 0, d_k, d_v, chunk, dtype);
    if (st != EFLA_OK) return st;
    if (rule != EFLA_RULE_EXACT && rule != EFLA_RULE_EULER) return EFLA_ERR_INVALID_ARG;
    if (N < 1 || H < 1) return N == 0 || H == 0 ? EFLA_OK : EFLA_ERR_INVALID_ARG;
    const long chunks = varlen_chunks(cu_seqlens, N);
    if (chunks < 0) return EFLA_ERR_INVALID_ARG;
    const size_t need = efla_chunk_fwd_varlen_workspace_bytes(cu_seqlens, N, H, d_k, d_v, chunk, dtype, g != nullptr);
    if (need == 0) return EFLA_ERR_UNSUPPORTED;
    if (!workspace || !aligned16(workspace) || workspace_bytes < need) return EFLA_ERR_INVALID_ARG;
    const int total_T = cu_seqlens[N];
    const size_t es = elem_size(dtype);
    const size_t nqk = (size_t)H * total_T * d_k * es, nv = (size_t)H * total_T * d_v * es;
    const size_t nb = (size_t)H * total_T * es, ns = (size_t)N * H * d_k * d_v * sizeof(float);
    const size_t ng = g ? (size_t)H * total_T * sizeof(float) : 0;
    if ((S0 && !aligned16(S0)) || (S_T && !aligned16(S_T)) || (g && !aligned16(g))) return EFLA_ERR_INVALID_ARG;
    if (total_T > 0) {
        if (!q || !k || !v || !beta || !o) return EFLA_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(beta) || !aligned16(o))
            return EFLA_ERR_INVALID_ARG;
    }
    const void* ins[6] = {q, k, v, beta, S0, g};
    const size_t inn[6] = {nqk, nqk, nv, nb, ns, ng};
    for (int j = 0; j < 6; ++j)
        if (overlaps(o, nv, ins[j], inn[j]) || overlaps(workspace, workspace_bytes, ins[j], inn[j]) ||
            (S_T != S0 && overlaps(S_T, ns, ins[j], inn[j])))
            return EFLA_ERR_INVALID_ARG;
    if (overlaps(o, nv, S_T, ns) || overlaps(o, nv, workspace, workspace_bytes) ||
        overlaps(S_T, ns, workspace, workspace_bytes))
        return EFLA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    if (total_T == 0) {   // every sequence empty: the states pass through unchanged
        if (!S_T || S_T == S0) return EFLA_OK;
        return from_cuda(S0 ? cudaMemcpyAsync(S_T, S0, ns, cudaMemcpyDeviceToDevice, s) : cudaMemsetAsync(S_T, 0, ns, s));
    }
    char* ws = static_cast<char*>(workspace);
    int* cu_dev = reinterpret_cast<int*>(ws + kWorkspaceHeader);
    int* tileoff_dev = cu_dev + (N + 1);
    if (cudaMemcpyAsync(cu_dev, cu_seqlens, (size_t)(N + 1) * sizeof(int), cudaMemcpyHostToDevice, s) != cudaSuccess)
        return EFLA_ERR_CUDA;
    if (efla::launch_seq_prep(cu_dev, tileoff_dev, N, s) != cudaSuccess) return EFLA_ERR_CUDA;
    efla::Seqs seqs{cu_dev, tileoff_dev, N, H, 0, chunks};
    const long nstreams = (long)N * H;
    char* scratch = ws + kWorkspaceHeader + varlen_meta_bytes(N);
    if (dtype == EFLA_DTYPE_BF16 && d_k == 128)
        return from_cuda(efla::launch_chunk_tc(q, k, v, beta, S0, o, S_T, seqs, nstreams, H, total_T, chunks * H,
                                               static_cast<uint32_t*>(workspace), scratch, rule, s, g));
    return from_cuda(efla::launch_chunk_simt(q, k, v, beta, S0, o, S_T, seqs, nstreams, total_T, d_k,
                                             dtype == EFLA_DTYPE_BF16, rule, s, g));
}

int efla_chunk_fwd_ex(const void* q, const void* k, const void* v, const void* beta, const float* S0,
                      void* o, float* S_T, int B, int H, int T, int d_k, int d_v, int chunk, int dtype,
                      int rule, void* workspace, size_t workspace_bytes, efla_stream_t stream) {
    return chunk_fwd_impl(q, k, v, beta, nullptr, S0, o, S_T, B, H, T, d_k, d_v, chunk, dtype, rule, workspace,
                          workspace_bytes, stream);
}

int efla_chunk_fwd_gated(const void* q, const void* k, const void* v, const void* beta, const float* g,
                         const float* S0, void* o, float* S_T, int B, int H, int T, int d_k, int d_v, int chunk,
                         int dtype, int rule, void* workspace, size_t workspace_bytes, efla_stream_t stream) {
    if (!g && B > 0 && H > 0 && T > 0) return EFLA_ERR_INVALID_ARG;
    return chunk_fwd_impl(q, k, v, beta, g, S0, o, S_T, B, H, T, d_k, d_v, chunk, dtype, rule, workspace,
                          workspace_bytes, stream);
}

int efla_chunk_fwd(const void* q, const void* k, const void* v, const void* beta, const float* S0,
                   void* o, float* S_T, int B, int H, int T, int d_k, int d_v, int chunk, int dtype,
                   void* workspace, size_t workspace_bytes, efla_stream_t stream) {
    return efla_chunk_fwd_ex(q, k, v, beta, S0, o, S_T, B, H, T, d_k, d_v, chunk, dtype, EFLA_RULE_EXACT,
                             workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------- allocation-free variant
// Scratch for efla_chunk_fwd_noalloc: a file-scope device array, so that callers who
// cannot allocate device memory still get the chunked forward.  Every GPU that loads
// this library holds it until the process exits.  Host code cannot use the symbol
// itself as a device address; the address is looked up once per device below.
static constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;   // 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// The address is cached per device in an atomic slot (host threads may race on the first
// call; each writes the same value).  A cudaDeviceReset invalidates the module and with it
// the address: a process that resets a device must not call the no-alloc entry points on
// it afterwards.
static void* noalloc_scratch(int* status) {
    constexpr int kMaxDevices = 64;
    static std::atomic<void*> addr[kMaxDevices];
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *status = EFLA_ERR_CUDA;
        return nullptr;
    }
    void* p = addr[dev].load(std::memory_order_acquire);
    if (!p) {   // first call on this device (with it current): resolve the address
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            *status = EFLA_ERR_CUDA;
            return nullptr;
        }
        addr[dev].store(p, std::memory_order_release);
    }
    return p;
}

int efla_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const void* beta,
                           const float* S0, void* o, float* S_T, int B, int H, int T, int d_k,
                           int d_v, int chunk, int dtype, efla_stream_t stream) {
    int st = check_chunk_shape(B, H, T, d_k, d_v, chunk, dtype);
    if (st != EFLA_OK) return st;
    const size_t need = efla_chunk_fwd_workspace_bytes(B, H, T, d_k, d_v, chunk, dtype);
    if (need > kNoAllocScratchBytes) return EFLA_ERR_UNSUPPORTED;
    void* ws = noalloc_scratch(&st);
    if (!ws) return st;
    // the scratch keeps the previous call's contents: the device error word starts at zero
    if (cudaMemsetAsync(ws, 0, 16, (cudaStream_t)stream) != cudaSuccess) return EFLA_ERR_CUDA;
    return efla_chunk_fwd(q, k, v, beta, S0, o, S_T, B, H, T, d_k, d_v, chunk, dtype, ws, need, stream);
}

int efla_noalloc_status(int clear, efla_stream_t stream) {
    int st = EFLA_OK;
    void* ws = noalloc_scratch(&st);
    if (!ws) return st;
    return efla_workspace_status(ws, clear, stream);
}

int efla_workspace_status(void* workspace, int clear, efla_stream_t stream) {
    if (!workspace || !aligned16(workspace)) return EFLA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    uint32_t word = 0;
    if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return EFLA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return EFLA_ERR_CUDA;
    if (clear) {
        if (cudaMemsetAsync(workspace, 0, sizeof(word), s) != cudaSuccess) return EFLA_ERR_CUDA;
        if (cudaStreamSynchronize(s) != cudaSuccess) return EFLA_ERR_CUDA;
    }
    if (word == efla::kDevOk) return EFLA_OK;
    return (word & efla::kDevBounds) ? EFLA_ERR_BOUNDS : EFLA_ERR_TIMEOUT;
}

int efla_selftest_wait_timeout(void* workspace, long long limit_ns, efla_stream_t stream) {
    if (!workspace || !aligned16(workspace) || limit_ns < 0) return EFLA_ERR_INVALID_ARG;
    return from_cuda(efla::launch_wait_timeout_selftest(static_cast<uint32_t*>(workspace),
                                                        (unsigned long long)limit_ns,
                                                        (cudaStream_t)stream));
}

static int recurrent_step_impl(const void* q, const void* k, const void* v, const void* beta, const float* g,
                               float* S, void* o, int N, int H, int d_k, int d_v, int dtype, int rule,
                               efla_stream_t stream);

int efla_recurrent_step_ex(const void* q, const void* k, const void* v, const void* beta, float* S,
                           void* o, int N, int H, int d_k, int d_v, int dtype, int rule, efla_stream_t stream) {
    return recurrent_step_impl(q, k, v, beta, nullptr, S, o, N, H, d_k, d_v, dtype, rule, stream);
}

int efla_recurrent_step_gated(const void* q, const void* k, const void* v, const void* beta, const float* g,
                              float* S, void* o, int N, int H, int d_k, int d_v, int dtype, int rule,
                              efla_stream_t stream) {
    if (!g && N > 0 && H > 0) return EFLA_ERR_INVALID_ARG;
    return recurrent_step_impl(q, k, v, beta, g, S, o, N, H, d_k, d_v, dtype, rule, stream);
}

static int recurrent_step_impl(const void* q, const void* k, const void* v, const void* beta, const float* g,
                               float* S, void* o, int N, int H, int d_k, int d_v, int dtype, int rule,
                               efla_stream_t stream) {
    if (N < 0 || H < 0 || d_k <= 0 || d_v <= 0) return EFLA_ERR_INVALID_ARG;
    if (rule != EFLA_RULE_EXACT && rule != EFLA_RULE_EULER) return EFLA_ERR_INVALID_ARG;
    if (dtype != EFLA_DTYPE_F32 && dtype != EFLA_DTYPE_BF16) return EFLA_ERR_UNSUPPORTED;
    if (d_k != d_v || (d_k != 64 && d_k != 128)) return EFLA_ERR_UNSUPPORTED;
    const long NH = (long)N * H;
    if (NH == 0) return EFLA_OK;
    if (NH * (d_k / 32) >= (1l << 31)) return EFLA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !beta || !S || !o) return EFLA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(beta) || !aligned16(S) ||
        !aligned16(o))
        return EFLA_ERR_INVALID_ARG;
    const size_t es = elem_size(dtype);
    const size_t nq = (size_t)NH * d_k * es, nv = (size_t)NH * d_v * es, nb = (size_t)NH * es;
    const size_t ns = (size_t)NH * d_k * d_v * sizeof(float);
    const size_t ng = g ? (size_t)NH * sizeof(float) : 0;
    if (g && !aligned16(g)) return EFLA_ERR_INVALID_ARG;
    if (overlaps(o, nv, S, ns) || overlaps(o, nv, q, nq) || overlaps(o, nv, k, nq) ||
        overlaps(o, nv, v, nv) || overlaps(o, nv, beta, nb) || overlaps(S, ns, q, nq) ||
        overlaps(S, ns, k, nq) || overlaps(S, ns, v, nv) || overlaps(S, ns, beta, nb) ||
        overlaps(o, nv, g, ng) || overlaps(S, ns, g, ng))
        return EFLA_ERR_INVALID_ARG;
    return from_cuda(efla::launch_decode(q, k, v, beta, S, o, NH, d_k, dtype == EFLA_DTYPE_BF16, rule,
                                         (cudaStream_t)stream, g));
}

int efla_recurrent_step(const void* q, const void* k, const void* v, const void* beta, float* S,
                        void* o, int N, int H, int d_k, int d_v, int dtype, efla_stream_t stream) {
    return efla_recurrent_step_ex(q, k, v, beta, S, o, N, H, d_k, d_v, dtype, EFLA_RULE_EXACT, stream);
}

// ---------------------------------------------------------------- backward
static int check_bwd_shape(int B, int H, int T, int d_k, int d_v, int dtype) {
    if (B < 0 || H < 0 || T < 0 || d_k <= 0 || d_v <= 0) return EFLA_ERR_INVALID_ARG;
    if (dtype != EFLA_DTYPE_F32 && dtype != EFLA_DTYPE_BF16) return EFLA_ERR_UNSUPPORTED;
    if (d_k != d_v || (d_k != 64 && d_k != 128)) return EFLA_ERR_UNSUPPORTED;
    if ((long long)B * H * (d_k / 32) >= (1ll << 31)) return EFLA_ERR_UNSUPPORTED;
    return EFLA_OK;
}

// bf16 with d = 128 takes the backward through the chunkwise form (tensor cores); the rest
// the token-by-token reverse sweep (fp32 CUDA cores).
static bool bwd_chunked(int d_k, int dtype) { return dtype == EFLA_DTYPE_BF16 && d_k == 128; }

size_t efla_backward_workspace_bytes(int B, int H, int T, int d_k, int d_v, int dtype) {
    if (check_bwd_shape(B, H, T, d_k, d_v, dtype) != EFLA_OK) return 0;
    if (bwd_chunked(d_k, dtype)) return kWorkspaceHeader + efla::bwd_chunk_workspace_bytes((long)B * H, T);
    return efla::bwd_workspace_bytes((long)B * H, T, d_k);
}

int efla_backward_ex(const void* q, const void* k, const void* v, const void* beta, const float* S0,
                     const void* dO, const float* dS_T, float* dq, float* dk, float* dv, float* dbeta,
                     float* dS0, int B, int H, int T, int d_k, int d_v, int dtype, int rule, void* workspace,
                     size_t workspace_bytes, efla_stream_t stream) {
    int st = check_bwd_shape(B, H, T, d_k, d_v, dtype);
    if (st != EFLA_OK) return st;
    if (rule != EFLA_RULE_EXACT && rule != EFLA_RULE_EULER) return EFLA_ERR_INVALID_ARG;
    const long BH = (long)B * H;
    const size_t ns = (size_t)BH * d_k * d_v * sizeof(float);
    cudaStream_t s = (cudaStream_t)stream;
    if ((S0 && !aligned16(S0)) || (dS_T && !aligned16(dS_T)) || (dS0 && !aligned16(dS0)))
        return EFLA_ERR_INVALID_ARG;
    if (BH == 0) return EFLA_OK;
    if (T == 0) {   // no token: the state gradient passes through
        if (!dS0 || dS0 == dS_T) return EFLA_OK;
        return from_cuda(dS_T ? cudaMemcpyAsync(dS0, dS_T, ns, cudaMemcpyDeviceToDevice, s)
                              : cudaMemsetAsync(dS0, 0, ns, s));
    }
    const size_t need = efla_backward_workspace_bytes(B, H, T, d_k, d_v, dtype);
    if (!workspace || !aligned16(workspace) || workspace_bytes < need) return EFLA_ERR_INVALID_ARG;
    if (!q || !k || !v || !beta || !dO || !dq || !dk || !dv || !dbeta) return EFLA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(beta) || !aligned16(dO) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(dbeta))
        return EFLA_ERR_INVALID_ARG;
    const size_t es = elem_size(dtype);
    const size_t nqk = (size_t)BH * T * d_k * es, nv = (size_t)BH * T * d_v * es, nb = (size_t)BH * T * es;
    const size_t gqk = (size_t)BH * T * d_k * 4, gv = (size_t)BH * T * d_v * 4, gb = (size_t)BH * T * 4;
    // every output must be disjoint from every input, from the workspace and from the others
    const void* outs[5] = {dq, dk, dv, dbeta, dS0};
    const size_t outn[5] = {gqk, gqk, gv, gb, ns};
    const void* ins[8] = {q, k, v, beta, dO, S0, dS_T, workspace};
    const size_t inn[8] = {nqk, nqk, nv, nb, nv, ns, ns, workspace_bytes};
    for (int i = 0; i < 5; ++i) {
        for (int j = 0; j < 8; ++j)
            if (overlaps(outs[i], outn[i], ins[j], inn[j])) return EFLA_ERR_INVALID_ARG;
        for (int j = i + 1; j < 5; ++j)
            if (overlaps(outs[i], outn[i], outs[j], outn[j])) return EFLA_ERR_INVALID_ARG;
    }
    // the forward sweep writes its residuals into the workspace before the reverse sweep
    // reads the inputs: no input may share bytes with it
    for (int j = 0; j < 7; ++j)
        if (overlaps(workspace, workspace_bytes, ins[j], inn[j])) return EFLA_ERR_INVALID_ARG;
    if (bwd_chunked(d_k, dtype))
        return from_cuda(efla::launch_bwd_chunk(q, k, v, beta, S0, dO, dS_T, dq, dk, dv, dbeta, dS0, BH, T, rule,
                                                static_cast<uint32_t*>(workspace),
                                                static_cast<char*>(workspace) + kWorkspaceHeader, s));
    return from_cuda(efla::launch_bwd(q, k, v, beta, S0, dO, dS_T, dq, dk, dv, dbeta, dS0, BH, T, d_k,
                                      dtype == EFLA_DTYPE_BF16, rule, workspace, s));
}

// ---------------------------------------------------------------- training: saved residuals
size_t efla_train_saved_bytes(int B, int H, int T, int d_k, int d_v, int chunk, int dtype) {
    if (check_chunk_shape(B, H, T, d_k, d_v, chunk, dtype) != EFLA_OK) return 0;
    if (dtype != EFLA_DTYPE_BF16 || d_k != 128) return 0;
    const long BH = (long)B * H;
    return kWorkspaceHeader + efla::bwd_saved_t_bytes(BH, T) + efla::bwd_saved_x_bytes(BH, T) +
           efla::bwd_saved_state_bytes(BH, T);
}

int efla_chunk_fwd_save(const void* q, const void* k, const void* v, const void* beta, const float* S0, void* o,
                        float* S_T, int B, int H, int T, int d_k, int d_v, int chunk, int dtype, int rule,
                        void* saved, size_t saved_bytes, efla_stream_t stream) {
    if (check_chunk_shape(B, H, T, d_k, d_v, chunk, dtype) == EFLA_OK && (dtype != EFLA_DTYPE_BF16 || d_k != 128))
        return EFLA_ERR_UNSUPPORTED;
    return chunk_fwd_impl(q, k, v, beta, nullptr, S0, o, S_T, B, H, T, d_k, d_v, chunk, dtype, rule, saved,
                          saved_bytes, stream, true);
}

size_t efla_backward_saved_workspace_bytes(int B, int H, int T, int d_k, int d_v, int dtype) {
    if (check_bwd_shape(B, H, T, d_k, d_v, dtype) != EFLA_OK || !bwd_chunked(d_k, dtype)) return 0;
    return kWorkspaceHeader + efla::bwd_saved_state_bytes((long)B * H, T);   // every chunk's dS'
}

int efla_backward_saved(const void* q, const void* k, const void* v, const void* beta, const void* dO,
                        const float* dS_T, float* dq, float* dk, float* dv, float* dbeta, float* dS0, int B, int H,
                        int T, int d_k, int d_v, int dtype, int rule, const void* saved, size_t saved_bytes,
                        void* workspace, size_t workspace_bytes, efla_stream_t stream) {
    int st = check_bwd_shape(B, H, T, d_k, d_v, dtype);
    if (st != EFLA_OK) return st;
    if (!bwd_chunked(d_k, dtype)) return EFLA_ERR_UNSUPPORTED;
    if (rule != EFLA_RULE_EXACT && rule != EFLA_RULE_EULER) return EFLA_ERR_INVALID_ARG;
    const long BH = (long)B * H;
    const size_t ns = (size_t)BH * d_k * d_v * sizeof(float);
    cudaStream_t s = (cudaStream_t)stream;
    if ((dS_T && !aligned16(dS_T)) || (dS0 && !aligned16(dS0))) return EFLA_ERR_INVALID_ARG;
    if (BH == 0) return EFLA_OK;
    if (T == 0) {   // no token: the state gradient passes through
        if (!dS0 || dS0 == dS_T) return EFLA_OK;
        return from_cuda(dS_T ? cudaMemcpyAsync(dS0, dS_T, ns, cudaMemcpyDeviceToDevice, s)
                              : cudaMemsetAsync(dS0, 0, ns, s));
    }
    const size_t need_ws = efla_backward_saved_workspace_bytes(B, H, T, d_k, d_v, dtype);
    const size_t need_saved = efla_train_saved_bytes(B, H, T, d_k, d_v, 64, dtype);
    if (!workspace || !aligned16(workspace) || workspace_bytes < need_ws) return EFLA_ERR_INVALID_ARG;
    if (!saved || !aligned16(saved) || saved_bytes < need_saved) return EFLA_ERR_INVALID_ARG;
    if (!q || !k || !v || !beta || !dO || !dq || !dk || !dv || !dbeta) return EFLA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(beta) || !aligned16(dO) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(dbeta))
        return EFLA_ERR_INVALID_ARG;
    const size_t es = elem_size(dtype);
    const size_t nqk = (size_t)BH * T * d_k * es, nv = (size_t)BH * T * d_v * es, nb = (size_t)BH * T * es;
    const size_t gqk = (size_t)BH * T * d_k * 4, gv = (size_t)BH * T * d_v * 4, gb = (size_t)BH * T * 4;
    // every output and the workspace must be disjoint from every input and from each other
    const void* outs[6] = {dq, dk, dv, dbeta, dS0, workspace};
    const size_t outn[6] = {gqk, gqk, gv, gb, ns, workspace_bytes};
    const void* ins[7] = {q, k, v, beta, dO, dS_T, saved};
    const size_t inn[7] = {nqk, nqk, nv, nb, nv, ns, saved_bytes};
    for (int i = 0; i < 6; ++i) {
        for (int j = 0; j < 7; ++j)
            if (overlaps(outs[i], outn[i], ins[j], inn[j])) return EFLA_ERR_INVALID_ARG;
        for (int j = i + 1; j < 6; ++j)
            if (overlaps(outs[i], outn[i], outs[j], outn[j])) return EFLA_ERR_INVALID_ARG;
    }
    const char* sv = static_cast<const char*>(saved) + kWorkspaceHeader;
    return from_cuda(efla::launch_bwd_chunk_saved(q, k, v, beta, dO, dS_T, dq, dk, dv, dbeta, dS0, BH, T, rule,
                                                  static_cast<uint32_t*>(workspace), sv,
                                                  reinterpret_cast<const float*>(sv + efla::bwd_saved_t_bytes(BH, T)),
                                                  sv + efla::bwd_saved_t_bytes(BH, T) + efla::bwd_saved_x_bytes(BH, T),
                                                  static_cast<char*>(workspace) + kWorkspaceHeader, s));
}

int efla_backward(const void* q, const void* k, const void* v, const void* beta, const float* S0,
                  const void* dO, const float* dS_T, float* dq, float* dk, float* dv, float* dbeta,
                  float* dS0, int B, int H, int T, int d_k, int d_v, int dtype, void* workspace,
                  size_t workspace_bytes, efla_stream_t stream) {
    return efla_backward_ex(q, k, v, beta, S0, dO, dS_T, dq, dk, dv, dbeta, dS0, B, H, T, d_k, d_v, dtype,
                            EFLA_RULE_EXACT, workspace, workspace_bytes, stream);
}

}  // extern "C"
