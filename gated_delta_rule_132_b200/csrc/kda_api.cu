// kda_api.cu — the exported C ABI: argument checks, workspace sizing, dispatch.
//
// Every check here runs on the host before any launch and touches no device
// state, so a rejected call has no side effects (and can be made without a GPU).
#include <math.h>
#include <stdlib.h>

#include <atomic>

#include "kda_internal.cuh"

namespace {

std::atomic<unsigned long long> g_launches{0};
std::atomic<uint32_t> g_wait_limit{0};
std::atomic<int> g_starve_carry{0};

// KDA_DEBUG_SYNC=1 in the environment: every prefill call waits for its work
// and returns KDA_ERR_DEVICE_STATUS if a bounded wait ran out.
bool debug_sync()
{
    static const bool on = [] {
        const char *e = getenv("KDA_DEBUG_SYNC");
        return e != nullptr && e[0] != '\0' && e[0] != '0';
    }();
    return on;
}

bool aligned16(const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool head_ok(int dk, int dv) { return dk == dv && (dk == 32 || dk == 64 || dk == 128); }
bool dtype_ok(kda_dtype_t t) { return t == KDA_DTYPE_F32 || t == KDA_DTYPE_BF16; }

// Shapes -> Problem (pointers left null); returns KDA_OK or the first problem found.
kda_status_t describe(int B, int T, int H, int dk, int dv, int n_seqs, bool varlen,
                      kda_dtype_t dt, kda::Problem *p)
{
    if (B < 1 || T < 0 || H < 1 || dk < 1 || dv < 1) return KDA_ERR_INVALID_ARG;
    if (!dtype_ok(dt)) return KDA_ERR_UNSUPPORTED;
    if (!head_ok(dk, dv)) return KDA_ERR_UNSUPPORTED;
    if (H > 65535) return KDA_ERR_UNSUPPORTED;
    if (varlen && (B != 1 || n_seqs < 1)) return KDA_ERR_INVALID_ARG;
    const long long total = (long long)B * T;
    if (total > (long long)INT32_MAX - kda::kChunk) return KDA_ERR_UNSUPPORTED;
    const int N = varlen ? n_seqs : B;
    if ((long long)N * H * 4 > (long long)INT32_MAX) return KDA_ERR_UNSUPPORTED;  // carry grid
    long long chunks = varlen ? total / kda::kChunk + N
                              : (long long)B * ((T + kda::kChunk - 1) / kda::kChunk);
    if (chunks > (long long)INT32_MAX) return KDA_ERR_UNSUPPORTED;
    *p = kda::Problem{};
    p->N = N; p->B = B; p->T = T; p->H = H; p->dk = dk; p->dv = dv; p->dtype = dt;
    p->total_tokens = total;
    p->max_chunks = (int)chunks;
    p->gate_per_channel = 1;
    p->nseg = 1;
    return KDA_OK;
}

bool use_tc(const kda::Problem &p, int algo) {
    if (algo == KDA_ALGO_SIMT) return false;
    return kda::tc_supported(p);
}

bool tc_only(int algo) { return algo != KDA_ALGO_AUTO && algo != KDA_ALGO_SIMT; }

// Algorithm values beyond the public kda_algo_t: the tensor-core path with an
// explicit number of time segments (kda_chunk_fwd_timesplit).
constexpr int kAlgoSegmentsBase = 1000;

bool algo_ok(int algo)
{
    return algo == KDA_ALGO_AUTO || algo == KDA_ALGO_SIMT || algo == KDA_ALGO_TCGEN05 ||
           algo == KDA_ALGO_TCGEN05_SEQUENTIAL ||
           (algo > kAlgoSegmentsBase && algo <= kAlgoSegmentsBase + kda::kMaxSegments);
}

// Time segments of the sequential phase on the tensor-core path for `algo`.
int segments_for(const kda::Problem &p, int algo)
{
    if (algo == KDA_ALGO_TCGEN05_SEQUENTIAL) return 1;
    if (algo > kAlgoSegmentsBase) return algo - kAlgoSegmentsBase;
    return kda::tc_auto_segments(p);
}

size_t required_bytes(kda::Problem &p, bool tc, int algo) {
    if (!tc) return kda::simt_workspace_layout(p).total;
    p.nseg = segments_for(p, algo);
    return kda::tc_workspace_layout(p).total;
}

}  // namespace

namespace kda {

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

DebugKnobs debug_knobs()
{
    return DebugKnobs{g_wait_limit.load(std::memory_order_relaxed),
                      g_starve_carry.load(std::memory_order_relaxed)};
}

}  // namespace kda

extern "C" {

unsigned long long kda_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

kda_status_t kda_debug_set_wait_limit(unsigned int polls, int starve_carry)
{
    g_wait_limit.store(polls, std::memory_order_relaxed);
    g_starve_carry.store(starve_carry ? 1 : 0, std::memory_order_relaxed);
    return KDA_OK;
}

kda_status_t kda_chunk_fwd_status(const void *workspace, size_t workspace_bytes,
                                  int *device_code, void *stream)
{
    if (!workspace || !device_code) return KDA_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return KDA_ERR_ALIGNMENT;
    if (workspace_bytes < kda::kWsHeader) return KDA_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int code = 0;
    if (cudaMemcpyAsync(&code, workspace, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return KDA_ERR_CUDA;
    *device_code = code;
    return code != 0 ? KDA_ERR_DEVICE_STATUS : KDA_OK;
}

const char *kda_status_string(kda_status_t s)
{
    switch (s) {
    case KDA_OK: return "ok";
    case KDA_ERR_INVALID_ARG: return "invalid argument";
    case KDA_ERR_UNSUPPORTED: return "unsupported size or dtype";
    case KDA_ERR_ALIGNMENT: return "buffer not 16-byte aligned";
    case KDA_ERR_WORKSPACE: return "workspace missing or too small";
    case KDA_ERR_CUDA: return "CUDA error";
    case KDA_ERR_DEVICE_STATUS: return "device reported an out-of-domain input";
    }
    return "unknown status";
}

int kda_version(void) { return 310; }  // 0.3.1: backward algorithm selection

size_t kda_chunk_fwd_workspace_size_ex(int B, int T, int H, int dk, int dv, int n_seqs,
                                       kda_dtype_t dt, int algo)
{
    if (!algo_ok(algo)) return 0;
    kda::Problem p;
    const bool varlen = n_seqs > 0 && B == 1;
    if (describe(B, T, H, dk, dv, n_seqs, varlen, dt, &p) != KDA_OK) return 0;
    const bool tc = use_tc(p, algo);
    if (tc_only(algo) && !tc) return 0;
    return required_bytes(p, tc, algo);
}

size_t kda_chunk_fwd_timesplit_workspace_size(int B, int T, int H, int dk, int dv, int n_seqs,
                                              kda_dtype_t dt, int segments)
{
    if (segments < 0 || segments > kda::kMaxSegments) return 0;
    return kda_chunk_fwd_workspace_size_ex(
        B, T, H, dk, dv, n_seqs, dt, segments == 0 ? KDA_ALGO_TCGEN05 : kAlgoSegmentsBase + segments);
}

size_t kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int n_seqs,
                                    kda_dtype_t dt)
{
    return kda_chunk_fwd_workspace_size_ex(B, T, H, dk, dv, n_seqs, dt, KDA_ALGO_AUTO);
}

}  // extern "C"

static kda_status_t chunk_fwd_phases(const void *q, const void *k, const void *v,
                                     kda_dtype_t dt, const float *log_alpha,
                                     const float *beta, const float *S0,
                                     const int32_t *cu_seqlens, int n_seqs, int B, int T,
                                     int H, int dk, int dv, float scale, void *o,
                                     float *S_final, void *workspace, size_t workspace_bytes,
                                     int algo, int phases, int gate_per_channel, void *stream)
{
    if (!algo_ok(algo)) return KDA_ERR_INVALID_ARG;
    kda::Problem p;
    kda_status_t st = describe(B, T, H, dk, dv, n_seqs, cu_seqlens != nullptr, dt, &p);
    if (st != KDA_OK) return st;
    if (!isfinite(scale)) return KDA_ERR_INVALID_ARG;
    if (p.total_tokens > 0 && (!q || !k || !v || !log_alpha || !beta || !o))
        return KDA_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, log_alpha, beta, S0, o, S_final, workspace};
    for (const void *ptr : ptrs)
        if (!aligned16(ptr)) return KDA_ERR_ALIGNMENT;
    if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return KDA_ERR_ALIGNMENT;
    const bool tc = use_tc(p, algo);
    if (tc_only(algo) && !tc) return KDA_ERR_UNSUPPORTED;
    const size_t need = required_bytes(p, tc, algo);
    if (need > 0 && (!workspace || workspace_bytes < need)) return KDA_ERR_WORKSPACE;

    p.q = q; p.k = k; p.v = v; p.log_alpha = log_alpha; p.beta = beta; p.S0 = S0;
    p.cu_seqlens = cu_seqlens; p.scale = scale; p.o = o; p.S_final = S_final;
    p.gate_per_channel = gate_per_channel;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const cudaError_t e = tc ? kda::launch_tc_prefill(p, workspace, phases, s)
                             : kda::launch_simt_prefill(p, workspace, phases, s);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    if (debug_sync()) {
        int code = 0;
        return kda_chunk_fwd_status(workspace, workspace_bytes, &code, stream);
    }
    return KDA_OK;
}

extern "C" {

#define KDA_CHUNK_ARGS q, k, v, dt, log_alpha, beta, S0, cu_seqlens, n_seqs, B, T, H, dk, dv, \
    scale, o, S_final, workspace, workspace_bytes

kda_status_t kda_chunk_fwd_ex(const void *q, const void *k, const void *v, kda_dtype_t dt,
                              const float *log_alpha, const float *beta, const float *S0,
                              const int32_t *cu_seqlens, int n_seqs, int B, int T, int H,
                              int dk, int dv, float scale, void *o, float *S_final,
                              void *workspace, size_t workspace_bytes, int algo, void *stream)
{
    return chunk_fwd_phases(KDA_CHUNK_ARGS, algo, kda::kPhaseAll, 1, stream);
}

kda_status_t kda_gdn_chunk_fwd(const void *q, const void *k, const void *v, kda_dtype_t dt,
                               const float *log_alpha, const float *beta, const float *S0,
                               const int32_t *cu_seqlens, int n_seqs, int B, int T, int H,
                               int dk, int dv, float scale, void *o, float *S_final,
                               void *workspace, size_t workspace_bytes, int algo, void *stream)
{
    return chunk_fwd_phases(KDA_CHUNK_ARGS, algo, kda::kPhaseAll, 0, stream);
}

kda_status_t kda_gdn_chunk_fwd_prepare(const void *q, const void *k, const void *v,
                                       kda_dtype_t dt, const float *log_alpha,
                                       const float *beta, const float *S0,
                                       const int32_t *cu_seqlens, int n_seqs, int B, int T,
                                       int H, int dk, int dv, float scale, void *o,
                                       float *S_final, void *workspace, size_t workspace_bytes,
                                       int algo, void *stream)
{
    return chunk_fwd_phases(KDA_CHUNK_ARGS, algo, kda::kPhasePrepare, 0, stream);
}

kda_status_t kda_chunk_fwd_prepare(const void *q, const void *k, const void *v, kda_dtype_t dt,
                                   const float *log_alpha, const float *beta, const float *S0,
                                   const int32_t *cu_seqlens, int n_seqs, int B, int T, int H,
                                   int dk, int dv, float scale, void *o, float *S_final,
                                   void *workspace, size_t workspace_bytes, int algo,
                                   void *stream)
{
    return chunk_fwd_phases(KDA_CHUNK_ARGS, algo, kda::kPhasePrepare, 1, stream);
}

kda_status_t kda_chunk_fwd_carry(const void *q, const void *k, const void *v, kda_dtype_t dt,
                                 const float *log_alpha, const float *beta, const float *S0,
                                 const int32_t *cu_seqlens, int n_seqs, int B, int T, int H,
                                 int dk, int dv, float scale, void *o, float *S_final,
                                 void *workspace, size_t workspace_bytes, int algo, void *stream)
{
    return chunk_fwd_phases(KDA_CHUNK_ARGS, algo, kda::kPhaseCarry, 1, stream);
}

kda_status_t kda_chunk_fwd_timesplit(const void *q, const void *k, const void *v,
                                     kda_dtype_t dt, const float *log_alpha, const float *beta,
                                     const float *S0, const int32_t *cu_seqlens, int n_seqs,
                                     int B, int T, int H, int dk, int dv, float scale, void *o,
                                     float *S_final, void *workspace, size_t workspace_bytes,
                                     int segments, void *stream)
{
    if (segments < 0 || segments > kda::kMaxSegments) return KDA_ERR_INVALID_ARG;
    const int algo = segments == 0 ? KDA_ALGO_TCGEN05 : kAlgoSegmentsBase + segments;
    return chunk_fwd_phases(KDA_CHUNK_ARGS, algo, kda::kPhaseAll, 1, stream);
}

kda_status_t kda_chunk_fwd(const void *q, const void *k, const void *v, kda_dtype_t dt,
                           const float *log_alpha, const float *beta, const float *S0,
                           const int32_t *cu_seqlens, int n_seqs, int B, int T, int H,
                           int dk, int dv, float scale, void *o, float *S_final,
                           void *workspace, size_t workspace_bytes, void *stream)
{
    return kda_chunk_fwd_ex(q, k, v, dt, log_alpha, beta, S0, cu_seqlens, n_seqs, B, T, H,
                            dk, dv, scale, o, S_final, workspace, workspace_bytes,
                            KDA_ALGO_AUTO, stream);
}

}  // extern "C"

// The backward algorithm AUTO stands for: the chunk-parallel form (faster than
// the token walk on long sequences, with a smaller workspace).
static bool bwd_chunked(int algo) { return algo != KDA_BWD_TOKEN; }

static kda_status_t chunk_bwd(const void *q, const void *k, const void *v, kda_dtype_t dt,
                              const float *log_alpha, const float *beta, const float *S0,
                              const int32_t *cu_seqlens, int n_seqs, int B, int T, int H,
                              int dk, int dv, float scale, const void *dO,
                              const float *dS_final, float *grad_q, float *grad_k,
                              float *grad_v, float *grad_log_alpha, float *grad_beta,
                              float *grad_S0, void *workspace, size_t workspace_bytes,
                              int gate_per_channel, int algo, void *stream)
{
    if (algo != KDA_BWD_AUTO && algo != KDA_BWD_TOKEN && algo != KDA_BWD_CHUNKED)
        return KDA_ERR_INVALID_ARG;
    kda::Problem p;
    kda_status_t st = describe(B, T, H, dk, dv, n_seqs, cu_seqlens != nullptr, dt, &p);
    if (st != KDA_OK) return st;
    if (!isfinite(scale)) return KDA_ERR_INVALID_ARG;
    if (p.total_tokens > 0 && (!q || !k || !v || !log_alpha || !beta || !dO || !grad_q ||
                               !grad_k || !grad_v || !grad_log_alpha || !grad_beta))
        return KDA_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, log_alpha, beta, S0, dO, dS_final, grad_q, grad_k, grad_v,
                          grad_log_alpha, grad_beta, grad_S0, workspace};
    for (const void *ptr : ptrs)
        if (!aligned16(ptr)) return KDA_ERR_ALIGNMENT;
    if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return KDA_ERR_ALIGNMENT;
    const bool chunked = bwd_chunked(algo);
    const size_t need = chunked ? kda::cbwd_workspace_bytes(p) : kda::bwd_workspace_layout(p).total;
    if (!workspace || workspace_bytes < need) return KDA_ERR_WORKSPACE;
    p.q = q; p.k = k; p.v = v; p.log_alpha = log_alpha; p.beta = beta; p.S0 = S0;
    p.cu_seqlens = cu_seqlens; p.scale = scale; p.gate_per_channel = gate_per_channel;
    const cudaError_t e =
        chunked ? kda::launch_backward_chunked(p, dO, dS_final, grad_q, grad_k, grad_v,
                                               grad_log_alpha, grad_beta, grad_S0, workspace,
                                               static_cast<cudaStream_t>(stream))
                : kda::launch_backward(p, dO, dS_final, grad_q, grad_k, grad_v, grad_log_alpha,
                                       grad_beta, grad_S0, workspace,
                                       static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

extern "C" {

size_t kda_chunk_bwd_workspace_size_ex(int B, int T, int H, int dk, int dv, int n_seqs,
                                       kda_dtype_t dt, int algo)
{
    if (algo != KDA_BWD_AUTO && algo != KDA_BWD_TOKEN && algo != KDA_BWD_CHUNKED) return 0;
    kda::Problem p;
    const bool varlen = n_seqs > 0 && B == 1;
    if (describe(B, T, H, dk, dv, n_seqs, varlen, dt, &p) != KDA_OK) return 0;
    return bwd_chunked(algo) ? kda::cbwd_workspace_bytes(p) : kda::bwd_workspace_layout(p).total;
}

size_t kda_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv, int n_seqs,
                                    kda_dtype_t dt)
{
    return kda_chunk_bwd_workspace_size_ex(B, T, H, dk, dv, n_seqs, dt, KDA_BWD_AUTO);
}

#define KDA_BWD_ARGS q, k, v, dt, log_alpha, beta, S0, cu_seqlens, n_seqs, B, T, H, dk, dv, \
    scale, dO, dS_final, grad_q, grad_k, grad_v, grad_log_alpha, grad_beta, grad_S0, \
    workspace, workspace_bytes

kda_status_t kda_chunk_bwd(const void *q, const void *k, const void *v, kda_dtype_t dt,
                           const float *log_alpha, const float *beta, const float *S0,
                           const int32_t *cu_seqlens, int n_seqs, int B, int T, int H, int dk,
                           int dv, float scale, const void *dO, const float *dS_final,
                           float *grad_q, float *grad_k, float *grad_v, float *grad_log_alpha,
                           float *grad_beta, float *grad_S0, void *workspace,
                           size_t workspace_bytes, void *stream)
{
    return chunk_bwd(KDA_BWD_ARGS, 1, KDA_BWD_AUTO, stream);
}

kda_status_t kda_gdn_chunk_bwd(const void *q, const void *k, const void *v, kda_dtype_t dt,
                               const float *log_alpha, const float *beta, const float *S0,
                               const int32_t *cu_seqlens, int n_seqs, int B, int T, int H,
                               int dk, int dv, float scale, const void *dO,
                               const float *dS_final, float *grad_q, float *grad_k,
                               float *grad_v, float *grad_log_alpha, float *grad_beta,
                               float *grad_S0, void *workspace, size_t workspace_bytes,
                               void *stream)
{
    return chunk_bwd(KDA_BWD_ARGS, 0, KDA_BWD_AUTO, stream);
}

kda_status_t kda_chunk_bwd_ex(const void *q, const void *k, const void *v, kda_dtype_t dt,
                              const float *log_alpha, const float *beta, const float *S0,
                              const int32_t *cu_seqlens, int n_seqs, int B, int T, int H,
                              int dk, int dv, float scale, const void *dO,
                              const float *dS_final, float *grad_q, float *grad_k,
                              float *grad_v, float *grad_log_alpha, float *grad_beta,
                              float *grad_S0, void *workspace, size_t workspace_bytes,
                              int gate_per_channel, int algo, void *stream)
{
    return chunk_bwd(KDA_BWD_ARGS, gate_per_channel ? 1 : 0, algo, stream);
}

}  // extern "C"

static kda_status_t decode_tokens(const void *q, const void *k, const void *v, kda_dtype_t dt,
                                  const float *log_alpha, const float *beta, float *S, int N,
                                  int T, int H, int dk, int dv, float scale, void *o,
                                  int gate_per_channel, void *stream)
{
    if (N < 1 || T < 0 || H < 1 || dk < 1 || dv < 1) return KDA_ERR_INVALID_ARG;
    if (!dtype_ok(dt) || !head_ok(dk, dv)) return KDA_ERR_UNSUPPORTED;
    if ((long long)N * H > (long long)INT32_MAX) return KDA_ERR_UNSUPPORTED;
    if ((long long)N * T > (long long)INT32_MAX) return KDA_ERR_UNSUPPORTED;
    if (!isfinite(scale)) return KDA_ERR_INVALID_ARG;
    if (!S) return KDA_ERR_INVALID_ARG;
    if (T == 0) return KDA_OK;  // no token: S unchanged, nothing launched
    if (!q || !k || !v || !log_alpha || !beta || !o) return KDA_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, log_alpha, beta, S, o};
    for (const void *ptr : ptrs)
        if (!aligned16(ptr)) return KDA_ERR_ALIGNMENT;
    const cudaError_t e = kda::launch_decode(q, k, v, dt, log_alpha, beta, S, N, T, H, dk, dv,
                                             scale, o, gate_per_channel,
                                             static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

extern "C" {

kda_status_t kda_decode_tokens(const void *q, const void *k, const void *v, kda_dtype_t dt,
                               const float *log_alpha, const float *beta, float *S, int N,
                               int T, int H, int dk, int dv, float scale, void *o,
                               void *stream)
{
    return decode_tokens(q, k, v, dt, log_alpha, beta, S, N, T, H, dk, dv, scale, o, 1, stream);
}

kda_status_t kda_gdn_decode_tokens(const void *q, const void *k, const void *v, kda_dtype_t dt,
                                   const float *log_alpha, const float *beta, float *S, int N,
                                   int T, int H, int dk, int dv, float scale, void *o,
                                   void *stream)
{
    return decode_tokens(q, k, v, dt, log_alpha, beta, S, N, T, H, dk, dv, scale, o, 0, stream);
}

kda_status_t kda_decode_step(const void *q, const void *k, const void *v, kda_dtype_t dt,
                             const float *log_alpha, const float *beta, float *S, int N,
                             int H, int dk, int dv, float scale, void *o, void *stream)
{
    return kda_decode_tokens(q, k, v, dt, log_alpha, beta, S, N, 1, H, dk, dv, scale, o,
                             stream);
}

}  // extern "C"
