// kda_internal.cuh — declarations shared by the library's translation units.
// Nothing here is part of the public C ABI (include/kda.h is).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "kda.h"

namespace kda {

// Chunk length of the chunked prefill (tokens per chunk).
constexpr int kChunk = 64;
// Width of the value-column slice one sequential-carry CTA owns on the SIMT path.
constexpr int kSimtSlice = 32;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Problem description after host-side validation.
struct Problem {
    const void *q, *k, *v;
    const float *log_alpha, *beta, *S0;
    const int32_t *cu_seqlens;  // device, or null (uniform sequences of length T)
    int N;                      // number of sequences
    int B, T, H, dk, dv;
    float scale;
    void *o;
    float *S_final;
    kda_dtype_t dtype;
    long long total_tokens;     // B * T (packed time axis length)
    int max_chunks;             // upper bound on chunks over all sequences
    int gate_per_channel;       // 1: log_alpha [.., H, dk] (KDA); 0: [.., H] (one gate per head)
    int nseg;                   // tensor-core path: time segments of the sequential phase (1: none)
};

// Most time segments the tensor-core path splits a sequence into.
constexpr int kMaxSegments = 64;

// Sequence plan in the workspace: for n in [0, N], the sanitised packed start
// token seq_start[n] and first global chunk chunk_off[n] (both int32; entry N
// holds the totals), and order[0..N): the sequences by decreasing length, the
// order in which the sequential kernels take them (longest first keeps the
// last wave of CTAs short).
struct Plan {
    int32_t *seq_start;
    int32_t *chunk_off;
    int32_t *order;
};

// int32 entries of a plan for N sequences.
inline size_t plan_ints(int N) { return 3 * (size_t)N + 2; }

// Every prefill workspace starts with a header of kWsHeader bytes:
//   int32 [0]  device status word: 0, or the code of the first bounded wait
//              that ran out (cleared by the prepare phase; kda_chunk_fwd_status
//              reads it)
//   int32 [1]  tensor-core path: number of chunks listed for the exact fixup
// The plan follows the header.
constexpr size_t kWsHeader = 256;

// Process-wide debugging settings (kda_debug_set_wait_limit): the poll limit
// of every bounded wait in the tensor-core kernels (0: the default), and
// whether the sequential kernel's producer issues no copies, so that its
// first wait on a record runs out with nothing asynchronous in flight.
struct DebugKnobs {
    uint32_t wait_limit;
    int starve_carry;
};
DebugKnobs debug_knobs();

// Counts one kernel launch of this library (kda_launch_count reads the total).
void note_launch();

// Byte layout of one prefill workspace.
struct WorkspaceLayout {
    size_t plan_bytes;      // seq_start + chunk_off
    size_t chunk_bytes;     // per-chunk intermediates, all heads
    size_t total;
};

WorkspaceLayout simt_workspace_layout(const Problem &p);
WorkspaceLayout tc_workspace_layout(const Problem &p);

cudaError_t launch_plan(const Problem &p, Plan plan, cudaStream_t stream);
// T tokens per (sequence, head): q, k, log_alpha [N, T, H, dk], v, o [N, T, H, dv],
// beta [N, T, H]; S [N, H, dk, dv] read once and written once.
// gate_per_channel: log_alpha [N, T, H, dk] (1) or [N, T, H] (0).
cudaError_t launch_decode(const void *q, const void *k, const void *v, kda_dtype_t dt,
                          const float *log_alpha, const float *beta, float *S, int N, int T,
                          int H, int dk, int dv, float scale, void *o, int gate_per_channel,
                          cudaStream_t stream);
// Prefill phases: bit 0 = prepare (plan + chunk-parallel kernel), bit 1 = carry.
enum : int { kPhasePrepare = 1, kPhaseCarry = 2, kPhaseAll = 3 };
cudaError_t launch_simt_prefill(const Problem &p, void *workspace, int phases,
                                cudaStream_t stream);
cudaError_t launch_tc_prefill(const Problem &p, void *workspace, int phases,
                              cudaStream_t stream);
bool tc_supported(const Problem &p);
// Time segments the tensor-core path uses for this problem when left to choose.
int tc_auto_segments(const Problem &p);
// Backward of the prefill (fp32 CUDA cores): gradients of <dO, o> + <dS_final, S_final>.
WorkspaceLayout bwd_workspace_layout(const Problem &p);
cudaError_t launch_backward(const Problem &p, const void *dO, const float *dS_final,
                            float *gq, float *gk, float *gv, float *gla, float *gbeta,
                            float *gS0, void *workspace, cudaStream_t stream);

// Chunk-parallel backward (fp32 CUDA cores): per-chunk records, a forward and a
// reverse walk over the chunks, then the token gradients of all chunks at once.
size_t cbwd_workspace_bytes(const Problem &p);
cudaError_t launch_backward_chunked(const Problem &p, const void *dO, const float *dS_final,
                                    float *gq, float *gk, float *gv, float *gla, float *gbeta,
                                    float *gS0, void *workspace, cudaStream_t stream);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace kda
