// kda_plan.cu — the variable-length sequence plan shared by both prefill paths.
//
// Sequences are packed along one time axis. The plan maps every global chunk
// index to its sequence: seq_start[n] is the first packed token of sequence n
// and chunk_off[n] its first global chunk (ceil(len / 64) chunks per sequence;
// the last one may be partial). Entry N of each array holds the totals.
//
// cu_seqlens lives in device memory, so the host cannot check it without a
// synchronisation. The plan therefore sanitises it on the device: offsets are
// clamped to [0, total_tokens] and made non-decreasing with a running maximum.
// For well-formed input this changes nothing; for malformed input it keeps
// every later access inside the caller's buffers and the chunk count within
// floor(total / 64) + N, the bound the workspace is sized for.
//
// It also ranks the sequences by decreasing length (ties by index): the
// sequential kernels take them in that order, so the longest sequences start
// in the first wave of CTAs. Ranking is quadratic, so it is done for up to
// kRankMax sequences; beyond that the order is the identity.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kPlanThreads = 1024;
constexpr int kRankMax = 2048;

template <typename Op>
__device__ int block_inclusive_scan(int x, Op op, int identity, int *s_warp)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x = op(x, y);
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = (lane < kPlanThreads / 32) ? s_warp[lane] : identity;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w = op(w, y);
        }
        s_warp[lane] = w;
    }
    __syncthreads();
    if (warp > 0) x = op(x, s_warp[warp - 1]);
    __syncthreads();
    return x;
}

struct MaxOp { __device__ int operator()(int a, int b) const { return a > b ? a : b; } };
struct AddOp { __device__ int operator()(int a, int b) const { return a + b; } };

__global__ void __launch_bounds__(kPlanThreads)
plan_kernel(const int32_t *__restrict__ cu_seqlens, int N, int T, int total,
            int32_t *__restrict__ seq_start, int32_t *__restrict__ chunk_off,
            int32_t *__restrict__ order)
{
    __shared__ int s_warp[32];
    __shared__ int s_carry;
    __shared__ int s_len[kRankMax];
    if (cu_seqlens == nullptr) {
        const int per = (T + kChunk - 1) / kChunk;
        for (int n = threadIdx.x; n <= N; n += kPlanThreads) {
            seq_start[n] = n * T;
            chunk_off[n] = n * per;
            if (n < N) order[n] = n;
        }
        return;
    }
    // Pass 1: running maximum of the clamped offsets.
    if (threadIdx.x == 0) s_carry = 0;
    __syncthreads();
    for (int base = 0; base <= N; base += kPlanThreads) {
        const int n = base + threadIdx.x;
        int x = 0;
        if (n <= N) x = min(max(cu_seqlens[n], 0), total);
        x = max(x, s_carry);
        x = block_inclusive_scan(x, MaxOp(), 0, s_warp);
        if (n <= N) seq_start[n] = x;
        if (threadIdx.x == kPlanThreads - 1) s_carry = x;
        __syncthreads();
    }
    // Pass 2: exclusive prefix sum of the per-sequence chunk counts.
    if (threadIdx.x == 0) s_carry = 0;
    __syncthreads();
    for (int base = 0; base <= N; base += kPlanThreads) {
        const int n = base + threadIdx.x;
        int c = 0;
        if (n < N) c = (seq_start[n + 1] - seq_start[n] + kChunk - 1) / kChunk;
        const int incl = block_inclusive_scan(c, AddOp(), 0, s_warp);
        const int carry = s_carry;
        if (n <= N) chunk_off[n] = carry + incl - c;
        __syncthreads();
        if (threadIdx.x == kPlanThreads - 1) s_carry = carry + incl;
        __syncthreads();
    }
    // Pass 3: longest-first order.
    if (N > kRankMax) {
        for (int n = threadIdx.x; n < N; n += kPlanThreads) order[n] = n;
        return;
    }
    for (int n = threadIdx.x; n < N; n += kPlanThreads) s_len[n] = seq_start[n + 1] - seq_start[n];
    __syncthreads();
    for (int n = threadIdx.x; n < N; n += kPlanThreads) {
        const int ln = s_len[n];
        int rank = 0;
        for (int m = 0; m < N; ++m) {
            const int lm = s_len[m];
            rank += (lm > ln) || (lm == ln && m < n);
        }
        order[rank] = n;
    }
}

}  // namespace

cudaError_t launch_plan(const Problem &p, Plan plan, cudaStream_t stream)
{
    plan_kernel<<<1, kPlanThreads, 0, stream>>>(p.cu_seqlens, p.N, p.T, (int)p.total_tokens,
                                                plan.seq_start, plan.chunk_off, plan.order);
    note_launch();
    return cudaGetLastError();
}

}  // namespace kda
