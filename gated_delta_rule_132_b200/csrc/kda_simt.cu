// kda_simt.cu — chunked KDA prefill on CUDA cores in fp32 (any supported size).
//
// Source: the KDA update rule of "Kimi Linear：让长上下文大模型真正实用的线性注意力架构"
// (juejin.cn), section 三 5️⃣, S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1}
// + beta_t k_t v_t^T, with the per-channel gate of section 三 1️⃣ and the read-out
// o_t = scale * S_t^T q_t. The pages only say that the chunked (DPLR) form runs
// chunk-parallel (section 三 2️⃣); the chunked form below is derived from the
// rule itself and is exact.
//
// Chunked form. In a chunk of C tokens with entry state S_0, let g_r be the
// inclusive cumulative sum of log_alpha over the chunk's tokens (per channel),
// K~_r = e^{g_r} * k_r, Q~_r = e^{g_r} * q_r, K^_s = e^{g_C - g_s} * k_s. Unrolling
// the rule gives S_r = Diag(e^{g_r}) S_0 + sum_{s<=r} Diag(e^{g_r - g_s}) k_s u_s^T
// with u_r = beta_r (v_r - S'_r^T k_r), which is the unit-lower-triangular system
//     (I + A) U = Diag(beta) (V - K~ S_0),  A_rs = beta_r k_r^T Diag(e^{g_r-g_s}) k_s  (s < r).
// With X = (I + A)^{-1} Diag(beta) [K~ | V] = [W | U~]:
//     U   = U~ - W S_0
//     O   = scale * (Q~ S_0 + P U),   P_rs = q_r^T Diag(e^{g_r - g_s}) k_s  (s <= r)
//     S_C = Diag(e^{g_C}) S_0 + K^^T U.
// A tail chunk is padded with tokens that have k = q = v = 0, beta = 0 and
// log_alpha = 0: identity transitions that change nothing.
//
// Two kernels. prep (one CTA per chunk and head, all chunks in parallel)
// computes g, A, P, solves for W and U~ by forward substitution and stores
// W, U~, Q~, K^, P and gamma = e^{g_C} in the workspace. carry (one CTA per
// sequence, head and 32-column slice of the value dimension — the value
// columns of S never mix) walks the chunks in order with its slice of S in
// shared memory and writes o and S_final. This path computes every exponent
// of a difference exactly as exp(g_r - g_s), so it is valid for any gate.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int C = kChunk;
constexpr int kSimtThreads = 256;

struct SimtParams {
    const void *q, *k, *v;
    const float *log_alpha, *beta, *S0;
    int N, H;
    int gate_per_channel;  // log_alpha [.., H, D] (1) or [.., H] (0)
    float scale;
    void *o;
    float *S_final;
    const int32_t *seq_start, *chunk_off, *order;
    float *ws;  // per-chunk intermediates
};

// Floats per (chunk, head) in the workspace: W, U~, Q~, K^ (C x D each),
// P (C x C) and gamma (D).
template <int D> constexpr size_t simt_chunk_floats() { return 4 * C * D + C * C + D; }

template <int D>
__device__ __forceinline__ float *chunk_ptr(float *ws, int c, int h, int H)
{
    return ws + ((size_t)c * H + h) * simt_chunk_floats<D>();
}

// Locate global chunk c: returns the sequence n (or -1 when c is past the end).
__device__ __forceinline__ int find_seq(const int32_t *chunk_off, int N, int c)
{
    if (c >= chunk_off[N]) return -1;
    int lo = 0, hi = N - 1;  // largest n with chunk_off[n] <= c
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (chunk_off[mid] <= c) lo = mid; else hi = mid - 1;
    }
    return lo;
}

template <int D, typename TIn>
__global__ void __launch_bounds__(kSimtThreads, 1) simt_prep_kernel(SimtParams p)
{
    constexpr int DP = D + 1;  // padded row stride: lanes walking rows hit distinct banks
    extern __shared__ float smem[];
    float *sk = smem;               // [C][DP]  k, later beta*K~, later W
    float *sq = sk + C * DP;        // [C][DP]  q
    float *sg = sq + C * DP;        // [C][DP]  log_alpha, then g
    float *sv = sg + C * DP;        // [C][D]   v, later beta*V, later U~
    float *sA = sv + C * D;         // [C][C+1]
    float *sb = sA + C * (C + 1);   // [C]

    const int c = blockIdx.x, h = blockIdx.y, H = p.H;
    const int n = find_seq(p.chunk_off, p.N, c);
    if (n < 0) return;
    const int t0 = p.seq_start[n] + (c - p.chunk_off[n]) * C;
    const int L = min(C, p.seq_start[n + 1] - t0);
    const int tid = threadIdx.x;

    const TIn *q = static_cast<const TIn *>(p.q);
    const TIn *k = static_cast<const TIn *>(p.k);
    const TIn *v = static_cast<const TIn *>(p.v);
    for (int idx = tid; idx < C * D; idx += kSimtThreads) {
        const int r = idx / D, i = idx % D;
        float kq = 0.f, qq = 0.f, vv = 0.f, la = 0.f;
        if (r < L) {
            const size_t off = ((size_t)(t0 + r) * H + h) * D + i;
            kq = to_f32(k[off]); qq = to_f32(q[off]); vv = to_f32(v[off]);
            la = p.gate_per_channel ? p.log_alpha[off] : p.log_alpha[(size_t)(t0 + r) * H + h];
        }
        sk[r * DP + i] = kq; sq[r * DP + i] = qq; sv[r * D + i] = vv; sg[r * DP + i] = la;
    }
    for (int r = tid; r < C; r += kSimtThreads)
        sb[r] = r < L ? p.beta[(size_t)(t0 + r) * H + h] : 0.f;
    __syncthreads();
    // g: inclusive cumulative sum over the chunk, one thread per channel.
    for (int i = tid; i < D; i += kSimtThreads) {
        float g = 0.f;
        for (int r = 0; r < C; ++r) { g += sg[r * DP + i]; sg[r * DP + i] = g; }
    }
    __syncthreads();

    float *w = chunk_ptr<D>(p.ws, c, h, H);
    float *wW = w, *wU = w + C * D, *wQ = w + 2 * C * D, *wK = w + 3 * C * D;
    float *wP = w + 4 * C * D, *wG = wP + C * C;

    // A (strictly lower, beta-scaled) and P (lower incl. diagonal): one warp per
    // row, one lane per column, exact exp of every gate difference.
    const int warp = tid >> 5, lane = tid & 31;
    for (int r = warp; r < C; r += kSimtThreads / 32) {
        for (int s = lane; s < C; s += 32) {
            float akk = 0.f, pqk = 0.f;
            if (s <= r) {
                for (int i = 0; i < D; ++i) {
                    const float e = expf(sg[r * DP + i] - sg[s * DP + i]);
                    const float ke = sk[s * DP + i] * e;
                    akk += sk[r * DP + i] * ke;
                    pqk += sq[r * DP + i] * ke;
                }
            }
            sA[r * (C + 1) + s] = (s < r) ? sb[r] * akk : 0.f;
            wP[r * C + s] = pqk;
        }
    }
    // Q~, K^ and gamma (these read sk, which is overwritten below).
    for (int idx = tid; idx < C * D; idx += kSimtThreads) {
        const int r = idx / D, i = idx % D;
        const float g = sg[r * DP + i], gC = sg[(C - 1) * DP + i];
        wQ[idx] = expf(g) * sq[r * DP + i];
        wK[idx] = expf(gC - g) * sk[r * DP + i];
    }
    for (int i = tid; i < D; i += kSimtThreads) wG[i] = expf(sg[(C - 1) * DP + i]);
    __syncthreads();
    // Right-hand side Diag(beta) [K~ | V], in place.
    for (int idx = tid; idx < C * D; idx += kSimtThreads) {
        const int r = idx / D, i = idx % D;
        sk[r * DP + i] *= sb[r] * expf(sg[r * DP + i]);
        sv[r * D + i] *= sb[r];
    }
    __syncthreads();
    // Forward substitution, one thread per right-hand-side column:
    // X_r = B_r - sum_{s<r} A_rs X_s.
    for (int col = tid; col < 2 * D; col += kSimtThreads) {
        float *x = col < D ? sk + col : sv + (col - D);
        const int stride = col < D ? DP : D;
        for (int r = 1; r < C; ++r) {
            float acc = x[r * stride];
            for (int s = 0; s < r; ++s) acc -= sA[r * (C + 1) + s] * x[s * stride];
            x[r * stride] = acc;
        }
    }
    __syncthreads();
    for (int idx = tid; idx < C * D; idx += kSimtThreads) {
        const int r = idx / D, i = idx % D;
        wW[idx] = sk[r * DP + i];
        wU[idx] = sv[idx];
    }
}

template <int D, typename TIn>
__global__ void __launch_bounds__(kSimtThreads, 1) simt_carry_kernel(SimtParams p)
{
    constexpr int WV = kSimtSlice;
    extern __shared__ float smem[];
    float *sW = smem;            // [C][D]
    float *sQ = sW + C * D;      // [C][D]
    float *sK = sQ + C * D;      // [C][D]
    float *sP = sK + C * D;      // [C][C]
    float *sUt = sP + C * C;     // [C][WV]  U~ slice
    float *sU = sUt + C * WV;    // [C][WV]  U slice
    float *sS = sU + C * WV;     // [D][WV]  state slice
    float *sG = sS + D * WV;     // [D]

    // one CTA per (sequence, head, slice), sequences longest first
    constexpr int kSlices = D / WV;
    const int H = p.H;
    const int j0 = (blockIdx.x % kSlices) * WV;
    const int h = (blockIdx.x / kSlices) % H;
    const int n = p.order[blockIdx.x / (kSlices * H)];
    const int tid = threadIdx.x, j = tid % WV, grp = tid / WV;  // 8 groups
    constexpr int NG = kSimtThreads / WV;
    const size_t sbase = ((size_t)n * H + h) * D * D;

    for (int idx = tid; idx < D * WV; idx += kSimtThreads) {
        const int i = idx / WV, jj = idx % WV;
        sS[idx] = p.S0 ? p.S0[sbase + (size_t)i * D + j0 + jj] : 0.f;
    }
    const int ts = p.seq_start[n], te = p.seq_start[n + 1];
    const int c0 = p.chunk_off[n], nc = p.chunk_off[n + 1] - c0;
    TIn *o = static_cast<TIn *>(p.o);

    for (int lc = 0; lc < nc; ++lc) {
        const float *w = chunk_ptr<D>(p.ws, c0 + lc, h, H);
        const int t0 = ts + lc * C;
        const int L = min(C, te - t0);
        __syncthreads();  // previous chunk finished with the buffers
        for (int idx = tid; idx < C * D / 4; idx += kSimtThreads) {
            reinterpret_cast<float4 *>(sW)[idx] = reinterpret_cast<const float4 *>(w)[idx];
            reinterpret_cast<float4 *>(sQ)[idx] = reinterpret_cast<const float4 *>(w + 2 * C * D)[idx];
            reinterpret_cast<float4 *>(sK)[idx] = reinterpret_cast<const float4 *>(w + 3 * C * D)[idx];
        }
        for (int idx = tid; idx < C * C / 4; idx += kSimtThreads)
            reinterpret_cast<float4 *>(sP)[idx] = reinterpret_cast<const float4 *>(w + 4 * C * D)[idx];
        for (int idx = tid; idx < C * WV; idx += kSimtThreads) {
            const int r = idx / WV, jj = idx % WV;
            sUt[idx] = w[C * D + r * D + j0 + jj];
        }
        for (int i = tid; i < D; i += kSimtThreads) sG[i] = w[4 * C * D + C * C + i];
        __syncthreads();
        // U = U~ - W S and Oq = Q~ S for rows grp, grp+NG, ...
        float oq[C / NG];
#pragma unroll
        for (int rr = 0; rr < C / NG; ++rr) {
            const int r = rr * NG + grp;
            float ws = 0.f, qs = 0.f;
            for (int i = 0; i < D; ++i) {
                const float s = sS[i * WV + j];
                ws += sW[r * D + i] * s;
                qs += sQ[r * D + i] * s;
            }
            sU[r * WV + j] = sUt[r * WV + j] - ws;
            oq[rr] = qs;
        }
        __syncthreads();
        // O = scale (Q~ S + P U)
#pragma unroll
        for (int rr = 0; rr < C / NG; ++rr) {
            const int r = rr * NG + grp;
            float acc = oq[rr];
            for (int s = 0; s <= r; ++s) acc += sP[r * C + s] * sU[s * WV + j];
            if (r < L) o[((size_t)(t0 + r) * H + h) * D + j0 + j] = from_f32<TIn>(p.scale * acc);
        }
        // S = Diag(gamma) S + K^^T U (each thread owns rows grp, grp+NG, ... of column j)
        for (int i = grp; i < D; i += NG) {
            float acc = sG[i] * sS[i * WV + j];
            for (int r = 0; r < C; ++r) acc += sK[r * D + i] * sU[r * WV + j];
            sS[i * WV + j] = acc;
        }
    }
    __syncthreads();
    if (p.S_final) {
        for (int idx = tid; idx < D * WV; idx += kSimtThreads) {
            const int i = idx / WV, jj = idx % WV;
            p.S_final[sbase + (size_t)i * D + j0 + jj] = sS[idx];
        }
    }
}

template <int D> constexpr size_t prep_smem() { return sizeof(float) * (3 * C * (D + 1) + C * D + C * (C + 1) + C); }
template <int D> constexpr size_t carry_smem() {
    return sizeof(float) * (3 * C * D + C * C + 2 * C * kSimtSlice + D * kSimtSlice + D);
}

template <int D, typename TIn>
cudaError_t launch_simt_d(const Problem &pb, void *workspace, int phases, cudaStream_t st)
{
    const WorkspaceLayout lay = simt_workspace_layout(pb);
    SimtParams p;
    p.q = pb.q; p.k = pb.k; p.v = pb.v;
    p.log_alpha = pb.log_alpha; p.beta = pb.beta; p.S0 = pb.S0;
    p.N = pb.N; p.H = pb.H; p.scale = pb.scale; p.o = pb.o; p.S_final = pb.S_final;
    p.gate_per_channel = pb.gate_per_channel;
    Plan plan;
    plan.seq_start = reinterpret_cast<int32_t *>(static_cast<char *>(workspace) + kWsHeader);
    plan.chunk_off = plan.seq_start + (pb.N + 1);
    plan.order = plan.chunk_off + (pb.N + 1);
    p.seq_start = plan.seq_start; p.chunk_off = plan.chunk_off; p.order = plan.order;
    p.ws = reinterpret_cast<float *>(static_cast<char *>(workspace) + lay.plan_bytes);

    cudaError_t e;
    auto prep = simt_prep_kernel<D, TIn>;
    auto carry = simt_carry_kernel<D, TIn>;
    e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)prep_smem<D>());
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(carry, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)carry_smem<D>());
    if (e != cudaSuccess) return e;
    if (phases & kPhasePrepare) {
        // the status word: this path has no bounded waits, so it stays 0
        e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
        if (e != cudaSuccess) return e;
        e = launch_plan(pb, plan, st);
        if (e != cudaSuccess) return e;
        if (pb.max_chunks > 0) {
            prep<<<dim3(pb.max_chunks, pb.H), kSimtThreads, prep_smem<D>(), st>>>(p);
            note_launch();
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
    }
    if (phases & kPhaseCarry) {
        carry<<<(unsigned)(pb.N * pb.H * (D / kSimtSlice)), kSimtThreads, carry_smem<D>(), st>>>(p);
        note_launch();
        e = cudaGetLastError();
    }
    return e;
}

template <typename TIn>
cudaError_t launch_simt_t(const Problem &p, void *ws, int ph, cudaStream_t st)
{
    switch (p.dk) {
    case 32: return launch_simt_d<32, TIn>(p, ws, ph, st);
    case 64: return launch_simt_d<64, TIn>(p, ws, ph, st);
    case 128: return launch_simt_d<128, TIn>(p, ws, ph, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

WorkspaceLayout simt_workspace_layout(const Problem &p)
{
    WorkspaceLayout l;
    l.plan_bytes = kWsHeader + align_up(sizeof(int32_t) * plan_ints(p.N), 256);
    const size_t D = (size_t)p.dk;
    l.chunk_bytes = sizeof(float) * (4 * C * D + C * C + D) * (size_t)p.H * (size_t)p.max_chunks;
    l.total = l.plan_bytes + l.chunk_bytes;
    return l;
}

cudaError_t launch_simt_prefill(const Problem &p, void *workspace, int phases,
                                cudaStream_t stream)
{
    if (p.dtype == KDA_DTYPE_BF16)
        return launch_simt_t<__nv_bfloat16>(p, workspace, phases, stream);
    return launch_simt_t<float>(p, workspace, phases, stream);
}

}  // namespace kda
