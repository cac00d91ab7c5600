// kda_bwd.cu — reverse-mode derivatives of the chunked prefill (fp32 CUDA cores).
//
// Source: the KDA update rule of "Kimi Linear：让长上下文大模型真正实用的线性注意力架构"
// (juejin.cn), section 三 5️⃣, with the per-channel gate of section 三 1️⃣ and the
// read-out o_t = scale * S_t^T q_t. The page states only the forward rule; this
// file computes the derivatives of
//     L = <dO, o> + <dS_final, S_final>
// with respect to q, k, v, log_alpha, beta and S0 by differentiating each
// token's three steps in reverse order, with G = dL/dS_t the gradient reaching
// the state after token t:
//   read-out  o_t = scale S_t^T q_t:   G += scale q_t dO_t^T,  dq_t = scale S_t dO_t
//   update    S_t = S' + beta k w^T,   w = v - S'^T k:
//             g = G^T k;  dv_t = beta g;  dbeta_t = g . w;
//             dk_t = beta (G w - S' g);  dS' = G - beta k g^T
//   decay     S' = Diag(alpha) S_{t-1}: dlog_alpha_t[i] = sum_j dS'_ij S'_ij;
//             G <- Diag(alpha) dS'
// and dS0 = G once the first token is undone.
//
// One CTA per (sequence, head) with D threads (D = dk = dv): thread i owns row
// i of a matrix in the row phases and column i in the column phases; the two
// state buffers and G sit in shared memory with rows padded to D + 1 floats, so
// row and column sweeps are free of bank conflicts. The states the backward
// needs come from a replay of the forward: a first pass stores the state at
// every 64-token chunk start (per (chunk, head), like the prefill's records);
// each chunk, last to first, is then replayed from its checkpoint into a
// per-(sequence, head) buffer of its 65 states and walked backwards. The walk
// keeps S_t in one buffer and fetches S_{t-1} into the other (float4 loads
// issued before the read-out sweep), applying Diag(alpha) on the fly, so
// S_{t-1} is the next step's S_t unchanged. Plain fp32 loops throughout.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kBwdChunk = 64;  // tokens per checkpoint (= the prefill's chunk)

struct BwdParams {
    const void *q, *k, *v, *dO;
    const float *log_alpha, *beta, *S0, *dS_final;
    int N, H, gate_per_channel;
    float scale;
    float *gq, *gk, *gv, *gla, *gbeta, *gS0;
    const int32_t *seq_start, *chunk_off;
    float *ckpt;  // [chunks][H][D][D]
    float *blk;   // [N * H][kBwdChunk + 1][D][D]
};

template <typename TIn>
__device__ __forceinline__ float ld(const void *p, size_t i)
{
    return to_f32(static_cast<const TIn *>(p)[i]);
}

// Copy between a padded shared matrix [D][D+1] and a dense global one [D][D]
// (consecutive threads take consecutive columns).
template <int D>
__device__ __forceinline__ void store_mat(float *dst, const float *sm)
{
#pragma unroll 4
    for (int e4 = threadIdx.x; e4 < D * D / 4; e4 += D) {
        const int r = (4 * e4) / D, c = (4 * e4) % D;
        const float *x = sm + r * (D + 1) + c;
        reinterpret_cast<float4 *>(dst)[e4] = make_float4(x[0], x[1], x[2], x[3]);
    }
}

// Global -> registers (D / 4 float4 per thread, all in flight), then -> shared.
template <int D>
__device__ __forceinline__ void fetch_mat(float4 *reg, const float *src)
{
#pragma unroll
    for (int m = 0; m < D / 4; ++m) reg[m] = reinterpret_cast<const float4 *>(src)[threadIdx.x + D * m];
}

template <int D>
__device__ __forceinline__ void put_mat(float *sm, const float4 *reg)
{
#pragma unroll
    for (int m = 0; m < D / 4; ++m) {
        const int e = 4 * (threadIdx.x + D * m), r = e / D, c = e % D;
        float *x = sm + r * (D + 1) + c;
        x[0] = reg[m].x; x[1] = reg[m].y; x[2] = reg[m].z; x[3] = reg[m].w;
    }
}

template <int D>
__device__ __forceinline__ void load_mat(float *sm, const float *src)
{
    float4 reg[D / 4];
    fetch_mat<D>(reg, src);
    put_mat<D>(sm, reg);
}

template <int D, typename TIn>
__global__ void __launch_bounds__(D) bwd_kernel(BwdParams p)
{
    extern __shared__ float smem[];
    constexpr int P1 = D + 1;
    float *S = smem;             // [D][D+1]: state (forward, replay); S_t or S_{t-1} (backward)
    float *S2 = S + D * P1;      // [D][D+1]: the other of S_t, S_{t-1} (backward)
    float *G = S2 + D * P1;      // [D][D+1]: dL/dS
    float *sk = G + D * P1;      // token vectors
    float *sq = sk + D;
    float *sa = sq + D;          // alpha
    float *sv = sa + D;
    float *sdo = sv + D;
    float *sw = sdo + D;         // w = v - S'^T k
    float *sg = sw + D;          // g = G^T k
    float *sred = sg + D;        // [0, 32): dbeta partials, [32]: beta, [33, 65): gate-sum partials
    float *sred2 = sred + 33;

    const int unit = blockIdx.x, H = p.H;
    const int n = unit / H, h = unit - n * H;
    const int i = threadIdx.x;
    const int t0 = p.seq_start[n], t1 = p.seq_start[n + 1];
    const int c0 = p.chunk_off[n];
    const int nck = (t1 - t0 + kBwdChunk - 1) / kBwdChunk;
    float *blk = p.blk + (size_t)unit * (kBwdChunk + 1) * D * D;

    auto load_token = [&](int t) {  // token vectors of packed token t, then a barrier
        const size_t th = (size_t)t * H + h;
        sk[i] = ld<TIn>(p.k, th * D + i);
        sq[i] = ld<TIn>(p.q, th * D + i);
        sv[i] = ld<TIn>(p.v, th * D + i);
        sdo[i] = ld<TIn>(p.dO, th * D + i);
        sa[i] = expf(p.gate_per_channel ? p.log_alpha[th * D + i] : p.log_alpha[th]);
        if (i == 0) sred[32] = p.beta[th];
        __syncthreads();
    };
    // one forward token on S (row i, then column i, then row i)
    auto fwd_token = [&](int t) {
        load_token(t);
        const float b = sred[32];
        for (int j = 0; j < D; ++j) S[i * P1 + j] *= sa[i];
        __syncthreads();
        float ks = 0.f;
        for (int r = 0; r < D; ++r) ks += sk[r] * S[r * P1 + i];
        sw[i] = sv[i] - ks;  // v - S'^T k
        __syncthreads();
        for (int j = 0; j < D; ++j) S[i * P1 + j] += b * sk[i] * sw[j];
        __syncthreads();
    };

    // 1. forward, keeping the state at every chunk start
    for (int j = 0; j < D; ++j)
        S[i * P1 + j] = p.S0 ? p.S0[((size_t)unit * D + i) * D + j] : 0.f;
    __syncthreads();
    for (int t = t0; t < t1; ++t) {
        if ((t - t0) % kBwdChunk == 0) {
            store_mat<D>(p.ckpt + ((size_t)(c0 + (t - t0) / kBwdChunk) * H + h) * D * D, S);
            __syncthreads();
        }
        fwd_token(t);
    }
    for (int j = 0; j < D; ++j)
        G[i * P1 + j] = p.dS_final ? p.dS_final[((size_t)unit * D + i) * D + j] : 0.f;
    __syncthreads();

    // 2. chunks last to first: replay, then walk backwards
    for (int b = nck - 1; b >= 0; --b) {
        const int a = t0 + b * kBwdChunk, e = min(a + kBwdChunk, t1);
        load_mat<D>(S, p.ckpt + ((size_t)(c0 + b) * H + h) * D * D);
        __syncthreads();
        store_mat<D>(blk, S);
        for (int t = a; t < e; ++t) {
            fwd_token(t);
            store_mat<D>(blk + (size_t)(t - a + 1) * D * D, S);
        }
        __syncthreads();
        // S holds S_e, the state after the block: S_t for t = e - 1
        float *cur = S, *prev = S2;
        for (int t = e - 1; t >= a; --t) {
            const size_t th = (size_t)t * H + h;
            load_token(t);
            const float bt = sred[32];
            float4 reg[D / 4];
            fetch_mat<D>(reg, blk + (size_t)(t - a) * D * D);  // S_{t-1}, in flight
            // read-out with S_t
            {
                float acc = 0.f;
                for (int j = 0; j < D; ++j) {
                    G[i * P1 + j] += p.scale * sq[i] * sdo[j];
                    acc += cur[i * P1 + j] * sdo[j];
                }
                p.gq[th * D + i] = p.scale * acc;
            }
            put_mat<D>(prev, reg);
            __syncthreads();
            // column i: w_i, g_i, dv_i and this column's share of dbeta (S' = Diag(alpha) S_{t-1})
            {
                float ks = 0.f, gk = 0.f;
                for (int r = 0; r < D; ++r) {
                    ks += sa[r] * prev[r * P1 + i] * sk[r];
                    gk += G[r * P1 + i] * sk[r];
                }
                const float w = sv[i] - ks;
                sw[i] = w;
                sg[i] = gk;
                p.gv[th * D + i] = bt * gk;
                float part = gk * w;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
                if ((i & 31) == 0) sred[i >> 5] = part;
            }
            __syncthreads();
            if (i == 0) {
                float db = 0.f;
                for (int q = 0; q < D / 32; ++q) db += sred[q];
                p.gbeta[th] = db;
            }
            // row i: dk_i, dS' row, dlog_alpha_i, then G <- Diag(alpha) dS'
            {
                const float al = sa[i];
                float gw = 0.f, pg = 0.f;
                for (int j = 0; j < D; ++j) {
                    gw += G[i * P1 + j] * sw[j];
                    pg += prev[i * P1 + j] * sg[j];
                }
                p.gk[th * D + i] = bt * (gw - al * pg);
                float dl = 0.f;
                for (int j = 0; j < D; ++j) {
                    const float d = G[i * P1 + j] - bt * sk[i] * sg[j];
                    dl += d * prev[i * P1 + j];
                    G[i * P1 + j] = al * d;
                }
                dl *= al;
                if (p.gate_per_channel) p.gla[th * D + i] = dl;
                else {
                    // one gate per head: its gradient is the sum over the channels
                    float s2 = dl;
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, off);
                    if ((i & 31) == 0) sred2[i >> 5] = s2;
                }
            }
            __syncthreads();
            if (!p.gate_per_channel && i == 0) {
                float s2 = 0.f;
                for (int q = 0; q < D / 32; ++q) s2 += sred2[q];
                p.gla[th] = s2;
            }
            __syncthreads();
            float *tmp = cur; cur = prev; prev = tmp;  // S_{t-1} is the next step's S_t
        }
    }
    if (p.gS0)
        for (int j = 0; j < D; ++j) p.gS0[((size_t)unit * D + i) * D + j] = G[i * P1 + j];
}

template <int D> constexpr size_t bwd_smem() { return sizeof(float) * (3 * D * (D + 1) + 7 * D + 65); }

template <int D, typename TIn>
cudaError_t launch_d(const BwdParams &p, cudaStream_t st)
{
    auto kern = bwd_kernel<D, TIn>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)bwd_smem<D>());
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(p.N * p.H), D, bwd_smem<D>(), st>>>(p);
    return cudaGetLastError();
}

}  // namespace

WorkspaceLayout bwd_workspace_layout(const Problem &pb)
{
    WorkspaceLayout l;
    const size_t dd = (size_t)pb.dk * pb.dk * sizeof(float);
    l.plan_bytes = align_up(sizeof(int32_t) * plan_ints(pb.N), 256);
    const size_t ckpt = align_up(dd * (size_t)pb.max_chunks * pb.H, 256);
    l.chunk_bytes = ckpt + dd * (size_t)(kBwdChunk + 1) * pb.N * pb.H;
    l.total = l.plan_bytes + l.chunk_bytes;
    return l;
}

cudaError_t launch_backward(const Problem &pb, const void *dO, const float *dS_final,
                            float *gq, float *gk, float *gv, float *gla, float *gbeta,
                            float *gS0, void *workspace, cudaStream_t st)
{
    const WorkspaceLayout lay = bwd_workspace_layout(pb);
    Plan plan;
    plan.seq_start = static_cast<int32_t *>(workspace);
    plan.chunk_off = plan.seq_start + (pb.N + 1);
    plan.order = plan.chunk_off + (pb.N + 1);
    cudaError_t e = launch_plan(pb, plan, st);
    if (e != cudaSuccess) return e;
    BwdParams p;
    p.q = pb.q; p.k = pb.k; p.v = pb.v; p.dO = dO;
    p.log_alpha = pb.log_alpha; p.beta = pb.beta; p.S0 = pb.S0; p.dS_final = dS_final;
    p.N = pb.N; p.H = pb.H; p.gate_per_channel = pb.gate_per_channel; p.scale = pb.scale;
    p.gq = gq; p.gk = gk; p.gv = gv; p.gla = gla; p.gbeta = gbeta; p.gS0 = gS0;
    p.seq_start = plan.seq_start; p.chunk_off = plan.chunk_off;
    char *ws = static_cast<char *>(workspace) + lay.plan_bytes;
    p.ckpt = reinterpret_cast<float *>(ws);
    p.blk = reinterpret_cast<float *>(
        ws + align_up((size_t)pb.dk * pb.dk * sizeof(float) * (size_t)pb.max_chunks * pb.H, 256));
    const bool bf = pb.dtype == KDA_DTYPE_BF16;
    switch (pb.dk) {
    case 32: return bf ? launch_d<32, __nv_bfloat16>(p, st) : launch_d<32, float>(p, st);
    case 64: return bf ? launch_d<64, __nv_bfloat16>(p, st) : launch_d<64, float>(p, st);
    case 128: return bf ? launch_d<128, __nv_bfloat16>(p, st) : launch_d<128, float>(p, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace kda
