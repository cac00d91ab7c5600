// kda_decode.cu — one recurrent KDA step for a batch of independent sequences.
//
// Source: the KDA update rule of "Kimi Linear：让长上下文大模型真正实用的线性注意力架构"
// (juejin.cn), section 三 5️⃣, S_t = (I - beta k k^T) Diag(alpha) S_{t-1} + beta k v^T,
// read out as o = scale * S_t^T q. Written with S' = Diag(alpha) S_{t-1} and
// u = beta (v - S'^T k), the rule is S_t = S' + k u^T, and the read-out
// o = scale * (S'^T q + (k^T q) u) needs only reductions of S' — so each head's
// fp32 state is read once and written once, with no second pass.
//
// The step is bound by HBM: 2 * dk * dv * 4 bytes of state per (sequence, head)
// against a few hundred bytes of token data. One CTA owns one (sequence, head):
// its 256 threads hold the whole dk x dv state in registers (float4 per thread
// per row, a warp covering full 512-byte rows for dv = 128), issue every state
// load before any arithmetic, reduce S'^T k and S'^T q across row groups in
// shared memory, and stream the updated rows back. Loads and stores use the
// evict-first cache hint: the state is touched once per call.
//
// The same kernel applies T consecutive tokens per (sequence, head) with the
// state kept in registers between them (multi-token decode, or continuing a
// prefill by a few tokens): the state still crosses HBM once each way, and
// each token costs three CTA barriers and its own few hundred bytes, with the
// next token's vectors loaded while the current one is reduced.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kDecodeThreads = 256;

template <int DK, int DV, typename TIn>
__global__ void __launch_bounds__(kDecodeThreads, 2)
decode_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
              const float *__restrict__ log_alpha, const float *__restrict__ beta,
              float *__restrict__ S, int T, int H, int gate_per_channel, float scale,
              TIn *__restrict__ o)
{
    constexpr int CG = DV / 4;                  // float4 column groups per row
    constexpr int RG = kDecodeThreads / CG;     // row groups
    constexpr int RPT = DK / RG;                // rows per thread
    static_assert(DK % RG == 0 && RPT >= 1, "unsupported head size");
    static_assert(DK <= kDecodeThreads && DV <= kDecodeThreads, "one vector element per thread");

    __shared__ float s_alpha[DK], s_k[DK], s_q[DK];
    __shared__ __align__(16) float s_red[2][RG][DV];
    __shared__ __align__(16) float s_u[DV];
    __shared__ float s_kq;

    const int unit = blockIdx.x;  // n * H + h
    const int n = unit / H, h = unit - n * H;
    const int tid = threadIdx.x;
    const int cg = tid % CG, rg = tid / CG;
    float *Su = S + (size_t)unit * DK * DV;

    // 1. Put every state load in flight first.
    float4 st[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = r * RG + rg;
        st[r] = __ldcs(reinterpret_cast<const float4 *>(Su + (size_t)i * DV) + cg);
    }
    // Token vectors: thread i < DK holds element i of log_alpha, k, q and thread
    // j < DV element j of v (and beta) for the next token, loaded one token ahead.
    float nla = 0.f, nk = 0.f, nq = 0.f, nv = 0.f, nb = 0.f;
    auto fetch = [&](int t) {
        const size_t tok = ((size_t)n * T + t) * H + h;  // (n, t, h) of [N, T, H, ...]
        if (tid < DK) {
            nla = gate_per_channel ? log_alpha[tok * DK + tid] : log_alpha[tok];
            nk = to_f32(k[tok * DK + tid]);
            nq = to_f32(q[tok * DK + tid]);
        }
        if (tid < DV) {
            nv = to_f32(v[tok * DV + tid]);
            nb = beta[tok];
        }
    };
    if (T > 0) fetch(0);
    for (int t = 0; t < T; ++t) {
        const size_t tok = ((size_t)n * T + t) * H + h;
        if (tid < DK) { s_alpha[tid] = expf(nla); s_k[tid] = nk; s_q[tid] = nq; }
        const float vt = nv, bt = nb;
        if (t + 1 < T) fetch(t + 1);
        __syncthreads();
        if (tid < 32) {
            float acc = 0.f;
            for (int i = tid; i < DK; i += 32) acc += s_k[i] * s_q[i];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (tid == 0) s_kq = acc;
        }
        // 2. S' = Diag(alpha) S, and this thread's partial S'^T k and S'^T q.
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const int i = r * RG + rg;
            const float al = s_alpha[i], ki = s_k[i], qi = s_q[i];
            st[r].x *= al; st[r].y *= al; st[r].z *= al; st[r].w *= al;
            a.x += st[r].x * ki; a.y += st[r].y * ki; a.z += st[r].z * ki; a.w += st[r].w * ki;
            b.x += st[r].x * qi; b.y += st[r].y * qi; b.z += st[r].z * qi; b.w += st[r].w * qi;
        }
        reinterpret_cast<float4 *>(&s_red[0][rg][0])[cg] = a;
        reinterpret_cast<float4 *>(&s_red[1][rg][0])[cg] = b;
        __syncthreads();
        // 3. Per value column: u = beta (v - S'^T k), o = scale (S'^T q + (k^T q) u).
        if (tid < DV) {
            float sa = 0.f, sb = 0.f;
#pragma unroll
            for (int g = 0; g < RG; ++g) { sa += s_red[0][g][tid]; sb += s_red[1][g][tid]; }
            const float u = bt * (vt - sa);
            s_u[tid] = u;
            o[tok * DV + tid] = from_f32<TIn>(scale * (sb + s_kq * u));
        }
        __syncthreads();
        // 4. S_t = S' + k u^T, kept in registers for the next token.
        const float4 u4 = reinterpret_cast<const float4 *>(s_u)[cg];
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const float ki = s_k[r * RG + rg];
            st[r].x += ki * u4.x; st[r].y += ki * u4.y; st[r].z += ki * u4.z; st[r].w += ki * u4.w;
        }
        __syncthreads();  // the next token overwrites s_k, s_u and s_red
    }
    // 5. The state after the last token, streamed back.
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = r * RG + rg;
        __stcs(reinterpret_cast<float4 *>(Su + (size_t)i * DV) + cg, st[r]);
    }
}

template <int D, typename TIn>
cudaError_t launch_d(const void *q, const void *k, const void *v, const float *la,
                     const float *beta, float *S, int units, int T, int H, int gpc, float scale,
                     void *o, cudaStream_t st)
{
    decode_kernel<D, D, TIn><<<units, kDecodeThreads, 0, st>>>(
        static_cast<const TIn *>(q), static_cast<const TIn *>(k), static_cast<const TIn *>(v),
        la, beta, S, T, H, gpc, scale, static_cast<TIn *>(o));
    note_launch();
    return cudaGetLastError();
}

template <typename TIn>
cudaError_t launch_t(int d, const void *q, const void *k, const void *v, const float *la,
                     const float *beta, float *S, int units, int T, int H, int gpc, float scale,
                     void *o, cudaStream_t st)
{
    switch (d) {
    case 32: return launch_d<32, TIn>(q, k, v, la, beta, S, units, T, H, gpc, scale, o, st);
    case 64: return launch_d<64, TIn>(q, k, v, la, beta, S, units, T, H, gpc, scale, o, st);
    case 128: return launch_d<128, TIn>(q, k, v, la, beta, S, units, T, H, gpc, scale, o, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_decode(const void *q, const void *k, const void *v, kda_dtype_t dt,
                          const float *log_alpha, const float *beta, float *S, int N, int T,
                          int H, int dk, int dv, float scale, void *o, int gate_per_channel,
                          cudaStream_t stream)
{
    if (dk != dv) return cudaErrorInvalidValue;
    const int units = N * H;
    if (dt == KDA_DTYPE_BF16)
        return launch_t<__nv_bfloat16>(dk, q, k, v, log_alpha, beta, S, units, T, H,
                                       gate_per_channel, scale, o, stream);
    return launch_t<float>(dk, q, k, v, log_alpha, beta, S, units, T, H, gate_per_channel,
                           scale, o, stream);
}

}  // namespace kda
