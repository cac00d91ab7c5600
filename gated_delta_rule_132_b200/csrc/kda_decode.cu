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
// Several consecutive tokens per (sequence, head) (multi-token decode, or
// continuing a prefill by a few tokens) run in decode_tokens_kernel with the
// state kept in registers between them: the state still crosses HBM once each
// way, the tokens' vectors are staged in shared memory ahead of use, and each
// token costs two CTA barriers and its own few hundred bytes.
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

// Several tokens per call (T >= 2). The state stays in registers as in
// decode_kernel; the tokens' vectors are staged in shared memory in blocks of
// kTokBlock tokens with cp.async, two blocks in flight, so a token never waits
// for a global load. When a block lands, its log-decays become decays
// (alpha = exp(log_alpha)) and each warp forms one token's k^T q. Per token:
// partial S'^T k and S'^T q -> barrier -> u and o per value column -> barrier
// -> S += k u^T. The reduction and u buffers alternate between tokens, so those
// two barriers are the only ones a token needs.
constexpr int kTokBlock = 8;

// Packed fp32 pairs (sm_100 f32x2 arithmetic): each lane is one ordinary fp32
// multiply or fused multiply-add with round-to-nearest, so results equal the
// scalar operations bit for bit, at half the instruction count.
__device__ __forceinline__ uint64_t f2(float a, float b)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void f2_get(uint64_t v, float &a, float &b)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

template <int DK, int DV, typename TIn>
struct TokSmem {
    static constexpr int CG = DV / 4, RG = kDecodeThreads / CG;
    // one block of staged tokens
    static constexpr size_t kLa = 0;                                         // fp32 [TB][DK] (alpha after landing)
    static constexpr size_t kK = kLa + sizeof(float) * kTokBlock * DK;        // TIn [TB][DK]
    static constexpr size_t kQ = kK + sizeof(TIn) * kTokBlock * DK;          // TIn [TB][DK]
    static constexpr size_t kV = kQ + sizeof(TIn) * kTokBlock * DK;          // TIn [TB][DV]
    static constexpr size_t kB = kV + sizeof(TIn) * kTokBlock * DV;          // fp32 [TB] beta
    static constexpr size_t kKq = kB + sizeof(float) * kTokBlock;            // fp32 [TB] k^T q
    static constexpr size_t kBlock = (kKq + sizeof(float) * kTokBlock + 15) / 16 * 16;
    static constexpr size_t kRed = 2 * kBlock;                               // fp32 [2][2][RG][DV]
    static constexpr size_t kU = kRed + sizeof(float) * 2 * 2 * RG * DV;     // fp32 [2][DV]
    static constexpr size_t kBytes = kU + sizeof(float) * 2 * DV;
};

template <int DK, int DV, typename TIn>
__global__ void __launch_bounds__(kDecodeThreads, 2)
decode_tokens_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k,
                     const TIn *__restrict__ v, const float *__restrict__ log_alpha,
                     const float *__restrict__ beta, float *__restrict__ S, int T, int H,
                     int gate_per_channel, float scale, TIn *__restrict__ o)
{
    using L = TokSmem<DK, DV, TIn>;
    constexpr int CG = L::CG, RG = L::RG, RPT = DK / RG;
    static_assert(DK % RG == 0 && RPT >= 1, "unsupported head size");
    static_assert(DV <= kDecodeThreads, "one value column per thread");
    extern __shared__ __align__(16) uint8_t smem[];

    const int unit = blockIdx.x;  // n * H + h
    const int n = unit / H, h = unit - n * H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cg = tid % CG, rg = tid / CG;
    float *Su = S + (size_t)unit * DK * DV;

    // the state as packed pairs: st[r][0] = columns (4 cg, 4 cg + 1), st[r][1] = (+2, +3)
    uint64_t st[RPT][2];
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const float4 x = __ldcs(reinterpret_cast<const float4 *>(Su + (size_t)(r * RG + rg) * DV) + cg);
        st[r][0] = f2(x.x, x.y);
        st[r][1] = f2(x.z, x.w);
    }

    const int nblocks = (T + kTokBlock - 1) / kTokBlock;
    auto tok_index = [&](int t) { return ((size_t)n * T + t) * H + h; };  // (n, t, h)
    // Stage block b (tokens kTokBlock b ..) into buffer b & 1, as one cp.async group.
    auto stage = [&](int b) {
        uint8_t *buf = smem + (size_t)(b & 1) * L::kBlock;
        const int t0 = b * kTokBlock, nt = min(kTokBlock, T - t0);
        constexpr int kLaG = DK * 4 / 16, kKG = DK * (int)sizeof(TIn) / 16, kVG = DV * (int)sizeof(TIn) / 16;
        constexpr int kPer = kLaG + 2 * kKG + kVG;  // 16-byte granules per token
        for (int g = tid; g < nt * kPer; g += kDecodeThreads) {
            const int tt = g / kPer, r = g % kPer;
            const size_t tok = tok_index(t0 + tt);
            const void *src;
            uint8_t *dst;
            if (r < kLaG) {
                if (!gate_per_channel) continue;
                src = log_alpha + tok * DK + 4 * r;
                dst = buf + L::kLa + ((size_t)tt * DK + 4 * r) * 4;
            } else if (r < kLaG + kKG) {
                const int e = (r - kLaG) * (16 / (int)sizeof(TIn));
                src = k + tok * DK + e;
                dst = buf + L::kK + ((size_t)tt * DK + e) * sizeof(TIn);
            } else if (r < kLaG + 2 * kKG) {
                const int e = (r - kLaG - kKG) * (16 / (int)sizeof(TIn));
                src = q + tok * DK + e;
                dst = buf + L::kQ + ((size_t)tt * DK + e) * sizeof(TIn);
            } else {
                const int e = (r - kLaG - 2 * kKG) * (16 / (int)sizeof(TIn));
                src = v + tok * DV + e;
                dst = buf + L::kV + ((size_t)tt * DV + e) * sizeof(TIn);
            }
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                         ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src) : "memory");
        }
        if (tid < nt) {  // beta, and the scalar gate of one-gate-per-head calls
            const size_t tok = tok_index(t0 + tid);
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;"
                         ::"r"((uint32_t)__cvta_generic_to_shared(buf + L::kB + 4 * tid)),
                           "l"(beta + tok) : "memory");
            if (!gate_per_channel)
                asm volatile("cp.async.ca.shared.global [%0], [%1], 4;"
                             ::"r"((uint32_t)__cvta_generic_to_shared(buf + L::kLa + 4 * tid * DK)),
                               "l"(log_alpha + tok) : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    stage(0);
    if (nblocks > 1) stage(1);

    float *red = reinterpret_cast<float *>(smem + L::kRed);  // [2][2][RG][DV]
    float *su = reinterpret_cast<float *>(smem + L::kU);     // [2][DV]
    for (int b = 0; b < nblocks; ++b) {
        uint8_t *buf = smem + (size_t)(b & 1) * L::kBlock;
        const int t0 = b * kTokBlock, nt = min(kTokBlock, T - t0);
        // this block's copies (the later block's may stay in flight)
        if (b + 1 < nblocks) asm volatile("cp.async.wait_group 1;" ::: "memory");
        else asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();
        float *sa = reinterpret_cast<float *>(buf + L::kLa);
        const TIn *sk = reinterpret_cast<const TIn *>(buf + L::kK);
        const TIn *sq = reinterpret_cast<const TIn *>(buf + L::kQ);
        const TIn *sv = reinterpret_cast<const TIn *>(buf + L::kV);
        const float *sb = reinterpret_cast<const float *>(buf + L::kB);
        float *skq = reinterpret_cast<float *>(buf + L::kKq);
        // decays and k^T q of the block's tokens
        if (gate_per_channel) {
            for (int e = tid; e < nt * DK; e += kDecodeThreads) sa[e] = expf(sa[e]);
        } else if (tid < nt) {
            const float a = expf(sa[tid * DK]);
            for (int i = 0; i < DK; ++i) sa[tid * DK + i] = a;
        }
        if (warp < nt) {
            float acc = 0.f;
            for (int i = lane; i < DK; i += 32) acc += to_f32(sk[warp * DK + i]) * to_f32(sq[warp * DK + i]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (lane == 0) skq[warp] = acc;
        }
        __syncthreads();
        for (int tt = 0; tt < nt; ++tt) {
            const int t = t0 + tt, par = t & 1;
            const float *al = sa + tt * DK;
            const TIn *kt = sk + tt * DK;
            const TIn *qt = sq + tt * DK;
            // S' = Diag(alpha) S and this thread's partial S'^T k, S'^T q
            uint64_t a0 = f2(0.f, 0.f), a1 = a0, b0 = a0, b1 = a0;
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const int i = r * RG + rg;
                const float ali = al[i], ki = to_f32(kt[i]), qi = to_f32(qt[i]);
                const uint64_t al2 = f2(ali, ali), k2 = f2(ki, ki), q2 = f2(qi, qi);
                st[r][0] = mul2(st[r][0], al2);
                st[r][1] = mul2(st[r][1], al2);
                a0 = fma2(st[r][0], k2, a0); a1 = fma2(st[r][1], k2, a1);
                b0 = fma2(st[r][0], q2, b0); b1 = fma2(st[r][1], q2, b1);
            }
            float4 a, bq;
            f2_get(a0, a.x, a.y); f2_get(a1, a.z, a.w);
            f2_get(b0, bq.x, bq.y); f2_get(b1, bq.z, bq.w);
            float *rk = red + ((size_t)par * 2 + 0) * RG * DV, *rq = red + ((size_t)par * 2 + 1) * RG * DV;
            reinterpret_cast<float4 *>(rk + rg * DV)[cg] = a;
            reinterpret_cast<float4 *>(rq + rg * DV)[cg] = bq;
            __syncthreads();
            // u = beta (v - S'^T k), o = scale (S'^T q + (k^T q) u), per value column
            if (tid < DV) {
                float sk2 = 0.f, sq2 = 0.f;
#pragma unroll
                for (int g = 0; g < RG; ++g) { sk2 += rk[g * DV + tid]; sq2 += rq[g * DV + tid]; }
                const float u = sb[tt] * (to_f32(sv[tt * DV + tid]) - sk2);
                su[par * DV + tid] = u;
                o[tok_index(t) * DV + tid] = from_f32<TIn>(scale * (sq2 + skq[tt] * u));
            }
            __syncthreads();
            // S = S' + k u^T
            const float4 u4 = reinterpret_cast<const float4 *>(su + par * DV)[cg];
            const uint64_t u01 = f2(u4.x, u4.y), u23 = f2(u4.z, u4.w);
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const float ki = to_f32(kt[r * RG + rg]);
                const uint64_t k2 = f2(ki, ki);
                st[r][0] = fma2(k2, u01, st[r][0]);
                st[r][1] = fma2(k2, u23, st[r][1]);
            }
        }
        // every thread is done with this buffer before block b + 2 lands in it
        __syncthreads();
        if (b + 2 < nblocks) stage(b + 2);
    }
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        float4 x;
        f2_get(st[r][0], x.x, x.y);
        f2_get(st[r][1], x.z, x.w);
        __stcs(reinterpret_cast<float4 *>(Su + (size_t)(r * RG + rg) * DV) + cg, x);
    }
}

template <int D, typename TIn>
cudaError_t launch_d(const void *q, const void *k, const void *v, const float *la,
                     const float *beta, float *S, int units, int T, int H, int gpc, float scale,
                     void *o, cudaStream_t st)
{
    if (T == 1) {
        decode_kernel<D, D, TIn><<<units, kDecodeThreads, 0, st>>>(
            static_cast<const TIn *>(q), static_cast<const TIn *>(k), static_cast<const TIn *>(v),
            la, beta, S, T, H, gpc, scale, static_cast<TIn *>(o));
        note_launch();
        return cudaGetLastError();
    }
    using L = TokSmem<D, D, TIn>;
    auto kern = decode_tokens_kernel<D, D, TIn>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)L::kBytes);
    if (e != cudaSuccess) return e;
    kern<<<units, kDecodeThreads, L::kBytes, st>>>(
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
