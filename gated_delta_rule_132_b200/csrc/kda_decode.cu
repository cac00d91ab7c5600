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
// against a few hundred bytes of token data. One CTA owns one (sequence, head)
// and keeps the whole dk x dv state in registers, so the state crosses HBM once
// each way per call, however many tokens the call carries. Loads and stores of
// the state use the evict-first cache hint: it is touched once per call.
//  * decode_kernel (one token): float4 per thread per row, a warp covering full
//    512-byte rows for dv = 128; every state load is issued before any
//    arithmetic, and S'^T k and S'^T q are summed across row groups in shared
//    memory.
//  * decode_tokens_kernel (T >= 2): warp w owns dv / 8 value columns over all dk
//    key rows, lane l 4 consecutive columns (group l mod n_c of the warp's n_c
//    groups of 4) of the rows l / n_c + m (32 / n_c). The sums over the key rows
//    are then sums over the lanes of one column group, by recursive halving with
//    shuffles, so a warp needs no other warp inside a token and the CTA meets at
//    a barrier three times per block of staged tokens.
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

// Several tokens per call (T >= 2). Token vectors are staged in shared memory
// in blocks of kTokBlock tokens with cp.async, two blocks in flight, so a token
// never waits for a global load. When a block has landed, its rows become
// packed {alpha, k, q} per key row (alpha = exp(log_alpha)) and k^T q per token
// (barrier); then every warp runs the block's tokens on its own columns; o goes
// to a staging tile and leaves as full row pieces after a last barrier, when the
// buffer is also free for block b + 2. The value columns of a head never mix,
// so a head's 8 column slices of dv / 8 may be spread over kTokParts CTAs of
// 8 / kTokParts warps each; one CTA per head measured fastest (2 and 4 CTAs of
// fewer warps were slower at every T tried).
constexpr int kTokBlock = 8;
constexpr int kTokParts = 1;                      // CTAs per (sequence, head)
constexpr int kTokWarps = 8 / kTokParts;          // warps per CTA
constexpr int kTokThreads = 32 * kTokWarps;

// Packed fp32 pairs (sm_100 f32x2 arithmetic): each lane is one ordinary fp32
// multiply or fused multiply-add with round-to-nearest, at half the
// instruction count.
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
    // one block of staged tokens, as landed (two buffers)
    static constexpr size_t kLa = 0;                                         // fp32 [TB][DK]
    static constexpr size_t kK = kLa + sizeof(float) * kTokBlock * DK;        // TIn [TB][DK]
    static constexpr size_t kQ = kK + sizeof(TIn) * kTokBlock * DK;          // TIn [TB][DK]
    static constexpr size_t kV = kQ + sizeof(TIn) * kTokBlock * DK;          // TIn [TB][DV]
    static constexpr size_t kB = kV + sizeof(TIn) * kTokBlock * DV;          // fp32 [TB] beta
    static constexpr size_t kBlock = (kB + sizeof(float) * kTokBlock + 15) / 16 * 16;
    // the block being computed
    static constexpr size_t kRow = 2 * kBlock;                               // float4 [TB][DK] {alpha, k, q, 0}
    static constexpr size_t kKq = kRow + 16 * kTokBlock * DK;                // fp32 [TB] k^T q
    static constexpr size_t kO = kKq + sizeof(float) * kTokBlock;            // TIn [TB][DV] output rows
    static constexpr size_t kBytes = kO + sizeof(TIn) * kTokBlock * DV;
};

template <int DK, int DV, typename TIn>
__global__ void __launch_bounds__(kTokThreads, 2 * kTokParts)
decode_tokens_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k,
                     const TIn *__restrict__ v, const float *__restrict__ log_alpha,
                     const float *__restrict__ beta, float *__restrict__ S, int T, int H,
                     int gate_per_channel, float scale, TIn *__restrict__ o)
{
    using L = TokSmem<DK, DV, TIn>;
    constexpr int CPW = DV / 8;                 // value columns per warp
    constexpr int CPC = CPW * kTokWarps;        // value columns per CTA
    constexpr int NC = CPW / 4;                 // column groups of 4 per warp
    constexpr int LNC = NC == 4 ? 2 : NC == 2 ? 1 : 0;
    constexpr int NR = 32 / NC;                 // row sets (lanes per column group)
    constexpr int RPT = DK / NR;                // key rows per thread
    static_assert(NC == 1 || NC == 2 || NC == 4, "dv / 8 must be 4, 8 or 16 columns");
    static_assert(DK % NR == 0 && RPT >= 1, "unsupported head size");
    extern __shared__ __align__(16) uint8_t smem[];

    const int unit = blockIdx.x / kTokParts;  // n * H + h
    const int part = blockIdx.x % kTokParts;  // value columns CPC part ..
    const int n = unit / H, h = unit - n * H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cc = lane & (NC - 1), rs = lane >> LNC;
    const int c0 = CPC * part + CPW * warp + 4 * cc;  // this thread's first value column
    float *Su = S + (size_t)unit * DK * DV;

    const int nblocks = (T + kTokBlock - 1) / kTokBlock;
    auto tok_index = [&](int t) { return ((size_t)n * T + t) * H + h; };  // (n, t, h)
    // Stage block b (tokens kTokBlock b ..) into buffer b & 1, as one cp.async group.
    auto stage = [&](int b) {
        uint8_t *buf = smem + (size_t)(b & 1) * L::kBlock;
        const int t0 = b * kTokBlock, nt = min(kTokBlock, T - t0);
        constexpr int kLaG = DK * 4 / 16, kKG = DK * (int)sizeof(TIn) / 16, kVG = DV * (int)sizeof(TIn) / 16;
        constexpr int kPer = kLaG + 2 * kKG + kVG;  // 16-byte granules per token
        for (int g = tid; g < nt * kPer; g += kTokThreads) {
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
    if (nblocks > 0) stage(0);
    if (nblocks > 1) stage(1);

    // the state, as packed pairs: st[m][0] = columns (c0, c0 + 1), st[m][1] = (+2, +3) of
    // key row rs + NR m
    uint64_t st[RPT][2];
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const float4 x = __ldcs(reinterpret_cast<const float4 *>(Su + (size_t)(rs + NR * m) * DV + c0));
        st[m][0] = f2(x.x, x.y);
        st[m][1] = f2(x.z, x.w);
    }

    float4 *rows = reinterpret_cast<float4 *>(smem + L::kRow);
    float *skq = reinterpret_cast<float *>(smem + L::kKq);
    TIn *so = reinterpret_cast<TIn *>(smem + L::kO);
    // after the reduction: this lane's sum is S'^T k (bit 4 clear) or S'^T q (set)
    // of column c0 + e; duplicates (dv < 128) write no output
    const bool is_q = lane & 16;
    const int e_own = ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
    const bool primary = ((lane >> LNC) & ((4 >> LNC) - 1)) == 0;
    for (int b = 0; b < nblocks; ++b) {
        const uint8_t *buf = smem + (size_t)(b & 1) * L::kBlock;
        const int t0 = b * kTokBlock, nt = min(kTokBlock, T - t0);
        // this block's copies (the later block's may stay in flight)
        if (b + 1 < nblocks) asm volatile("cp.async.wait_group 1;" ::: "memory");
        else asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();
        const float *sa = reinterpret_cast<const float *>(buf + L::kLa);
        const TIn *sk = reinterpret_cast<const TIn *>(buf + L::kK);
        const TIn *sq = reinterpret_cast<const TIn *>(buf + L::kQ);
        const TIn *sv = reinterpret_cast<const TIn *>(buf + L::kV);
        const float *sb = reinterpret_cast<const float *>(buf + L::kB);
        for (int x = tid; x < nt * DK; x += kTokThreads) {
            const int tt = x / DK;
            const float la = gate_per_channel ? sa[x] : sa[tt * DK];
            rows[x] = make_float4(expf(la), to_f32(sk[x]), to_f32(sq[x]), 0.f);
        }
        for (int tt = warp; tt < nt; tt += kTokWarps) {
            float acc = 0.f;
            for (int i = lane; i < DK; i += 32) acc += to_f32(sk[tt * DK + i]) * to_f32(sq[tt * DK + i]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (lane == 0) skq[tt] = acc;
        }
        __syncthreads();
        for (int tt = 0; tt < nt; ++tt) {
            const float4 *rt = rows + tt * DK;
            // S' = Diag(alpha) S and this thread's partial S'^T k, S'^T q over its rows
            uint64_t k01 = f2(0.f, 0.f), k23 = k01, q01 = k01, q23 = k01;
#pragma unroll
            for (int m = 0; m < RPT; ++m) {
                const float4 x = rt[rs + NR * m];
                const uint64_t a2 = f2(x.x, x.x), k2 = f2(x.y, x.y), q2 = f2(x.z, x.z);
                st[m][0] = mul2(st[m][0], a2);
                st[m][1] = mul2(st[m][1], a2);
                k01 = fma2(st[m][0], k2, k01); k23 = fma2(st[m][1], k2, k23);
                q01 = fma2(st[m][0], q2, q01); q23 = fma2(st[m][1], q2, q23);
            }
            float w[8];
            f2_get(k01, w[0], w[1]); f2_get(k23, w[2], w[3]);
            f2_get(q01, w[4], w[5]); f2_get(q23, w[6], w[7]);
            // sum over the row-set lanes (bits LNC .. 4): the first three steps
            // halve the vector (k | q, then column pairs, then columns), any
            // further step adds its partner's copy
#pragma unroll
            for (int s = 0; s < 5 - LNC; ++s) {
                const int bit = 16 >> s;
                if (s < 3) {
                    const int half = 4 >> s;
                    const bool up = lane & bit;
#pragma unroll
                    for (int e = 0; e < half; ++e) {
                        const float send = up ? w[e] : w[e + half];
                        const float keep = up ? w[e + half] : w[e];
                        w[e] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
                    }
                } else {
                    w[0] += __shfl_xor_sync(0xffffffffu, w[0], bit);
                }
            }
            // u = beta (v - S'^T k) on the k lanes, o = scale (S'^T q + (k^T q) u)
            // on the q lanes, S = S' + k u^T everywhere
            const float u = is_q ? 0.f : sb[tt] * (to_f32(sv[tt * DV + c0 + e_own]) - w[0]);
            const float u_q = __shfl_xor_sync(0xffffffffu, u, 16);
            if (is_q && primary) so[tt * DV + c0 + e_own] = from_f32<TIn>(scale * (w[0] + skq[tt] * u_q));
            float u4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) u4[e] = __shfl_sync(0xffffffffu, u, cc + 4 * e);
            const uint64_t u01 = f2(u4[0], u4[1]), u23 = f2(u4[2], u4[3]);
#pragma unroll
            for (int m = 0; m < RPT; ++m) {
                const float km = rt[rs + NR * m].y;  // reread: keeps the registers for the state
                const uint64_t k2 = f2(km, km);
                st[m][0] = fma2(k2, u01, st[m][0]);
                st[m][1] = fma2(k2, u23, st[m][1]);
            }
        }
        // every warp is done with this block: its output rows leave whole, and
        // its buffer takes block b + 2
        __syncthreads();
        constexpr int kOG = CPC * (int)sizeof(TIn) / 16;  // 16-byte pieces of this CTA's columns
        for (int x = tid; x < nt * kOG; x += kTokThreads) {
            const int tt = x / kOG, r = x % kOG;
            *reinterpret_cast<uint4 *>(o + tok_index(t0 + tt) * DV + CPC * part + r * (16 / (int)sizeof(TIn))) =
                reinterpret_cast<const uint4 *>(so + tt * DV + CPC * part)[r];
        }
        if (b + 2 < nblocks) stage(b + 2);
    }
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        float4 x;
        f2_get(st[m][0], x.x, x.y);
        f2_get(st[m][1], x.z, x.w);
        __stcs(reinterpret_cast<float4 *>(Su + (size_t)(rs + NR * m) * DV + c0), x);
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
    kern<<<units * kTokParts, kTokThreads, L::kBytes, st>>>(
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
