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
// Parallel layout. Value columns never mix: column j of S_t depends only on
// column j of S_{t-1} and on v_t[j], and so does column j of G. Each (sequence,
// head) is split into dv / 32 slices of 32 value columns, one CTA per slice;
// kTpr threads share each of the dk state rows, each keeping kCols / kTpr
// columns of that row of S_t, S_{t-1} and G in registers. Sums over rows
// (S'^T k, G^T k) are a warp reduce-scatter — after log2(32 / kTpr) shuffle
// rounds lane l holds the warp's sum for one column — then a sum over the warps
// through shared memory, one barrier per token; sums over columns (dq, dk,
// dlog_alpha, dbeta) are a few register FMAs and log2(kTpr) shuffles. The
// derivatives that sum over all value columns (dq, dk, dlog_alpha, dbeta) are
// written per slice and added in slice order by a second kernel, so results do
// not depend on scheduling; dv and dS0 belong to one slice and are written
// directly.
//
// The states the walk needs come from a replay of the forward: a first pass
// keeps the state at every 32-token block start; each block, last to first, is
// replayed from its checkpoint into a per-CTA buffer of its 33 states and walked
// backwards, with S_{t-1} copied into shared memory by cp.async one token ahead.
#include <algorithm>

#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kBlk = 32;   // tokens per replay block (checkpoint interval)
constexpr int kCols = 32;  // value columns per CTA
constexpr int kTpr = 1;    // threads per state row (1 measured fastest of 1, 2, 4)

// A state slice in memory (checkpoints, replay buffer, shared staging) is 8 * D
// float4: the thread (row r, part u) holding columns u*CPT .. u*CPT+CPT-1 keeps
// its float4 m (columns u*CPT + 4m .. +3) at index (m * D + r) * TPR + u, so a
// warp's threads touch consecutive 16-byte words.
struct BwdParams {
    const void *q, *k, *v, *dO;
    const float *log_alpha, *beta, *S0, *dS_final;
    int N, H, gate_per_channel;
    float scale;
    float *gv, *gS0;              // written directly (one slice owns each element)
    float *pq, *pk, *pla, *pb;    // per-slice partials [slices][tokens * H][dk] ([..][tokens * H])
    size_t TH;                    // packed tokens x heads
    const int32_t *seq_start, *chunk_off, *order;
    float4 *ckpt;                 // [2 * max_chunks][H][slices][8 * dk]
    float4 *blk;                  // [CTAs][kBlk + 1][8 * dk]
};

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem)
{
    const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Reduce-scatter over the 32 / TPR lanes that share lane % TPR, each holding
// CPT = 32 / TPR values: lane l returns the sum over those lanes of x[l / TPR]
// (x is destroyed). Recursive halving: each round keeps the half of the values
// whose index bit matches the lane's and adds the partner's copy of that half.
template <int CPT, int TPR>
__device__ __forceinline__ float reduce_scatter(float (&x)[CPT], int lane)
{
#pragma unroll
    for (int hb = CPT / 2; hb >= 1; hb >>= 1) {
        const bool up = (lane & (hb * TPR)) != 0;
#pragma unroll
        for (int i = 0; i < hb; ++i) {
            const float lo = x[i], hi = x[i + hb];
            const float send = up ? lo : hi, keep = up ? hi : lo;
            x[i] = keep + __shfl_xor_sync(0xffffffffu, send, hb * TPR);
        }
    }
    return x[0];
}

// Sum over the TPR lanes of one row (every one of them gets the total).
template <int TPR>
__device__ __forceinline__ float row_sum(float v)
{
#pragma unroll
    for (int o = 1; o < TPR; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <int CPT>
__device__ __forceinline__ void put_part(float4 *dst, const float (&S)[CPT], int at, int stride)
{
#pragma unroll
    for (int m = 0; m < CPT / 4; ++m)
        dst[at + m * stride] = make_float4(S[4 * m], S[4 * m + 1], S[4 * m + 2], S[4 * m + 3]);
}

template <int CPT>
__device__ __forceinline__ void get_part(float (&S)[CPT], const float4 *src, int at, int stride)
{
#pragma unroll
    for (int m = 0; m < CPT / 4; ++m) {
        const float4 x = src[at + m * stride];
        S[4 * m] = x.x; S[4 * m + 1] = x.y; S[4 * m + 2] = x.z; S[4 * m + 3] = x.w;
    }
}

// CPT consecutive floats of a dense row (16-byte aligned) into registers, or zeros.
template <int CPT>
__device__ __forceinline__ void get_dense(float (&S)[CPT], const float *src)
{
#pragma unroll
    for (int m = 0; m < CPT / 4; ++m) {
        const float4 x = src ? reinterpret_cast<const float4 *>(src)[m] : make_float4(0.f, 0.f, 0.f, 0.f);
        S[4 * m] = x.x; S[4 * m + 1] = x.y; S[4 * m + 2] = x.z; S[4 * m + 3] = x.w;
    }
}

__device__ __forceinline__ void cp_async4(void *smem, const void *gmem)
{
    const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(sa), "l"(gmem) : "memory");
}

// The scalars one thread needs from one token: row r of k, q and log_alpha;
// column cl of v and dO; beta.
struct Tok { float k, q, la, v, d, b; };

template <int D, int TPR, typename TIn> struct BwdShape {
    static constexpr int NT = D * TPR, NW = NT / 32, CPT = kCols / TPR;
    // One block's token data, staged in shared memory: k, q [kBlk][D] and the
    // v, dO columns of the slice [kBlk][kCols] as given, log_alpha [kBlk][D]
    // (one gate per head: element 0 of each row), beta [kBlk].
    static constexpr size_t kTk = 0, kTq = kTk + kBlk * D * sizeof(TIn),
                            kTla = kTq + kBlk * D * sizeof(TIn), kTv = kTla + kBlk * D * 4,
                            kTd = kTv + kBlk * kCols * sizeof(TIn),
                            kTb = kTd + kBlk * kCols * sizeof(TIn), kTokBytes = kTb + kBlk * 4;
    // shared: S_{t-1} staging [2][8 D] float4, column sums [2][NW][32] float2,
    // per-warp broadcast [2][NW][3][32] floats (dO, w, g by column), token data [2]
    static constexpr size_t kSbuf = 0, kRed = 2 * 8 * D * 16, kBc = kRed + 2 * NW * 32 * 8,
                            kTok = kBc + 2 * NW * 3 * 32 * 4, kBytes = kTok + 2 * kTokBytes;
};

template <int D, int TPR, typename TIn>
__global__ void __launch_bounds__(D * TPR, 1) bwd_kernel(BwdParams p)
{
    using Sh = BwdShape<D, TPR, TIn>;
    constexpr int NT = Sh::NT, NW = Sh::NW, CPT = Sh::CPT, NS = D / kCols;
    constexpr int LT = TPR == 1 ? 0 : TPR == 2 ? 1 : TPR == 4 ? 2 : 3;
    static_assert((1 << LT) == TPR && CPT % 4 == 0, "threads per row: 1, 2, 4 or 8");
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float4 *sbuf = reinterpret_cast<float4 *>(smem_raw + Sh::kSbuf);
    float2 *red = reinterpret_cast<float2 *>(smem_raw + Sh::kRed);
    float *bc = reinterpret_cast<float *>(smem_raw + Sh::kBc);

    const int H = p.H, gpc = p.gate_per_channel;
    const int per_rank = H * NS;
    const int rank = blockIdx.x / per_rank, rem = blockIdx.x - rank * per_rank;
    const int h = rem / NS, s = rem - h * NS;
    const int n = p.order[rank], unit = n * H + h;
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int r = tid >> LT, u = tid & (TPR - 1);  // row, part of the row
    const int cl = u * CPT + (lane >> LT);         // the column whose sums this lane holds
    const int j0 = s * kCols;
    const int at = r * TPR + u, stride = D * TPR;  // this thread's float4s in a state slice
    const int t0 = p.seq_start[n], t1 = p.seq_start[n + 1];
    const int c0 = p.chunk_off[n];
    const int nb = (t1 - t0 + kBlk - 1) / kBlk;
    float4 *blk = p.blk + (size_t)blockIdx.x * (kBlk + 1) * 8 * D;
    // block b of this sequence: two slots per 64-token chunk of the plan
    auto ckpt_at = [&](int b) { return p.ckpt + (((size_t)(2 * c0 + b) * H + h) * NS + s) * 8 * D; };
    auto bcast = [&](int par, int slot) { return bc + ((par * NW + w) * 3 + slot) * 32; };
    auto tokbuf = [&](int b) { return smem_raw + Sh::kTok + (b & 1) * Sh::kTokBytes; };

    // Copy block b's token data into its buffer (b & 1): the forward part (k,
    // log_alpha, v, beta) and/or the backward part (q, dO). Every thread issues
    // a share of the copies; a wait and a barrier make them visible.
    auto stage = [&](int b, bool fwd_part, bool bwd_part) {
        const int a = t0 + b * kBlk, nt = min(kBlk, t1 - a);
        unsigned char *base = tokbuf(b);
        constexpr int RP = D * (int)sizeof(TIn) / 16, VP = kCols * (int)sizeof(TIn) / 16, LP = D / 4;
        const char *gk = static_cast<const char *>(p.k), *gq = static_cast<const char *>(p.q);
        const char *gv = static_cast<const char *>(p.v), *gd = static_cast<const char *>(p.dO);
        for (int idx = tid; idx < nt * RP; idx += NT) {
            const int i = idx / RP, pc = idx - i * RP;
            const size_t off = ((size_t)(a + i) * H + h) * D * sizeof(TIn) + pc * 16;
            if (fwd_part) cp_async16(base + Sh::kTk + (size_t)idx * 16, gk + off);
            if (bwd_part) cp_async16(base + Sh::kTq + (size_t)idx * 16, gq + off);
        }
        for (int idx = tid; idx < nt * VP; idx += NT) {
            const int i = idx / VP, pc = idx - i * VP;
            const size_t off = (((size_t)(a + i) * H + h) * D + j0) * sizeof(TIn) + pc * 16;
            if (fwd_part) cp_async16(base + Sh::kTv + (size_t)idx * 16, gv + off);
            if (bwd_part) cp_async16(base + Sh::kTd + (size_t)idx * 16, gd + off);
        }
        if (fwd_part) {
            if (gpc) {
                for (int idx = tid; idx < nt * LP; idx += NT) {
                    const int i = idx / LP, pc = idx - i * LP;
                    cp_async16(base + Sh::kTla + (size_t)idx * 16,
                               p.log_alpha + ((size_t)(a + i) * H + h) * D + 4 * pc);
                }
            } else {
                for (int i = tid; i < nt; i += NT)
                    cp_async4(base + Sh::kTla + (size_t)i * D * 4, p.log_alpha + (size_t)(a + i) * H + h);
            }
            for (int i = tid; i < nt; i += NT)
                cp_async4(base + Sh::kTb + (size_t)i * 4, p.beta + (size_t)(a + i) * H + h);
        }
    };
    // token i of block b, from its staged buffer
    auto tok = [&](int b, int i, bool bwd_part) {
        const unsigned char *base = tokbuf(b);
        const TIn *tk = reinterpret_cast<const TIn *>(base + Sh::kTk);
        const TIn *tv = reinterpret_cast<const TIn *>(base + Sh::kTv);
        const float *tla = reinterpret_cast<const float *>(base + Sh::kTla);
        Tok x;
        x.k = to_f32(tk[i * D + r]);
        x.la = tla[i * D + (gpc ? r : 0)];
        x.v = to_f32(tv[i * kCols + cl]);
        x.b = reinterpret_cast<const float *>(base + Sh::kTb)[i];
        x.q = 0.f;
        x.d = 0.f;
        if (bwd_part) {
            x.q = to_f32(reinterpret_cast<const TIn *>(base + Sh::kTq)[i * D + r]);
            x.d = to_f32(reinterpret_cast<const TIn *>(base + Sh::kTd)[i * kCols + cl]);
        }
        return x;
    };
    // one forward token on the slice: S <- (I - b k k^T) Diag(alpha) S + b k v^T
    auto fwd = [&](float (&S)[CPT], const Tok &x, int par) {
        const float al = expf(x.la);
        float y[CPT];
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            S[j] *= al;
            y[j] = x.k * S[j];
        }
        red[(par * NW + w) * 32 + lane].x = reduce_scatter<CPT, TPR>(y, lane);
        __syncthreads();
        float ks = 0.f;
#pragma unroll
        for (int v = 0; v < NW; ++v) ks += red[(par * NW + v) * 32 + lane].x;
        float *wb = bcast(par, 1);
        wb[cl] = x.v - ks;
        __syncwarp();
        const float bk = x.b * x.k;
        const float4 *w4 = reinterpret_cast<const float4 *>(wb + u * CPT);
#pragma unroll
        for (int m = 0; m < CPT / 4; ++m) {
            const float4 wv = w4[m];
            S[4 * m] += bk * wv.x; S[4 * m + 1] += bk * wv.y;
            S[4 * m + 2] += bk * wv.z; S[4 * m + 3] += bk * wv.w;
        }
    };

    // 1. forward, keeping the state at every block start; block b + 1's token
    //    data is copied in while block b runs
    float S[CPT];
    const size_t dense = ((size_t)unit * D + r) * D + j0 + u * CPT;  // row r of S0, dS_final, dS0
    get_dense<CPT>(S, p.S0 ? p.S0 + dense : nullptr);
    if (nb > 0) stage(0, true, false);
    cp_async_commit();
    for (int b = 0; b < nb; ++b) {
        const int a = t0 + b * kBlk, e = min(a + kBlk, t1);
        cp_async_wait<0>();
        __syncthreads();  // block b staged and visible; block b - 1's buffer free
        if (b + 1 < nb) stage(b + 1, true, false);
        cp_async_commit();
        put_part<CPT>(ckpt_at(b), S, at, stride);
        for (int t = a; t < e; ++t) fwd(S, tok(b, t - a, false), t & 1);
    }
    float G[CPT];
    get_dense<CPT>(G, p.dS_final ? p.dS_final + dense : nullptr);

    // 2. blocks last to first: replay, then walk backwards. The last block's
    //    forward part is still staged; its q and dO are added.
    const float scale = p.scale;
    const size_t TH = p.TH;
    if (nb > 0) stage(nb - 1, false, true);
    cp_async_commit();
    for (int b = nb - 1; b >= 0; --b) {
        const int a = t0 + b * kBlk, e = min(a + kBlk, t1);
        cp_async_wait<0>();
        __syncthreads();  // block b staged and visible; the previous phase's shared reads are done
        if (b > 0) stage(b - 1, true, true);
        cp_async_commit();
        get_part<CPT>(S, ckpt_at(b), at, stride);
        put_part<CPT>(blk, S, at, stride);
        for (int t = a; t < e; ++t) {
            fwd(S, tok(b, t - a, false), t & 1);
            if (t + 1 < e) put_part<CPT>(blk + (size_t)(t - a + 1) * 8 * D, S, at, stride);
        }
        __syncthreads();  // replayed states written before they are copied back
        // S holds S_{e-1}. blk[i] is the state before token a + i; it goes to sbuf[i & 1].
        auto fetch = [&](int i) {
#pragma unroll
            for (int m = 0; m < CPT / 4; ++m)
                cp_async16(sbuf + (i & 1) * 8 * D + at + m * stride,
                           blk + (size_t)i * 8 * D + at + m * stride);
        };
        fetch(e - 1 - a);
        cp_async_commit();
        for (int t = e - 1; t >= a; --t) {
            const int i = t - a, par = t & 1;
            const size_t th = (size_t)t * H + h;
            if (i > 0) fetch(i - 1);  // S_{t-2} for the next step
            cp_async_commit();
            const Tok cur = tok(b, i, true);

            // read-out with S_t
            float *db = bcast(par, 0);
            db[cl] = cur.d;
            __syncwarp();
            {
                const float sq = scale * cur.q;
                const float4 *d4 = reinterpret_cast<const float4 *>(db + u * CPT);
                float dq0 = 0.f, dq1 = 0.f;
#pragma unroll
                for (int m = 0; m < CPT / 4; ++m) {
                    const float4 dv = d4[m];
                    G[4 * m] += sq * dv.x; G[4 * m + 1] += sq * dv.y;
                    G[4 * m + 2] += sq * dv.z; G[4 * m + 3] += sq * dv.w;
                    dq0 += S[4 * m] * dv.x + S[4 * m + 2] * dv.z;
                    dq1 += S[4 * m + 1] * dv.y + S[4 * m + 3] * dv.w;
                }
                const float dq = row_sum<TPR>(dq0 + dq1);
                if (u == 0) p.pq[((size_t)s * TH + th) * D + r] = scale * dq;
            }
            // S_{t-1}: this thread's own copies have landed
            cp_async_wait<1>();
            float P[CPT];
            get_part<CPT>(P, sbuf + (i & 1) * 8 * D, at, stride);
            // columns: w = v - S'^T k and g = G^T k, S' = Diag(alpha) S_{t-1}
            const float al = expf(cur.la), ak = al * cur.k;
            {
                float x[CPT], y[CPT];
#pragma unroll
                for (int j = 0; j < CPT; ++j) {
                    x[j] = ak * P[j];
                    y[j] = cur.k * G[j];
                }
                const float xs = reduce_scatter<CPT, TPR>(x, lane);
                const float ys = reduce_scatter<CPT, TPR>(y, lane);
                red[(par * NW + w) * 32 + lane] = make_float2(xs, ys);
            }
            __syncthreads();
            float *wb = bcast(par, 1), *gb = bcast(par, 2);
            {
                float ks = 0.f, gl = 0.f;
#pragma unroll
                for (int v = 0; v < NW; ++v) {
                    const float2 z = red[(par * NW + v) * 32 + lane];
                    ks += z.x;
                    gl += z.y;
                }
                wb[cl] = cur.v - ks;
                gb[cl] = gl;
                if (w == 0) p.gv[th * D + j0 + cl] = cur.b * gl;
            }
            __syncwarp();
            // rows: dk, dlog_alpha, then G <- Diag(alpha) dS'; warp 0 also dbeta
            {
                const float bk = cur.b * cur.k;
                const float4 *w4 = reinterpret_cast<const float4 *>(wb + u * CPT);
                const float4 *g4 = reinterpret_cast<const float4 *>(gb + u * CPT);
                float gw = 0.f, pg = 0.f, dl = 0.f, gw1 = 0.f, pg1 = 0.f, dl1 = 0.f, bb = 0.f;
#pragma unroll
                for (int m = 0; m < CPT / 4; ++m) {
                    const float4 wv = w4[m], gv = g4[m];
                    const float wj[4] = {wv.x, wv.y, wv.z, wv.w}, gj[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int j = 4 * m + q;
                        const float d = G[j] - bk * gj[q];
                        if (q & 1) {
                            gw1 += G[j] * wj[q];
                            pg1 += P[j] * gj[q];
                            dl1 += d * P[j];
                        } else {
                            gw += G[j] * wj[q];
                            pg += P[j] * gj[q];
                            dl += d * P[j];
                        }
                        bb += gj[q] * wj[q];
                        G[j] = al * d;
                    }
                }
                const size_t o = ((size_t)s * TH + th) * D + r;
                const float dk = row_sum<TPR>(cur.b * ((gw + gw1) - al * (pg + pg1)));
                const float dla = row_sum<TPR>(dl + dl1);
                if (u == 0) p.pk[o] = dk;
                if (u == TPR - 1) p.pla[o] = al * dla;
                if (w == 0) {
                    bb = row_sum<TPR>(bb);
                    if (tid == 0) p.pb[(size_t)s * TH + th] = bb;
                }
            }
#pragma unroll
            for (int j = 0; j < CPT; ++j) S[j] = P[j];  // S_{t-1} is the next step's S_t
        }
    }
    cp_async_wait<0>();
    if (p.gS0) {
        float4 *dst = reinterpret_cast<float4 *>(p.gS0 + dense);
#pragma unroll
        for (int m = 0; m < CPT / 4; ++m) dst[m] = make_float4(G[4 * m], G[4 * m + 1], G[4 * m + 2], G[4 * m + 3]);
    }
}

// Sums the per-slice partials in slice order: one warp per (token, head),
// tokens outside every sequence untouched. With one gate per head the
// log-gate derivative also sums over the dk rows.
template <int D>
__global__ void __launch_bounds__(256) bwd_reduce_kernel(BwdParams p, int NS, float *gq, float *gk,
                                                         float *gla, float *gbeta)
{
    const size_t H = (size_t)p.H, TH = p.TH;
    const size_t lo = (size_t)p.seq_start[0] * H, hi = (size_t)p.seq_start[p.N] * H;
    const int lane = threadIdx.x & 31;
    const size_t nwarps = ((size_t)gridDim.x * blockDim.x) >> 5;
    const float4 *pq = reinterpret_cast<const float4 *>(p.pq);
    const float4 *pk = reinterpret_cast<const float4 *>(p.pk);
    const float4 *pl = reinterpret_cast<const float4 *>(p.pla);
    constexpr int D4 = D / 4;
    for (size_t th = lo + (((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5); th < hi; th += nwarps) {
        float hsum = 0.f;
        for (int r4 = lane; r4 < D4; r4 += 32) {
            float4 aq = make_float4(0.f, 0.f, 0.f, 0.f), ak = aq, al = aq;
            for (int s = 0; s < NS; ++s) {
                const size_t off = ((size_t)s * TH + th) * D4 + r4;
                const float4 x = pq[off], y = pk[off], z = pl[off];
                aq.x += x.x; aq.y += x.y; aq.z += x.z; aq.w += x.w;
                ak.x += y.x; ak.y += y.y; ak.z += y.z; ak.w += y.w;
                al.x += z.x; al.y += z.y; al.z += z.z; al.w += z.w;
            }
            reinterpret_cast<float4 *>(gq)[th * D4 + r4] = aq;
            reinterpret_cast<float4 *>(gk)[th * D4 + r4] = ak;
            if (p.gate_per_channel) reinterpret_cast<float4 *>(gla)[th * D4 + r4] = al;
            else hsum += (al.x + al.y) + (al.z + al.w);
        }
        if (!p.gate_per_channel) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) hsum += __shfl_xor_sync(0xffffffffu, hsum, off);
            if (lane == 0) gla[th] = hsum;
        }
        if (lane == 0) {
            float b = 0.f;
            for (int s = 0; s < NS; ++s) b += p.pb[(size_t)s * TH + th];
            gbeta[th] = b;
        }
    }
}

template <int D, typename TIn>
cudaError_t launch_d(const BwdParams &p, float *gq, float *gk, float *gla, float *gbeta,
                     cudaStream_t st)
{
    constexpr int NS = D / kCols;
    using Sh = BwdShape<D, kTpr, TIn>;
    auto kern = bwd_kernel<D, kTpr, TIn>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Sh::kBytes);
    if (e != cudaSuccess) return e;
    const unsigned ctas = (unsigned)p.N * p.H * NS;
    kern<<<ctas, Sh::NT, Sh::kBytes, st>>>(p);
    note_launch();
    e = cudaGetLastError();
    if (e != cudaSuccess || p.TH == 0) return e;
    const unsigned grid = (unsigned)std::min<size_t>((p.TH + 7) / 8, (size_t)148 * 32);
    bwd_reduce_kernel<D><<<grid, 256, 0, st>>>(p, NS, gq, gk, gla, gbeta);
    note_launch();
    return cudaGetLastError();
}

// Byte offsets, after the plan, of the checkpoints, the replay buffers and the
// partials, and the floats of one partial array (pq, pk or pla).
struct BwdRegions {
    size_t ckpt, blk, part, part_floats;
};

BwdRegions bwd_regions(const Problem &pb)
{
    const int D = pb.dk, NS = D / kCols;
    BwdRegions g;
    g.ckpt = 0;
    g.blk = align_up(sizeof(float) * (size_t)D * D * 2 * pb.max_chunks * pb.H, 256);
    g.part = g.blk + align_up(sizeof(float) * (size_t)D * D * (kBlk + 1) * pb.N * pb.H, 256);
    g.part_floats = (size_t)NS * pb.total_tokens * pb.H * D;
    return g;
}

}  // namespace

WorkspaceLayout bwd_workspace_layout(const Problem &pb)
{
    const BwdRegions g = bwd_regions(pb);
    const size_t NS = (size_t)pb.dk / kCols;
    WorkspaceLayout l;
    l.plan_bytes = align_up(sizeof(int32_t) * plan_ints(pb.N), 256);
    l.chunk_bytes = g.part + 3 * align_up(sizeof(float) * g.part_floats, 256) +
                    align_up(sizeof(float) * NS * pb.total_tokens * pb.H, 256);
    l.total = l.plan_bytes + l.chunk_bytes;
    return l;
}

cudaError_t launch_backward(const Problem &pb, const void *dO, const float *dS_final,
                            float *gq, float *gk, float *gv, float *gla, float *gbeta,
                            float *gS0, void *workspace, cudaStream_t st)
{
    const WorkspaceLayout lay = bwd_workspace_layout(pb);
    const BwdRegions g = bwd_regions(pb);
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
    p.gv = gv; p.gS0 = gS0;
    p.TH = (size_t)pb.total_tokens * pb.H;
    p.seq_start = plan.seq_start; p.chunk_off = plan.chunk_off; p.order = plan.order;
    char *ws = static_cast<char *>(workspace) + lay.plan_bytes;
    const size_t part_bytes = align_up(sizeof(float) * g.part_floats, 256);
    p.ckpt = reinterpret_cast<float4 *>(ws + g.ckpt);
    p.blk = reinterpret_cast<float4 *>(ws + g.blk);
    p.pq = reinterpret_cast<float *>(ws + g.part);
    p.pk = reinterpret_cast<float *>(ws + g.part + part_bytes);
    p.pla = reinterpret_cast<float *>(ws + g.part + 2 * part_bytes);
    p.pb = reinterpret_cast<float *>(ws + g.part + 3 * part_bytes);
    const bool bf = pb.dtype == KDA_DTYPE_BF16;
    switch (pb.dk) {
    case 32: return bf ? launch_d<32, __nv_bfloat16>(p, gq, gk, gla, gbeta, st)
                       : launch_d<32, float>(p, gq, gk, gla, gbeta, st);
    case 64: return bf ? launch_d<64, __nv_bfloat16>(p, gq, gk, gla, gbeta, st)
                       : launch_d<64, float>(p, gq, gk, gla, gbeta, st);
    case 128: return bf ? launch_d<128, __nv_bfloat16>(p, gq, gk, gla, gbeta, st)
                        : launch_d<128, float>(p, gq, gk, gla, gbeta, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace kda
