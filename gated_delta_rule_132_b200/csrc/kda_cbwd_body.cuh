// kda_cbwd_body.cuh — chunk-parallel backward of the prefill: kernel bodies.
//
// Source: the KDA update rule of "Kimi Linear：让长上下文大模型真正实用的线性注意力架构"
// (juejin.cn), section 三 5️⃣, with the per-channel gate of section 三 1️⃣ and the
// read-out o_t = scale * S_t^T q_t. The pages state only the forward rule; the
// derivatives here are those of L = <dO, o> + <dS_final, S_final> taken through
// the exact chunked form of the rule (the form the SIMT prefill also uses).
// In a chunk of C tokens with entry state S and inclusive cumulative log-decay
// g (per channel), with E_rs = e^{g_r - g_s} (r >= s, so E <= 1):
//   A_rs = beta_r kk_rs, kk_rs = k_r.(E_rs k_s) (s < r);  Pm_rs = q_r.(E_rs k_s) (s <= r)
//   T = (I + A)^{-1},  W = T Diag(beta) (e^g k),  Ut = T Diag(beta) V,  U = Ut - W S
//   O = scale ((e^g q) S + Pm U),  S_end = Diag(e^{g_C}) S + (e^{g_C - g} k)^T U.
// Reverse, with G = dL/dS_end:
//   dU = scale Pm^T dO + (e^{g_C - g} k) G;   G_entry = scale (e^g q)^T dO + Diag(e^{g_C}) G - W^T dU
//   dPm = tril(scale dO U^T),  dW = -dU S^T,  X_V = T^T dU,  X_K = T^T dW,
//   dA = tril(-(X_V Ut^T + X_K W^T), -1),  dv = beta X_V,
//   dbeta = rowsum(X_V o V) + rowsum(X_K o e^g k) + rowsum(dA o kk),
//   X_r = sum_{s<=r} dPm_rs E_rs k_s,  Y_s = sum_{r>=s} dPm_rs E_rs q_r,
//   Z_r = beta_r sum_{s<r} dA_rs E_rs k_s,  R_s = sum_{r>s} beta_r dA_rs E_rs k_r,
//   Kt_s = e^{g_C - g_s} o (G U_s),
//   dq = scale e^g o (S dO) + X,  dk = beta e^g o X_K + Z + Y + R + Kt,
//   dg = q o dq + k o (dk - 2 (Y + R + Kt)), plus sum_s k_s o Kt_s + e^{g_C} o rowsum(G o S)
//   on the chunk's last token; dlog_alpha is the reverse cumulative sum of dg.
// Only exponentials of non-positive numbers appear, so any gate is safe.
//
// Phases: prep writes the per-chunk records (W, Ut, e^g q, e^{g_C-g} k,
// Pm, e^{g_C}); fwd_carry walks the chunks keeping each entry state S and U;
// bwd_carry walks them in reverse keeping each chunk's G and dU and returning
// dS0; grad_a forms the products with S and G for every chunk in parallel;
// grad_b does the rest per chunk.
//
// The bodies are written against an execution context X (tid(), block(),
// block_y(), sync()) so that one source serves the CUDA kernels and a host
// runner that executes every CUDA thread as a fiber.
#pragma once

#include <cuda_bf16.h>
#include <vector_types.h>
#include <math.h>
#include <stddef.h>
#include <stdint.h>

#if defined(__CUDACC__)
#define CB_HD __host__ __device__ __forceinline__
#define CB_UNROLL _Pragma("unroll")
#else
#define CB_HD inline
#define CB_UNROLL
#endif
// e^x for x <= 0 (every exponential in these bodies): the hardware intrinsic on
// the device (a few ulp, far inside the fp32 parity tolerance), expf on the host.
#if defined(__CUDA_ARCH__)
#define CB_EXP(x) __expf(x)
#else
#define CB_EXP(x) expf(x)
#endif

namespace kda {
namespace cbwd {

constexpr int C = 64;    // chunk length (tokens)
constexpr int WV = 32;   // value columns per carry CTA
constexpr int NT = 256;  // threads per CTA, every phase

CB_HD float cvt(float x) { return x; }
CB_HD float from_f(float x, float *) { return x; }
CB_HD __nv_bfloat16 from_f(float x, __nv_bfloat16 *) { return __float2bfloat16_rn(x); }
// Four consecutive floats from a 16-byte-aligned address.
CB_HD void ld4(float (&o)[4], const float *a)
{
    const float4 v = *reinterpret_cast<const float4 *>(a);
    o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}

// n floats (a multiple of 4, both ends 16-byte aligned) copied as float4 by
// the NT threads of a CTA.
template <int NTH>
CB_HD void copy4(float *dst, const float *src, int n, int tid)
{
    for (int i = tid; i < n / 4; i += NTH)
        reinterpret_cast<float4 *>(dst)[i] = reinterpret_cast<const float4 *>(src)[i];
}
CB_HD float cvt(__nv_bfloat16 x) { return __bfloat162float(x); }

// Floats of one prep record: W, Ut, Qt, Kh (C x D each), Pm (C x C), gamma (D).
template <int D> CB_HD constexpr size_t rec_floats() { return 4 * (size_t)C * D + C * C + D; }
// Floats of one grad_a scratch block: dW, UdS, dOS (C x D each), dPm (C x C), rsum (D).
template <int D> CB_HD constexpr size_t scr_floats() { return 3 * (size_t)C * D + C * C + D; }

template <int D> CB_HD constexpr size_t prep_smem() { return sizeof(float) * (3 * C * (D + 4) + C * D + C * C + C); }
// forward walk: two buffers of one chunk's W, K^, U~ slice and gamma, then U and S
template <int D> CB_HD constexpr size_t fwd_buf_floats() { return 2 * (size_t)C * D + C * WV + D; }
template <int D> CB_HD constexpr size_t fwd_carry_smem() { return sizeof(float) * (2 * fwd_buf_floats<D>() + C * WV + D * WV); }
// reverse walk: two buffers of one chunk's K^, P and gamma, then W, Q~, P^T, dO, dU and G
template <int D> CB_HD constexpr size_t bwd_buf_floats() { return (size_t)C * D + C * C + D; }
template <int D> CB_HD constexpr size_t bwd_carry_smem() { return sizeof(float) * (2 * bwd_buf_floats<D>() + 2 * C * D + C * C + 2 * C * WV + D * WV); }
template <int D> CB_HD constexpr size_t grad_a_smem() { return sizeof(float) * (3 * C * D + 2 * D * (D < 64 ? D : 64)); }
template <int D> CB_HD constexpr size_t grad_b_smem() { return sizeof(float) * (3 * C * (D + 4) + 2 * C * D + 2 * C * C + C); }

struct CbParams {
    const void *q, *k, *v, *dO;
    const float *log_alpha, *beta, *S0, *dS_final;
    int N, H, gate_per_channel;
    float scale;
    const int32_t *seq_start, *chunk_off, *order;
    const float *rec;   // prep records [chunks][H][rec_floats]
    float *Sst, *dSst;  // entry states, chunk-end gradients [chunks][H][D][D]
    float *Ust, *dUst;  // U and dU [chunks][H][C][D]
    float *scr;         // grad_a results [chunks][H][scr_floats]
    float *gq, *gk, *gv, *gla, *gbeta, *gS0;
};

// The sequence that global chunk c belongs to, or -1 past the last chunk.
CB_HD int seq_of_chunk(const int32_t *chunk_off, int N, int c)
{
    if (c >= chunk_off[N]) return -1;
    int lo = 0, hi = N - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (chunk_off[mid] <= c) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Per (chunk, head): the record the walks and grad_b read — W, Ut, Qt = e^g q,
// Kh = e^{g_C - g} k (C x D each), Pm (C x C, lower with diagonal), gamma =
// e^{g_C}, fp32 rows. A tail chunk is padded
// with identity tokens (k = q = v = 0, beta = 0, log_alpha = 0). The unit
// lower-triangular solve (I + A) [W | Ut] = Diag(beta) [e^g k | V] runs one
// column per thread with the column in registers and the rows of A read as float4.
template <int D, typename TIn, class X>
CB_HD void prep(const CbParams &p, X &x, float *smem, float *rec_out)
{
    constexpr int DP = D + 4;
    static_assert(2 * D <= NT, "one thread per solve column");
    float *sk = smem;            // [C][DP] k
    float *sq = sk + C * DP;     // [C][DP] q
    float *sg = sq + C * DP;     // [C][DP] g
    float *sv = sg + C * DP;     // [C][D]  v
    float *sA = sv + C * D;      // [C][C]  A (strictly lower, beta-scaled)
    float *sb = sA + C * C;      // [C]     beta
    const int c = x.block(), h = x.block_y(), H = p.H, tid = x.tid();
    const int n = seq_of_chunk(p.chunk_off, p.N, c);
    if (n < 0) return;
    const int t0 = p.seq_start[n] + (c - p.chunk_off[n]) * C;
    const int L = p.seq_start[n + 1] - t0 < C ? p.seq_start[n + 1] - t0 : C;
    const TIn *q = static_cast<const TIn *>(p.q), *k = static_cast<const TIn *>(p.k);
    const TIn *v = static_cast<const TIn *>(p.v);
    auto tok = [&](int r) { return ((size_t)(t0 + r) * H + h); };
    float *w = rec_out + ((size_t)c * H + h) * rec_floats<D>();
    float *wW = w, *wU = w + C * D, *wQ = w + 2 * C * D, *wK = w + 3 * C * D;
    float *wP = w + 4 * C * D, *wG = wP + C * C;

    for (int idx = tid; idx < C * D; idx += NT) {
        const int r = idx / D, i = idx % D;
        float kv = 0.f, qv = 0.f, vv = 0.f, la = 0.f;
        if (r < L) {
            kv = cvt(k[tok(r) * D + i]);
            qv = cvt(q[tok(r) * D + i]);
            vv = cvt(v[tok(r) * D + i]);
            la = p.gate_per_channel ? p.log_alpha[tok(r) * D + i] : p.log_alpha[tok(r)];
        }
        sk[r * DP + i] = kv;
        sq[r * DP + i] = qv;
        sv[idx] = vv;
        sg[r * DP + i] = la;
    }
    for (int r = tid; r < C; r += NT) sb[r] = r < L ? p.beta[tok(r)] : 0.f;
    x.sync();
    for (int i = tid; i < D; i += NT) {
        float acc = 0.f;
        for (int r = 0; r < C; ++r) {
            acc += sg[r * DP + i];
            sg[r * DP + i] = acc;
        }
    }
    x.sync();
    // A and Pm, four channels per step
    for (int idx = tid; idx < C * C; idx += NT) {
        const int r = idx / C, s2 = idx % C;
        float akk = 0.f, pqk = 0.f;
        if (s2 <= r)
            for (int i = 0; i < D; i += 4) {
                float kr[4], qr[4], ks[4], gr[4], gs[4];
                ld4(kr, sk + r * DP + i); ld4(qr, sq + r * DP + i); ld4(ks, sk + s2 * DP + i);
                ld4(gr, sg + r * DP + i); ld4(gs, sg + s2 * DP + i);
                for (int e = 0; e < 4; ++e) {
                    const float ke = ks[e] * CB_EXP(gr[e] - gs[e]);
                    akk += kr[e] * ke;
                    pqk += qr[e] * ke;
                }
            }
        sA[idx] = s2 < r ? sb[r] * akk : 0.f;
        wP[idx] = pqk;
    }
    for (int idx = tid; idx < C * D; idx += NT) {
        const int r = idx / D, i = idx % D;
        const float g = sg[r * DP + i], gC = sg[(C - 1) * DP + i];
        wQ[idx] = CB_EXP(g) * sq[r * DP + i];
        wK[idx] = CB_EXP(gC - g) * sk[r * DP + i];
    }
    for (int i = tid; i < D; i += NT) wG[i] = CB_EXP(sg[(C - 1) * DP + i]);
    x.sync();
    // forward substitution X_r = B_r - sum_{s<r} A_rs X_s, B = Diag(beta) [e^g k | V]
    if (tid < 2 * D) {
        const bool isk = tid < D;
        const int col = isk ? tid : tid - D;
        float xc[C];
        CB_UNROLL
        for (int r = 0; r < C; ++r)
            xc[r] = sb[r] * (isk ? sk[r * DP + col] * CB_EXP(sg[r * DP + col]) : sv[r * D + col]);
        CB_UNROLL
        for (int r = 1; r < C; ++r) {
            float acc = xc[r];
            CB_UNROLL
            for (int s4 = 0; s4 < r; s4 += 4) {
                float a[4];
                ld4(a, sA + r * C + s4);
                CB_UNROLL
                for (int e = 0; e < 4; ++e)
                    if (s4 + e < r) acc -= a[e] * xc[s4 + e];
            }
            xc[r] = acc;
        }
        float *out = isk ? wW : wU;
        CB_UNROLL
        for (int r = 0; r < C; ++r) out[r * D + col] = xc[r];
    }
}

// Forward walk over one (sequence, head, 32-column slice): keeps S at every
// chunk entry and U = Ut - W S. Thread (grp, j) owns column j; it forms U for
// rows grp + 8 m and updates the state rows 16 grp .. 16 grp + 15, reading
// the shared row operands (W, K^) as float4. The next chunk's W, K^, U~
// slice and gamma arrive by asynchronous copies into the other of two
// buffers while this chunk computes.
template <int D, class X>
CB_HD void fwd_carry(const CbParams &p, X &x, float *smem)
{
    constexpr int NS = D / WV, NG = NT / WV, RPG = D / NG;  // state rows per group
    static_assert(RPG % 4 == 0 && RPG >= 4, "state rows per thread group");
    constexpr size_t RS = rec_floats<D>();
    constexpr size_t BUF = fwd_buf_floats<D>();
    float *sU = smem + 2 * BUF, *sS = sU + C * WV;
    const int H = p.H, bx = x.block();
    const int j0 = (bx % NS) * WV, h = (bx / NS) % H, n = p.order[bx / (NS * H)];
    const int tid = x.tid(), j = tid % WV, grp = tid / WV, i0 = grp * RPG;
    const size_t sbase = ((size_t)n * H + h) * D * D;
    const int c0 = p.chunk_off[n], nc = p.chunk_off[n + 1] - c0;
    // chunk lc's operands into buffer b, as one group of 16-byte copies
    auto fetch = [&](int lc, int b) {
        const float *w = p.rec + ((size_t)(c0 + lc) * H + h) * RS;
        float *bW = smem + b * BUF, *bK = bW + C * D, *bUt = bK + C * D, *bG = bUt + C * WV;
        for (int i = tid; i < C * D / 4; i += NT) {
            x.cp16(bW + 4 * i, w + 4 * i);
            x.cp16(bK + 4 * i, w + 3 * C * D + 4 * i);
        }
        for (int i = tid; i < C * WV / 4; i += NT) {
            const int r = i / (WV / 4), q4 = i % (WV / 4);
            x.cp16(bUt + r * WV + 4 * q4, w + C * D + (size_t)r * D + j0 + 4 * q4);
        }
        for (int i = tid; i < D / 4; i += NT) x.cp16(bG + 4 * i, w + 4 * C * D + C * C + 4 * i);
        x.cp_commit();
    };
    for (int i = i0; i < i0 + RPG; ++i) sS[i * WV + j] = p.S0 ? p.S0[sbase + (size_t)i * D + j0 + j] : 0.f;
    if (nc > 0) fetch(0, 0);
    for (int lc = 0; lc < nc; ++lc) {
        const int b = lc & 1;
        const size_t ch = (size_t)(c0 + lc) * H + h;
        const float *sW = smem + b * BUF, *sK = sW + C * D, *sUt = sK + C * D, *sG = sUt + C * WV;
        float *Sst = p.Sst + ch * D * D, *Ust = p.Ust + ch * C * D;
        for (int i = i0; i < i0 + RPG; ++i) Sst[(size_t)i * D + j0 + j] = sS[i * WV + j];
        x.sync();  // the previous chunk is done with the other buffer, U and S
        if (lc + 1 < nc) {
            fetch(lc + 1, b ^ 1);
            x.cp_wait(1);  // this chunk's group has landed; the next one may still fly
        } else {
            x.cp_wait(0);
        }
        x.sync();
        {
            float acc[C / NG];
            for (int m = 0; m < C / NG; ++m) acc[m] = sUt[(grp + NG * m) * WV + j];
            for (int i = 0; i < D; i += 4) {
                const float s0 = sS[i * WV + j], s1 = sS[(i + 1) * WV + j];
                const float s2 = sS[(i + 2) * WV + j], s3 = sS[(i + 3) * WV + j];
                for (int m = 0; m < C / NG; ++m) {
                    float wv[4];
                    ld4(wv, sW + (grp + NG * m) * D + i);
                    acc[m] -= wv[0] * s0 + wv[1] * s1 + wv[2] * s2 + wv[3] * s3;
                }
            }
            for (int m = 0; m < C / NG; ++m) {
                const int r = grp + NG * m;
                sU[r * WV + j] = acc[m];
                Ust[(size_t)r * D + j0 + j] = acc[m];
            }
        }
        x.sync();
        {
            float acc[RPG];
            for (int m = 0; m < RPG; ++m) acc[m] = sG[i0 + m] * sS[(i0 + m) * WV + j];
            for (int r = 0; r < C; ++r) {
                const float u = sU[r * WV + j];
                for (int m = 0; m < RPG; m += 4) {
                    float kv[4];
                    ld4(kv, sK + r * D + i0 + m);
                    acc[m] += kv[0] * u; acc[m + 1] += kv[1] * u;
                    acc[m + 2] += kv[2] * u; acc[m + 3] += kv[3] * u;
                }
            }
            for (int m = 0; m < RPG; ++m) sS[(i0 + m) * WV + j] = acc[m];
        }
    }
}

// Reverse walk over one (sequence, head, 32-column slice): keeps G (the gradient
// at each chunk's end) and dU, and returns the slice of dS0. Same thread layout
// as the forward walk; Pm is kept transposed so its column reads are float4.
// The operands of the dU step (K^, P, gamma) come one chunk ahead into the
// other of two buffers, and dO one chunk ahead into registers; W and Q~,
// needed only by the G step, are copied at the start of the chunk and land
// while the dU step runs.
template <int D, typename TIn, class X>
CB_HD void bwd_carry(const CbParams &p, X &x, float *smem)
{
    constexpr int NS = D / WV, NG = NT / WV, RPG = D / NG;
    static_assert(RPG % 4 == 0 && RPG >= 4, "state rows per thread group");
    constexpr size_t RS = rec_floats<D>();
    constexpr size_t BUF = bwd_buf_floats<D>();
    constexpr int DOPT = C * WV / NT;  // dO values per thread
    static_assert(C * WV % NT == 0, "dO slice per thread");
    float *sW = smem + 2 * BUF, *sQ = sW + C * D, *sPt = sQ + C * D;
    float *sdO = sPt + C * C, *sdU = sdO + C * WV, *sG = sdU + C * WV;
    const int H = p.H, bx = x.block();
    const int j0 = (bx % NS) * WV, h = (bx / NS) % H, n = p.order[bx / (NS * H)];
    const int tid = x.tid(), j = tid % WV, grp = tid / WV, i0 = grp * RPG;
    const size_t sbase = ((size_t)n * H + h) * D * D;
    const TIn *dO = static_cast<const TIn *>(p.dO);
    const float scale = p.scale;
    for (int i = i0; i < i0 + RPG; ++i)
        sG[i * WV + j] = p.dS_final ? p.dS_final[sbase + (size_t)i * D + j0 + j] : 0.f;
    const int ts = p.seq_start[n], te = p.seq_start[n + 1];
    const int c0 = p.chunk_off[n], nc = p.chunk_off[n + 1] - c0;
    auto rec_of = [&](int lc) { return p.rec + ((size_t)(c0 + lc) * H + h) * RS; };
    // chunk lc's K^, P and gamma into buffer b, as one group
    auto fetch = [&](int lc, int b) {
        const float *w = rec_of(lc);
        float *bK = smem + b * BUF, *bP = bK + C * D, *bg = bP + C * C;
        for (int i = tid; i < C * D / 4; i += NT) x.cp16(bK + 4 * i, w + 3 * C * D + 4 * i);
        for (int i = tid; i < C * C / 4; i += NT) x.cp16(bP + 4 * i, w + 4 * C * D + 4 * i);
        for (int i = tid; i < D / 4; i += NT) x.cp16(bg + 4 * i, w + 4 * C * D + C * C + 4 * i);
        x.cp_commit();
    };
    // chunk lc's dO slice (zero past the sequence's end) into registers
    float dOr[DOPT];
    auto load_dO = [&](int lc) {
        const int t0 = ts + lc * C, L = te - t0 < C ? te - t0 : C;
        for (int e = 0; e < DOPT; ++e) {
            const int idx = tid + NT * e, r = idx / WV, jj = idx % WV;
            dOr[e] = r < L ? cvt(dO[((size_t)(t0 + r) * H + h) * D + j0 + jj]) : 0.f;
        }
    };
    if (nc > 0) {
        fetch(nc - 1, (nc - 1) & 1);
        load_dO(nc - 1);
    }
    for (int lc = nc - 1; lc >= 0; --lc) {
        const int b = lc & 1;
        const size_t ch = (size_t)(c0 + lc) * H + h;
        const float *w = rec_of(lc);
        const float *sK = smem + b * BUF, *sP = sK + C * D, *sgam = sP + C * C;
        float *dSst = p.dSst + ch * D * D, *dUst = p.dUst + ch * C * D;
        for (int i = i0; i < i0 + RPG; ++i) dSst[(size_t)i * D + j0 + j] = sG[i * WV + j];
        x.sync();  // the previous chunk is done with W, Q~, P^T, dO, dU and the other buffer
        for (int i = tid; i < C * D / 4; i += NT) {
            x.cp16(sW + 4 * i, w + 4 * i);
            x.cp16(sQ + 4 * i, w + 2 * C * D + 4 * i);
        }
        x.cp_commit();
        if (lc > 0) fetch(lc - 1, b ^ 1);
        else x.cp_commit();  // an empty group keeps the count of groups in flight
        x.cp_wait(2);        // this chunk's K^, P and gamma have landed
        for (int e = 0; e < DOPT; ++e) sdO[tid + NT * e] = dOr[e];
        x.sync();
        for (int idx = tid; idx < C * C; idx += NT) sPt[(idx % C) * C + idx / C] = sP[idx];
        if (lc > 0) load_dO(lc - 1);
        x.sync();
        {
            float acc[C / NG], pa[C / NG];
            for (int m = 0; m < C / NG; ++m) acc[m] = pa[m] = 0.f;
            // scale * sum_{s >= r} Pm_sr dO_s (Pm is lower triangular, so s < r adds zero)
            for (int s = 0; s < C; s += 4) {
                const float d0 = sdO[s * WV + j], d1 = sdO[(s + 1) * WV + j];
                const float d2 = sdO[(s + 2) * WV + j], d3 = sdO[(s + 3) * WV + j];
                for (int m = 0; m < C / NG; ++m) {
                    float pv[4];
                    ld4(pv, sPt + (grp + NG * m) * C + s);
                    pa[m] += pv[0] * d0 + pv[1] * d1 + pv[2] * d2 + pv[3] * d3;
                }
            }
            for (int i = 0; i < D; i += 4) {
                const float g0 = sG[i * WV + j], g1 = sG[(i + 1) * WV + j];
                const float g2 = sG[(i + 2) * WV + j], g3 = sG[(i + 3) * WV + j];
                for (int m = 0; m < C / NG; ++m) {
                    float kv[4];
                    ld4(kv, sK + (grp + NG * m) * D + i);
                    acc[m] += kv[0] * g0 + kv[1] * g1 + kv[2] * g2 + kv[3] * g3;
                }
            }
            for (int m = 0; m < C / NG; ++m) {
                const int r = grp + NG * m;
                const float du = scale * pa[m] + acc[m];
                sdU[r * WV + j] = du;
                dUst[(size_t)r * D + j0 + j] = du;
            }
        }
        x.cp_wait(1);  // W and Q~ have landed (the next chunk's group may still fly)
        x.sync();
        {
            float qd[RPG], wd[RPG];
            for (int m = 0; m < RPG; ++m) qd[m] = wd[m] = 0.f;
            for (int r = 0; r < C; ++r) {
                const float d = sdO[r * WV + j], du = sdU[r * WV + j];
                for (int m = 0; m < RPG; m += 4) {
                    float qv[4], wv[4];
                    ld4(qv, sQ + r * D + i0 + m);
                    ld4(wv, sW + r * D + i0 + m);
                    for (int e = 0; e < 4; ++e) {
                        qd[m + e] += qv[e] * d;
                        wd[m + e] += wv[e] * du;
                    }
                }
            }
            for (int m = 0; m < RPG; ++m) {
                const int i = i0 + m;
                sG[i * WV + j] = scale * qd[m] + sgam[i] * sG[i * WV + j] - wd[m];
            }
        }
    }
    x.cp_wait(0);
    if (p.gS0)
        for (int i = i0; i < i0 + RPG; ++i) p.gS0[sbase + (size_t)i * D + j0 + j] = sG[i * WV + j];
}

// Per (chunk, head): the products with the chunk's entry state S and end
// gradient G — dW = -dU S^T, UdS = U G^T, dOS = dO S^T, rowsum(G o S) — and dPm.
// Operands sit transposed in shared memory ([j][row]) so that every thread
// computes a 4 x 4 block of outputs from float4 loads (8 loads per 16 FMAs
// and product).
template <int D, typename TIn, class X>
CB_HD void grad_a(const CbParams &p, X &x, float *smem)
{
    constexpr int TJ = D < 64 ? D : 64;  // state rows per tile
    constexpr int CB = TJ / 4;           // 4-column blocks per tile
    static_assert(16 * CB <= NT && 16 * 16 <= NT, "one 4 x 4 block per thread");
    float *uT = smem, *duT = uT + D * C, *doT = duT + D * C, *sT = doT + D * C, *gT = sT + D * TJ;
    const int c = x.block(), h = x.block_y(), H = p.H, tid = x.tid();
    const int n = seq_of_chunk(p.chunk_off, p.N, c);
    if (n < 0) return;
    const int t0 = p.seq_start[n] + (c - p.chunk_off[n]) * C;
    const int L = p.seq_start[n + 1] - t0 < C ? p.seq_start[n + 1] - t0 : C;
    const size_t ch = (size_t)c * H + h;
    const TIn *dO = static_cast<const TIn *>(p.dO);
    const float *Ug = p.Ust + ch * C * D, *dUg = p.dUst + ch * C * D;
    for (int idx = tid; idx < C * D; idx += NT) {
        const int r = idx / D, jj = idx % D;
        uT[jj * C + r] = Ug[idx];
        duT[jj * C + r] = dUg[idx];
        doT[jj * C + r] = r < L ? cvt(dO[((size_t)(t0 + r) * H + h) * D + jj]) : 0.f;
    }
    float *scr = p.scr + ch * scr_floats<D>();
    float *dW = scr, *UdS = scr + C * D, *dOS = scr + 2 * C * D, *dPm = scr + 3 * C * D;
    float *rsum = dPm + C * C;
    const float *S = p.Sst + ch * D * D, *G = p.dSst + ch * D * D;
    const int rb = tid / CB, ib = tid % CB;  // rows 4 rb .. 4 rb + 3, tile columns 4 ib .. + 3
    for (int i0 = 0; i0 < D; i0 += TJ) {
        x.sync();  // the previous tile is done (and, first time, the loads above)
        for (int idx = tid; idx < TJ * D; idx += NT) {
            const int ii = idx / D, jj = idx % D;
            sT[jj * TJ + ii] = S[(size_t)(i0 + ii) * D + jj];
            gT[jj * TJ + ii] = G[(size_t)(i0 + ii) * D + jj];
        }
        x.sync();
        if (tid < 16 * CB) {
            float a[4][4] = {}, b[4][4] = {}, e[4][4] = {};
            for (int jj = 0; jj < D; ++jj) {
                float u[4], du[4], d[4], sv[4], gv[4];
                ld4(u, uT + jj * C + 4 * rb);
                ld4(du, duT + jj * C + 4 * rb);
                ld4(d, doT + jj * C + 4 * rb);
                ld4(sv, sT + jj * TJ + 4 * ib);
                ld4(gv, gT + jj * TJ + 4 * ib);
                for (int m = 0; m < 4; ++m)
                    for (int q = 0; q < 4; ++q) {
                        a[m][q] += du[m] * sv[q];
                        b[m][q] += u[m] * gv[q];
                        e[m][q] += d[m] * sv[q];
                    }
            }
            for (int m = 0; m < 4; ++m)
                for (int q = 0; q < 4; ++q) {
                    const int o = (4 * rb + m) * D + i0 + 4 * ib + q;
                    dW[o] = -a[m][q];
                    UdS[o] = b[m][q];
                    dOS[o] = e[m][q];
                }
        }
        for (int ii = tid; ii < TJ; ii += NT) {
            float acc = 0.f;
            for (int jj = 0; jj < D; ++jj) acc += gT[jj * TJ + ii] * sT[jj * TJ + ii];
            rsum[i0 + ii] = acc;
        }
    }
    // dPm = tril(scale dO U^T): 16 x 16 blocks of 4 x 4
    {
        const int pr = tid / 16, ps = tid % 16;
        float acc[4][4] = {};
        for (int jj = 0; jj < D; ++jj) {
            float d[4], u[4];
            ld4(d, doT + jj * C + 4 * pr);
            ld4(u, uT + jj * C + 4 * ps);
            for (int m = 0; m < 4; ++m)
                for (int q = 0; q < 4; ++q) acc[m][q] += d[m] * u[q];
        }
        for (int m = 0; m < 4; ++m)
            for (int q = 0; q < 4; ++q) {
                const int r = 4 * pr + m, s2 = 4 * ps + q;
                dPm[r * C + s2] = s2 <= r ? p.scale * acc[m][q] : 0.f;
            }
    }
}

// Per (chunk, head): the triangular solves, dA, dv, dbeta, the pairwise-decayed
// contractions, dq, dk and dlog_alpha. Row buffers read as float4 by many rows
// at once (k, g, the staged operand) have a padded stride of D + 4 floats.
template <int D, typename TIn, class X>
CB_HD void grad_b(const CbParams &p, X &x, float *smem)
{
    constexpr int DP = D + 4, D4 = D / 4;
    static_assert(2 * D <= NT && C <= NT && 16 * 16 <= NT, "thread mapping");
    float *sk = smem;            // [C][DP] k
    float *sg = sk + C * DP;     // [C][DP] g, the inclusive cumulative log-decay
    float *st = sg + C * DP;     // [C][DP] staging: Ut, then W, then v, then q
    float *sXV = st + C * DP;    // [C][D] X_V, then the partial dk
    float *sXK = sXV + C * D;    // [C][D] X_K, then dq, then dg and dlog_alpha
    float *skk = sXK + C * D;    // [C][C] kk, then dPm
    float *sdA = skk + C * C;    // [C][C] A^T during the solves, then dA
    float *sb = sdA + C * C;     // [C] beta
    const int c = x.block(), h = x.block_y(), H = p.H, tid = x.tid();
    const int n = seq_of_chunk(p.chunk_off, p.N, c);
    if (n < 0) return;
    const int t0 = p.seq_start[n] + (c - p.chunk_off[n]) * C;
    const int L = p.seq_start[n + 1] - t0 < C ? p.seq_start[n + 1] - t0 : C;
    const size_t ch = (size_t)c * H + h;
    const TIn *q = static_cast<const TIn *>(p.q), *k = static_cast<const TIn *>(p.k);
    const TIn *v = static_cast<const TIn *>(p.v);
    const float *w = p.rec + ch * rec_floats<D>();
    const float *scr = p.scr + ch * scr_floats<D>();
    const float *dW = scr, *UdS = scr + C * D, *dOS = scr + 2 * C * D, *dPm = scr + 3 * C * D;
    const float *rsum = dPm + C * C;
    const float scale = p.scale;
    auto tok = [&](int r) { return ((size_t)(t0 + r) * H + h); };

    // 1. k, log_alpha -> g, beta (padded tokens: zero, identity), dU, dW
    for (int idx = tid; idx < C * D; idx += NT) {
        const int r = idx / D, i = idx % D;
        float kv = 0.f, la = 0.f;
        if (r < L) {
            kv = cvt(k[tok(r) * D + i]);
            la = p.gate_per_channel ? p.log_alpha[tok(r) * D + i] : p.log_alpha[tok(r)];
        }
        sk[r * DP + i] = kv;
        sg[r * DP + i] = la;
        sXV[idx] = p.dUst[ch * C * D + idx];
        sXK[idx] = dW[idx];
    }
    for (int r = tid; r < C; r += NT) sb[r] = r < L ? p.beta[tok(r)] : 0.f;
    x.sync();
    for (int i = tid; i < D; i += NT) {
        float acc = 0.f;
        for (int r = 0; r < C; ++r) {
            acc += sg[r * DP + i];
            sg[r * DP + i] = acc;
        }
    }
    x.sync();
    // 2. kk (strictly lower), four channels per step
    for (int idx = tid; idx < C * C; idx += NT) {
        const int r = idx / C, s2 = idx % C;
        float a = 0.f;
        if (s2 < r)
            for (int i = 0; i < D; i += 4) {
                float kr[4], ks[4], gr[4], gs[4];
                ld4(kr, sk + r * DP + i); ld4(ks, sk + s2 * DP + i);
                ld4(gr, sg + r * DP + i); ld4(gs, sg + s2 * DP + i);
                for (int e = 0; e < 4; ++e) a += kr[e] * ks[e] * CB_EXP(gr[e] - gs[e]);
            }
        skk[idx] = a;
    }
    x.sync();
    // 3. X_V = T^T dU and X_K = T^T dW: back substitution with (I + A)^T, one
    //    column per thread held in registers, A^T[r][s] = beta_s kk_sr read as float4
    for (int idx = tid; idx < C * C; idx += NT) {
        const int r = idx / C, s2 = idx % C;
        sdA[idx] = sb[s2] * skk[s2 * C + r];
    }
    x.sync();
    if (tid < 2 * D) {
        float *col = tid < D ? sXV + tid : sXK + (tid - D);
        float xc[C];
        CB_UNROLL
        for (int r = 0; r < C; ++r) xc[r] = col[r * D];
        CB_UNROLL
        for (int r = C - 2; r >= 0; --r) {
            float acc = xc[r];
            CB_UNROLL
            for (int s4 = (r + 1) & ~3; s4 < C; s4 += 4) {
                float a[4];
                ld4(a, sdA + r * C + s4);
                CB_UNROLL
                for (int e = 0; e < 4; ++e)
                    if (s4 + e > r) acc -= a[e] * xc[s4 + e];
            }
            xc[r] = acc;
        }
        CB_UNROLL
        for (int r = 0; r < C; ++r) col[r * D] = xc[r];
    }
    x.sync();
    // 4. dA = tril(-(X_V Ut^T + X_K W^T), -1) in 4 x 4 blocks, one staged operand at a time
    for (int idx = tid; idx < C * D; idx += NT) st[(idx / D) * DP + idx % D] = w[C * D + idx];  // Ut
    x.sync();
    const int rb = tid / 16, cb = tid % 16;
    const bool live = tid < 256 && cb <= rb;
    float dacc[4][4] = {};
    if (live)
        for (int jj = 0; jj < D; jj += 4) {
            float xr[4][4], us[4][4];
            for (int m = 0; m < 4; ++m) {
                ld4(xr[m], sXV + (4 * rb + m) * D + jj);
                ld4(us[m], st + (4 * cb + m) * DP + jj);
            }
            for (int m = 0; m < 4; ++m)
                for (int q2 = 0; q2 < 4; ++q2)
                    dacc[m][q2] += xr[m][0] * us[q2][0] + xr[m][1] * us[q2][1] +
                                   xr[m][2] * us[q2][2] + xr[m][3] * us[q2][3];
        }
    x.sync();
    for (int idx = tid; idx < C * D; idx += NT) st[(idx / D) * DP + idx % D] = w[idx];  // W
    x.sync();
    if (live)
        for (int ii = 0; ii < D; ii += 4) {
            float xr[4][4], ws[4][4];
            for (int m = 0; m < 4; ++m) {
                ld4(xr[m], sXK + (4 * rb + m) * D + ii);
                ld4(ws[m], st + (4 * cb + m) * DP + ii);
            }
            for (int m = 0; m < 4; ++m)
                for (int q2 = 0; q2 < 4; ++q2)
                    dacc[m][q2] += xr[m][0] * ws[q2][0] + xr[m][1] * ws[q2][1] +
                                   xr[m][2] * ws[q2][2] + xr[m][3] * ws[q2][3];
        }
    if (tid < 256)
        for (int m = 0; m < 4; ++m)
            for (int q2 = 0; q2 < 4; ++q2) {
                const int r = 4 * rb + m, s2 = 4 * cb + q2;
                sdA[r * C + s2] = s2 < r ? -dacc[m][q2] : 0.f;
            }
    x.sync();
    // 5. dv, dbeta
    for (int idx = tid; idx < C * D; idx += NT) {
        const int r = idx / D;
        st[r * DP + idx % D] = r < L ? cvt(v[tok(r) * D + idx % D]) : 0.f;
    }
    x.sync();
    for (int idx = tid; idx < C * D; idx += NT) {
        const int r = idx / D;
        if (r < L) p.gv[tok(r) * D + idx % D] = sb[r] * sXV[idx];
    }
    for (int r = tid; r < C; r += NT) {
        float a = 0.f;
        for (int i = 0; i < D; ++i)
            a += sXV[r * D + i] * st[r * DP + i] + sXK[r * D + i] * sk[r * DP + i] * CB_EXP(sg[r * DP + i]);
        for (int s2 = 0; s2 < r; ++s2) a += sdA[r * C + s2] * skk[r * C + s2];
        if (r < L) p.gbeta[tok(r)] = a;
    }
    x.sync();
    // 6. q and dPm
    for (int idx = tid; idx < C * D; idx += NT) {
        const int r = idx / D;
        st[r * DP + idx % D] = r < L ? cvt(q[tok(r) * D + idx % D]) : 0.f;
    }
    for (int idx = tid; idx < C * C; idx += NT) skk[idx] = dPm[idx];
    x.sync();
    const float *sq = st, *sdP = skk;
    // 7. per (r, 4 channels): X, Z -> dq and the partial dk = beta e^g X_K + Z + Kt
    for (int idx = tid; idx < C * D4; idx += NT) {
        const int r = idx / D4, i0 = 4 * (idx % D4);
        float gr[4], xr[4] = {}, zr[4] = {};
        ld4(gr, sg + r * DP + i0);
        for (int s2 = 0; s2 <= r; ++s2) {
            float gs[4], ks[4];
            ld4(gs, sg + s2 * DP + i0);
            ld4(ks, sk + s2 * DP + i0);
            const float dp = sdP[r * C + s2], da = s2 < r ? sdA[r * C + s2] : 0.f;
            for (int e = 0; e < 4; ++e) {
                const float ee = CB_EXP(gr[e] - gs[e]) * ks[e];
                xr[e] += dp * ee;
                zr[e] += da * ee;
            }
        }
        for (int e = 0; e < 4; ++e) {
            const int i = i0 + e, o = r * D + i;
            const float eg = CB_EXP(gr[e]), Kt = CB_EXP(sg[(C - 1) * DP + i] - gr[e]) * UdS[o];
            const float dq = scale * eg * dOS[o] + xr[e];
            sXV[o] = sb[r] * eg * sXK[o] + sb[r] * zr[e] + Kt;
            sXK[o] = dq;
        }
    }
    x.sync();
    // 8. per (s, 4 channels): Y, R -> dk, dq out; dg kept
    for (int idx = tid; idx < C * D4; idx += NT) {
        const int s2 = idx / D4, i0 = 4 * (idx % D4);
        float gs[4], ys[4] = {}, rs[4] = {};
        ld4(gs, sg + s2 * DP + i0);
        for (int r = s2; r < C; ++r) {
            float gr[4], qr[4], kr[4];
            ld4(gr, sg + r * DP + i0);
            ld4(qr, sq + r * DP + i0);
            ld4(kr, sk + r * DP + i0);
            const float dp = sdP[r * C + s2], da = r > s2 ? sb[r] * sdA[r * C + s2] : 0.f;
            for (int e = 0; e < 4; ++e) {
                const float ee = CB_EXP(gr[e] - gs[e]);
                ys[e] += dp * ee * qr[e];
                rs[e] += da * ee * kr[e];
            }
        }
        for (int e = 0; e < 4; ++e) {
            const int i = i0 + e, o = s2 * D + i;
            const float Kt = CB_EXP(sg[(C - 1) * DP + i] - gs[e]) * UdS[o];
            const float dk = sXV[o] + ys[e] + rs[e], dq = sXK[o];
            if (s2 < L) {
                p.gq[tok(s2) * D + i] = dq;
                p.gk[tok(s2) * D + i] = dk;
            }
            sXK[o] = sq[s2 * DP + i] * dq + sk[s2 * DP + i] * (dk - 2.f * (ys[e] + rs[e] + Kt));
        }
    }
    x.sync();
    // 9. last-token terms, then the reverse cumulative sum over the chunk
    if (tid < D) {
        const int i = tid;
        const float gC = sg[(C - 1) * DP + i];
        float extra = CB_EXP(gC) * rsum[i];
        for (int s2 = 0; s2 < C; ++s2) extra += sk[s2 * DP + i] * CB_EXP(gC - sg[s2 * DP + i]) * UdS[s2 * D + i];
        sXK[(C - 1) * D + i] += extra;
        float acc = 0.f;
        for (int r = C - 1; r >= 0; --r) {
            acc += sXK[r * D + i];
            sXK[r * D + i] = acc;
            if (p.gate_per_channel && r < L) p.gla[tok(r) * D + i] = acc;
        }
    }
    if (!p.gate_per_channel) {
        x.sync();
        for (int r = tid; r < L; r += NT) {
            float a = 0.f;
            for (int i = 0; i < D; ++i) a += sXK[r * D + i];
            p.gla[tok(r)] = a;
        }
    }
}

}  // namespace cbwd
}  // namespace kda
