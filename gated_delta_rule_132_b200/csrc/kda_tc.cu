// kda_tc.cu — chunked KDA prefill on the tcgen05 tensor cores (bf16 q/k/v,
// dk = dv = 128, fp32 gates and state).
//
// Source: the KDA update rule of "Kimi Linear：让长上下文大模型真正实用的线性注意力架构"
// (juejin.cn), section 三 5️⃣, with the per-channel gate of section 三 1️⃣ and the
// read-out o_t = scale * S_t^T q_t. The chunked form (64-token chunks) is the one
// derived in kda_simt.cu: per chunk, with entry state S,
//     U = U~ - W S,   O = scale (Q~ S + P U),   S <- Diag(gamma) S + K^^T U,
// where W, U~ = (I + A)^{-1} Diag(beta) [K~ | V], and Q~, K^, P, gamma carry the
// per-channel decay inside the chunk.
//
// Two kernels:
//  * prep (chunk-parallel, one CTA per chunk and head) computes the chunk's
//    matrices and writes them to the workspace as a ready-made shared-memory
//    image: bf16 operands already in the 128-byte-swizzled UMMA layouts, fp32
//    gamma and U~. One record per (chunk, head), see Record below.
//  * carry (sequential, one CTA per sequence, head and 64-column half of the
//    value dimension; the value columns of S never mix) walks the chunks in
//    order. Warp 8 streams each record into a two-stage shared-memory ring
//    with bulk async copies; warp 9 issues the tcgen05 MMAs; warps 0-7 own the
//    transposed state slice S^T (fp32, in registers), read the accumulators out
//    of TMEM and write the bf16 operands the next MMA needs:
//        MMA1: D1 = S^T . [W; Q~]^T            -> (W S)^T | (Q~ S)^T
//        U^T  = U~^T - (W S)^T
//        MMA2: D2 = U^T . K^                    -> state increment (K^^T U)^T
//        MMA3: D1[:, 64:] += U^T . P^T          -> (Q~ S + P U)^T
//        S^T  = S^T Diag(gamma) + D2;  o = scale * D1[:, 64:]^T
//    The state never leaves the SM between chunks; S_final is written once.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "kda_internal.cuh"
#include "tc_primitives.cuh"

namespace kda {
namespace {

constexpr int C = kChunk;   // 64 tokens per chunk
constexpr int D = 128;      // dk = dv
constexpr int kSlice = 64;  // value columns per carry CTA
constexpr int kSlices = D / kSlice;

// Workspace record per (chunk, head), bytes. Every piece is a verbatim image of
// a shared-memory operand of the carry kernel, which bulk-copies it. The carry
// needs one group of MMAs per chunk (see the carry below):
//     D = [S^T | U~^T] . [[-N, Q']^T ; [K^, P^T]]   (N = K^^T W, Q' = Q~ - P W)
// so the record holds the B operand of that group in two K ranges (keys, then
// tokens), each as 192 K-major rows: 128 state rows (one per key channel) and
// 64 output rows (one per token).
struct Record {
    static constexpr uint32_t kBk = 0;        // [2 key blocks][192 rows][128 B] bf16 K-major SW128:
                                              //   rows 0..127: -N[i][i'], rows 128..191: Q'[t][i]
    static constexpr uint32_t kBt = 49152;    // [192 rows][128 B] bf16 K-major SW128:
                                              //   rows 0..127: K^[t][i] (row i), rows 128..191: P[t][s]
    static constexpr uint32_t kU = 73728;     // U~^T bf16 [2 halves][64 value cols][128 B] K-major SW128
    static constexpr uint32_t kG = 90112;     // gamma fp32 [128]
    static constexpr uint32_t kBytes = 90624;
    static constexpr uint32_t kBlk = 24576;   // one 192-row block
    static constexpr uint32_t kOut = 16384;   // rows 128..191 start 16 KB into a block
};
static_assert(Record::kG + 512 == Record::kBytes, "record size");

// Shared-memory layout of the carry kernel (offsets from a 1024-aligned base).
struct CarrySmem {
    static constexpr uint32_t kBk = 0;         // 49152: B over the keys (K-major, 2 K-blocks)
    static constexpr uint32_t kBt = 49152;     // 24576: B over the tokens (K-major)
    static constexpr uint32_t kU = 73728;      // 8192:  U~^T of this half, A over the tokens
    static constexpr uint32_t kG = 81920;      // 512:   gamma
    static constexpr uint32_t kStage = 82944;  // stage stride (1024-aligned)
    static constexpr uint32_t kSt = 2 * kStage;        // 2 x S^T bf16 64x128, A over the keys (K-major, 2 K-blocks)
    static constexpr uint32_t kOs = kSt + 2 * 16384;   // output staging, 1 KB per state warp
    static constexpr uint32_t kBar = kOs + 8192;       // mbarriers
    static constexpr uint32_t kBytes = kBar + 256 + 1024;  // + alignment slack
};
static_assert(CarrySmem::kSt % 1024 == 0 && CarrySmem::kStage % 1024 == 0, "operand alignment");
static_assert(CarrySmem::kBytes <= 227 * 1024, "carry shared memory");

struct TcParams {
    const __nv_bfloat16 *q, *k, *v;
    const float *log_alpha, *beta, *S0;
    int N, H;
    float scale;
    __nv_bfloat16 *o;
    float *S_final;
    const int32_t *seq_start, *chunk_off, *order;
    uint8_t *rec;      // records
    int *err;          // device status word (the code of the first wait that ran out)
    int *fix_count;    // number of chunks listed for the exact fixup
    uint32_t spin;     // poll limit of every bounded wait
    int starve;        // debugging: the carry's producer issues no copies
    // time split of the sequential phase (see the carry kernel): segments per
    // sequence, the launch's pass, and the segment states
    // [3 kinds][nseg][N][H][D][D] fp32 (kind 0: state from a zero start,
    // 1: transition, 2: state at the segment's end)
    int nseg;
    int pass;          // 0: no split, 1: first pass, 2: second pass
    float *seg;
    int T_uniform;     // sequences of T_uniform tokens each (no cu_seqlens), else 0
    int *fix_list;     // chunk * H + head, one per listed chunk
    // q, k, v and log_alpha as 3-D tensors {channel, head, token} for TMA tile
    // loads of 128 bytes of channels x 1 head x 64 tokens in the 128-byte
    // swizzle (64 bf16 or 32 fp32 channels); tm_la only for per-channel gates
    CUtensorMap tm_q, tm_k, tm_v, tm_la;
};

__device__ __forceinline__ int find_seq(const int32_t *chunk_off, int N, int c)
{
    if (c >= chunk_off[N]) return -1;
    int lo = 0, hi = N - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (chunk_off[mid] <= c) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Sequence, first packed token and length of global chunk c: arithmetic for
// uniform batches, a search of the plan for packed sequences. False past the
// last chunk.
struct ChunkLoc {
    int n, t0, L;
};

__device__ __forceinline__ bool locate_chunk(const TcParams &p, int c, ChunkLoc &loc)
{
    if (p.T_uniform > 0) {
        const int per = (p.T_uniform + C - 1) / C;
        const int n = c / per;
        if (n >= p.N) return false;
        const int lc = c - n * per;
        loc.n = n;
        loc.t0 = n * p.T_uniform + lc * C;
        loc.L = min(C, p.T_uniform - lc * C);
        return true;
    }
    const int n = find_seq(p.chunk_off, p.N, c);
    if (n < 0) return false;
    loc.n = n;
    loc.t0 = p.seq_start[n] + (c - p.chunk_off[n]) * C;
    loc.L = min(C, p.seq_start[n + 1] - loc.t0);
    return true;
}

// ------------------------------------------------------------------- exact fixup
// fp32 CUDA-core recomputation of one chunk's record with an exact exponential
// for every gate difference in A and P and forward substitution for W and U~.
// Used only for the chunks the tensor-core prep lists as outside the range of
// its factorised exponentials (a decay of more than 80 nats inside half a
// chunk); for ordinary gates the list is empty and the kernel exits at once.
constexpr int kPrepThreads = 256;
constexpr int DP = D + 1;  // padded fp32 row of the fixup's [C][D] arrays

// bf16 element (row, k) of a K-major SW128 block whose rows are 128 bytes
__device__ __forceinline__ __nv_bfloat16 *kmaj(uint8_t *block, int row, int k)
{
    return reinterpret_cast<__nv_bfloat16 *>(block + tc::sw128((uint32_t)row, 2u * (uint32_t)k));
}

__device__ void prep_exact_chunk(const TcParams &p, int c, int h, float *smem)
{
    float *sk = smem;               // [C][DP]  k, then beta e^g k, then W
    float *sq = sk + C * DP;        // [C][DP]  q, then Q~
    float *sg = sq + C * DP;        // [C][DP]  cumulative log-decay g
    float *skh = sg + C * DP;       // [C][DP]  K^
    float *sv = skh + C * DP;       // [C][D]   v, then beta v, then U~
    float *sA = sv + C * D;         // [C][C+1]
    float *sP = sA + C * (C + 1);   // [C][C+1]
    float *sb = sP + C * (C + 1);   // [C]

    const int H = p.H;
    ChunkLoc loc;
    if (!locate_chunk(p, c, loc)) return;
    const int t0 = loc.t0, L = loc.L;
    const int tid = threadIdx.x;

    for (int idx = tid; idx < C * D; idx += kPrepThreads) {
        const int r = idx / D, i = idx % D;
        float kk = 0.f, qq = 0.f, vv = 0.f, la = 0.f;
        if (r < L) {
            const size_t off = ((size_t)(t0 + r) * H + h) * D + i;
            kk = __bfloat162float(p.k[off]); qq = __bfloat162float(p.q[off]);
            vv = __bfloat162float(p.v[off]); la = p.log_alpha[off];
        }
        sk[r * DP + i] = kk; sq[r * DP + i] = qq; sv[r * D + i] = vv; sg[r * DP + i] = la;
    }
    for (int r = tid; r < C; r += kPrepThreads)
        sb[r] = r < L ? p.beta[(size_t)(t0 + r) * H + h] : 0.f;
    __syncthreads();
    for (int i = tid; i < D; i += kPrepThreads) {
        float g = 0.f;
        for (int r = 0; r < C; ++r) { g += sg[r * DP + i]; sg[r * DP + i] = g; }
    }
    __syncthreads();

    uint8_t *rec = p.rec + ((size_t)c * H + h) * Record::kBytes;
    const int warp = tid >> 5, lane = tid & 31;
    for (int r = warp; r < C; r += kPrepThreads / 32) {
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
            sP[r * (C + 1) + s] = (s <= r) ? pqk : 0.f;
        }
    }
    __syncthreads();
    // Q~ in place, K^, gamma; then the solve's right-hand sides
    for (int idx = tid; idx < C * D; idx += kPrepThreads) {
        const int r = idx / D, i = idx % D;
        const float g = sg[r * DP + i], gC = sg[(C - 1) * DP + i];
        sq[r * DP + i] *= expf(g);
        skh[r * DP + i] = expf(gC - g) * sk[r * DP + i];
        sk[r * DP + i] *= sb[r] * expf(g);
        sv[r * D + i] *= sb[r];
    }
    for (int i = tid; i < D; i += kPrepThreads)
        reinterpret_cast<float *>(rec + Record::kG)[i] = expf(sg[(C - 1) * DP + i]);
    __syncthreads();
    for (int col = tid; col < 2 * D; col += kPrepThreads) {  // W and U~ by forward substitution
        float *x = col < D ? sk + col : sv + (col - D);
        const int stride = col < D ? DP : D;
        for (int r = 1; r < C; ++r) {
            float acc = x[r * stride];
            for (int s = 0; s < r; ++s) acc -= sA[r * (C + 1) + s] * x[s * stride];
            x[r * stride] = acc;
        }
    }
    __syncthreads();
    // -N = -K^^T W (rows i of the key block i'/64), Q' = Q~ - P W (rows 128 + t)
    for (int idx = tid; idx < D * D; idx += kPrepThreads) {
        const int i = idx / D, i2 = idx % D;
        float acc = 0.f;
        for (int t = 0; t < C; ++t) acc += skh[t * DP + i] * sk[t * DP + i2];
        *kmaj(rec + Record::kBk + (i2 >> 6) * Record::kBlk, i, i2 & 63) = __float2bfloat16_rn(-acc);
    }
    for (int idx = tid; idx < C * D; idx += kPrepThreads) {
        const int t = idx / D, i2 = idx % D;
        float acc = sq[t * DP + i2];
        for (int s2 = 0; s2 <= t; ++s2) acc -= sP[t * (C + 1) + s2] * sk[s2 * DP + i2];
        *kmaj(rec + Record::kBk + (i2 >> 6) * Record::kBlk, 128 + t, i2 & 63) = __float2bfloat16_rn(acc);
    }
    // K^ as rows i over the tokens, P as rows 128 + t, U~^T as rows j of its half
    for (int idx = tid; idx < D * C; idx += kPrepThreads) {
        const int i = idx / C, t = idx % C;
        *kmaj(rec + Record::kBt, i, t) = __float2bfloat16_rn(skh[t * DP + i]);
        *kmaj(rec + Record::kU + (i >> 6) * 8192, i & 63, t) = __float2bfloat16_rn(sv[t * D + i]);
    }
    for (int idx = tid; idx < C * C; idx += kPrepThreads) {
        const int t = idx / C, s2 = idx % C;
        *kmaj(rec + Record::kBt, 128 + t, s2) = __float2bfloat16_rn(sP[t * (C + 1) + s2]);
    }
    __syncthreads();  // the caller reuses shared memory for its next chunk
}

__global__ void __launch_bounds__(kPrepThreads, 1) tc_prep_fixup_kernel(TcParams p)
{
    extern __shared__ float smem[];
    const int count = *p.fix_count;
    for (int idx = blockIdx.x; idx < count; idx += gridDim.x) {
        const int e = p.fix_list[idx];
        prep_exact_chunk(p, e / p.H, e % p.H, smem);
    }
}

// ------------------------------------------------------------------- prep
// Tensor-core prep. Per chunk and head (256 threads):
//  1. Each thread owns 8 key channels x 4 tokens: loads q, k, v, log_alpha (TMA
//     tiles), forms the in-chunk cumulative log-decay g (token-group totals
//     exchanged in shared memory), E_r = e^{g_r} and H_r = e^{g_C - g_r}, writes
//     K^ = H k to the record (as rows over the tokens, swapped between lane
//     pairs so that every store is 16 bytes) and Q~ = E q to the record's Q'
//     slot, and the MMA operands below to shared memory.
//  2. The intra-chunk matrices A and P need e^{g_r - g_s} inside a contraction
//     over channels, so it is split into a row factor and a column factor
//     around a reference token: rows/cols of the first half use g_15, rows of
//     the second half and every column against them use g_31. One MMA,
//         D (128x96) = [K'_0; Q'_0; K'_1; Q'_1] (128x128) . [K''_0 | K''_1]^T,
//     yields both diagonal 32x32 blocks and the off-diagonal 32x32 block of
//     A (from k rows) and P (from q rows). Every factor is <= 1 except within a
//     half, where it is bounded by the decay across at most 32 tokens; a chunk
//     that would exceed e^80 there is listed for the exact fixup kernel.
//  3. T = (I + A)^{-1} in fp32 by blocks of 16: a 2x2 block inverse of 32-row
//     blocks over 16-row ones (invert_unit_lower64).
//  4. W = [T Diag(beta); P] (128x64) . K~ (64x128), whose accumulator rows
//     0..63 are the 64 tokens, and U~^T = V^T (128x64) . (T Diag(beta))^T
//     (64x64), whose rows are the 128 value columns: two MMA groups on the same
//     operand images (the v tile is used as it landed).
//  5. N = K^^T W and P W (finish_record): the reference-31 rows of step 2's B
//     operand, k_s e^{g_31 - g_s} for every token s, are K^ up to the channel
//     factor e^{g_C - g_31}, so they serve as the A operand of N and the factor
//     scales N's rows; Q' = Q~ - P W with Q~ read back from the record.
//  6. Everything goes to the record in the carry kernel's operand layouts.
constexpr int kPrep2Threads = 256;

constexpr uint32_t kLdBytes = 68 * 4;  // one row of the fp32 A / T matrices (kLd floats)

struct Prep2Smem {
    static constexpr uint32_t kAop = 0;        // 32768: [kb][128 rows][128B]
    static constexpr uint32_t kA = 0;          // fp32 A [64][kLd], after MMA-AP
    static constexpr uint32_t kBop = 32768;    // 24576: [kb][96 rows][128B]
    static constexpr uint32_t kBK = 57344;     // 16384: K~ = e^g k MN-major image
    static constexpr uint32_t kBV = 73728;     // 16384: the v tile as landed (MN-major), A of U~^T
    // log_alpha lands over [kBop, kBop + 32768) (the B operand and K~'s buffer
    // are written only after every thread holds its inputs in registers)
    static constexpr uint32_t kTt = 90112;     // 8192:  [T; P], K-major rows r (P from 8 KB on)
    // During step 1 the [T; P] buffer is free: it holds the token-group totals
    // and the per-channel constants.
    static constexpr uint32_t kTot = kTt;          // 8192:  token-group totals [16][128]
    static constexpr uint32_t kCst = kTt + 8192;   // 3584:  per-channel constants [7][128]
    static constexpr uint32_t kB = 106496;     // 256:   beta [64]
    static constexpr uint32_t kBar = 106752;   // barriers + tmem slot + flags
    static constexpr uint32_t kF = 106816;     // 512:   e^{g_C - g_31} per channel
    static constexpr uint32_t kBytes = kF + 512 + 1024;
    // Later tenants of the same memory (each region is dead by then):
    static constexpr uint32_t kT = 17408;      // fp32 T [64][kLd], after MMA-AP (over the
                                               // first key block's reference-15 rows)
    static constexpr uint32_t kKh = 36864;     // the reference-31 rows of the B operand: k e^{g_31 - g}
                                               // for tokens 0..63, per key block (12 KB apart);
                                               // A of MMA-NP until it completes
    static constexpr uint32_t kP = kTt + 8192; // 8192:  P (K-major rows t), from the A/P read-out on
    static constexpr uint32_t kW = 0;          // 16384: W bf16 MN-major image, after MMA-WU
    static constexpr uint32_t kQp = 0;         // 16384: Q' staging (2 key blocks of 8 KB), after MMA-NP
    static constexpr uint32_t kN0 = 57344;     // 16384: -N staging, key block 0, after MMA-WU
    static constexpr uint32_t kUs = 73728;     // 16384: U~^T bf16 staging, after MMA-WU
    static constexpr uint32_t kN1 = 90112;     // 16384: -N staging, key block 1, after MMA-NP
};
static_assert(Prep2Smem::kT == 64 * kLdBytes && Prep2Smem::kT + 64 * kLdBytes <= Prep2Smem::kKh &&
              Prep2Smem::kKh == Prep2Smem::kBop + 32 * 128 && Prep2Smem::kKh % 1024 == 0,
              "T lies between A and the reference-31 rows it must not touch");

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Row stride (floats) of the fp32 A and T matrices: rows stay 16-byte aligned,
// and float4 stores of 8 consecutive rows hit distinct bank groups.
constexpr int kLd = 68;

// One 1x4 strip of a 16x16 block product:
//     acc[q] += sum_k X[xr + rr][xc + k] * Y[yr + k][yc + 4*c4 + q],  k < 16, q < 4,
// X with row stride kLd, Y with row stride ys. 4 + 16 vector loads feed 64 FMAs
// in four independent chains.
__device__ __forceinline__ void strip_dot(const float *X, int xr, int xc, const float *Y, int yr,
                                          int yc, int ys, int rr, int c4, float4 &acc)
{
    float a[16];
#pragma unroll
    for (int k = 0; k < 16; k += 4) {
        const float4 v = *reinterpret_cast<const float4 *>(X + (xr + rr) * kLd + xc + k);
        a[k] = v.x; a[k + 1] = v.y; a[k + 2] = v.z; a[k + 3] = v.w;
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const float4 y = *reinterpret_cast<const float4 *>(Y + (yr + k) * ys + yc + 4 * c4);
        acc.x += a[k] * y.x; acc.y += a[k] * y.y; acc.z += a[k] * y.z; acc.w += a[k] * y.w;
    }
}

__device__ __forceinline__ float4 neg4(float4 v) { return make_float4(-v.x, -v.y, -v.z, -v.w); }

// T = (I + A)^{-1} for the 64x64 strictly lower A (fp32, row stride kLd) on
// 256 threads, as a 2x2 block inverse of 32-row blocks whose own inverses are
// 2x2 block inverses of 16-row blocks: with T_ii the inverses of the four
// 16x16 diagonal blocks (by substitution),
//     T_10 = -T_11 A_10 T_00,  T_32 = -T_33 A_32 T_22,
//     Y = A_[23][01] T_[01][01],  T_[23][01] = -T_[23][23] Y.
// The 16x16 products are grouped into four phases of up to four independent
// block tasks (64 threads each, one 1x4 strip per thread); the blocks above
// T's diagonal, never read by the callers, hold the intermediates:
//   (0,1) A_10 T_00   (0,2) A_32 T_22   (0,3) Y_21   (1,2) Y_31
//   (1,3) Y_20        (2,3) Y_30        and T_33 Y_31 sits in (3,1) until T_31.
// Ts (row stride kLd) receives the blocks on and below the diagonal. Ends with
// a CTA barrier.
__device__ __forceinline__ void invert_unit_lower64(const float *As, float *Ts, int tid)
{
    if (tid < 64) {  // diagonal blocks: one column of one block per thread, right-looking
        const int b = tid >> 4, cc = tid & 15, o = 16 * b;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = (r == cc) ? 1.f : 0.f;
#pragma unroll
        for (int s2 = 0; s2 < 15; ++s2) {
            float col[15];
#pragma unroll
            for (int r = s2 + 1; r < 16; ++r) col[r - 1] = As[(o + r) * kLd + o + s2];
            const float xs = x[s2];
#pragma unroll
            for (int r = s2 + 1; r < 16; ++r) x[r] -= col[r - 1] * xs;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Ts[(o + r) * kLd + o + cc] = x[r];
    }
    __syncthreads();
    const int rr = (tid & 63) >> 2, c4 = tid & 3, task = tid >> 6;
    auto strip = [&](float *M, int bi, int bj) {  // this thread's 1x4 strip of block (bi, bj)
        return reinterpret_cast<float4 *>(M + (16 * bi + rr) * kLd + 16 * bj + 4 * c4);
    };
    const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
    {   // phase 1: A_10 T_00, A_32 T_22, Y_21 = A_21 T_11, Y_31 = A_31 T_11
        float4 acc = zero;
        const int ar = task == 0 ? 16 : (task == 1 ? 48 : (task == 2 ? 32 : 48));
        const int ac = task == 0 ? 0 : (task == 1 ? 32 : 16);
        strip_dot(As, ar, ac, Ts, ac, ac, kLd, rr, c4, acc);
        const int sj = task == 3 ? 2 : task + 1, si = task == 3 ? 1 : 0;
        *strip(Ts, si, sj) = acc;
    }
    __syncthreads();
    {   // phase 2: T_10 = -T_11 (A_10 T_00), T_32 = -T_33 (A_32 T_22), Y_20, Y_30 = A_[23]0 T_00
        float4 acc = zero;
        if (task < 2) {
            const int d = task == 0 ? 16 : 48;               // T_11 or T_33
            strip_dot(Ts, d, d, Ts, 0, task == 0 ? 16 : 32, kLd, rr, c4, acc);
            *strip(Ts, task == 0 ? 1 : 3, task == 0 ? 0 : 2) = neg4(acc);
        } else {
            strip_dot(As, task == 2 ? 32 : 48, 0, Ts, 0, 0, kLd, rr, c4, acc);
            *strip(Ts, task - 1, 3) = acc;                   // (1,3) Y_20, (2,3) Y_30
        }
    }
    __syncthreads();
    {   // phase 3: Y_20 += A_21 T_10, Y_30 += A_31 T_10, T_21 = -T_22 Y_21, (3,1) = T_33 Y_31
        if (task < 2) {
            float4 acc = *strip(Ts, task + 1, 3);
            strip_dot(As, task == 0 ? 32 : 48, 16, Ts, 16, 0, kLd, rr, c4, acc);
            *strip(Ts, task + 1, 3) = acc;
        } else if (task == 2) {
            float4 acc = zero;
            strip_dot(Ts, 32, 32, Ts, 0, 48, kLd, rr, c4, acc);
            *strip(Ts, 2, 1) = neg4(acc);
        } else {
            float4 acc = zero;
            strip_dot(Ts, 48, 48, Ts, 16, 32, kLd, rr, c4, acc);
            *strip(Ts, 3, 1) = acc;
        }
    }
    __syncthreads();
    {   // phase 4: T_20 = -T_22 Y_20, T_30 = -(T_32 Y_20 + T_33 Y_30), T_31 = -(T_33 Y_31 + T_32 Y_21)
        if (task == 0) {
            float4 acc = zero;
            strip_dot(Ts, 32, 32, Ts, 16, 48, kLd, rr, c4, acc);
            *strip(Ts, 2, 0) = neg4(acc);
        } else if (task == 1) {
            float4 acc = zero;
            strip_dot(Ts, 48, 32, Ts, 16, 48, kLd, rr, c4, acc);
            strip_dot(Ts, 48, 48, Ts, 32, 48, kLd, rr, c4, acc);
            *strip(Ts, 3, 0) = neg4(acc);
        } else if (task == 2) {
            float4 acc = *strip(Ts, 3, 1);
            strip_dot(Ts, 48, 32, Ts, 0, 48, kLd, rr, c4, acc);
            *strip(Ts, 3, 1) = neg4(acc);
        }
    }
    __syncthreads();
}

// The same inverse by block distance, T_ij = -T_ii sum_{k=j}^{i-1} A_ik T_kj:
// six phases after the diagonal blocks, with 192, 128 and 64 threads busy at
// distances 1, 2 and 3 (Ys is 3 x 16 x 16 fp32 scratch). Slower on its own
// than the grouping above, but the scalar-gate prep, whose two co-resident
// CTAs fill the idle threads' issue slots, measured faster with it. Ends with
// a CTA barrier.
__device__ __forceinline__ void invert_unit_lower64_by_distance(const float *As, float *Ts,
                                                                float *Ys, int tid)
{
    if (tid < 64) {  // diagonal blocks: one column of one block per thread, right-looking
        const int b = tid >> 4, cc = tid & 15, o = 16 * b;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = (r == cc) ? 1.f : 0.f;
#pragma unroll
        for (int s2 = 0; s2 < 15; ++s2) {
            float col[15];
#pragma unroll
            for (int r = s2 + 1; r < 16; ++r) col[r - 1] = As[(o + r) * kLd + o + s2];
            const float xs = x[s2];
#pragma unroll
            for (int r = s2 + 1; r < 16; ++r) x[r] -= col[r - 1] * xs;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Ts[(o + r) * kLd + o + cc] = x[r];
    }
    __syncthreads();
    // Off-diagonal blocks by distance, T_ij = -T_ii sum_{k=j}^{i-1} A_ik T_kj, in
    // 1x4 strips: thread -> (block, row rr, column group c4).
    const int rr = (tid & 63) >> 2, c4 = tid & 3, blk = tid >> 6;
    // distance 1: i = 1..3 on threads 0..191
    if (blk < 3) {
        const int i = 1 + blk;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        strip_dot(As, 16 * i, 16 * (i - 1), Ts, 16 * (i - 1), 16 * (i - 1), kLd, rr, c4, acc);
        *reinterpret_cast<float4 *>(Ys + blk * 256 + rr * 16 + 4 * c4) = acc;
    }
    __syncthreads();
    if (blk < 3) {
        const int i = 1 + blk;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        strip_dot(Ts, 16 * i, 16 * i, Ys + blk * 256, 0, 0, 16, rr, c4, acc);
        *reinterpret_cast<float4 *>(Ts + (16 * i + rr) * kLd + 16 * (i - 1) + 4 * c4) = neg4(acc);
    }
    __syncthreads();
    // distance 2: i = 2, 3 on threads 0..127
    if (blk < 2) {
        const int i = 2 + blk;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        strip_dot(As, 16 * i, 16 * (i - 2), Ts, 16 * (i - 2), 16 * (i - 2), kLd, rr, c4, acc);
        strip_dot(As, 16 * i, 16 * (i - 1), Ts, 16 * (i - 1), 16 * (i - 2), kLd, rr, c4, acc);
        *reinterpret_cast<float4 *>(Ys + blk * 256 + rr * 16 + 4 * c4) = acc;
    }
    __syncthreads();
    if (blk < 2) {
        const int i = 2 + blk;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        strip_dot(Ts, 16 * i, 16 * i, Ys + blk * 256, 0, 0, 16, rr, c4, acc);
        *reinterpret_cast<float4 *>(Ts + (16 * i + rr) * kLd + 16 * (i - 2) + 4 * c4) = neg4(acc);
    }
    __syncthreads();
    // distance 3: T_30 = -T_33 (A_30 T_00 + A_31 T_10 + A_32 T_20) on threads 0..63
    if (blk == 0) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        strip_dot(As, 48, 0, Ts, 0, 0, kLd, rr, c4, acc);
        strip_dot(As, 48, 16, Ts, 16, 0, kLd, rr, c4, acc);
        strip_dot(As, 48, 32, Ts, 32, 0, kLd, rr, c4, acc);
        *reinterpret_cast<float4 *>(Ys + rr * 16 + 4 * c4) = acc;
    }
    __syncthreads();
    if (blk == 0) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        strip_dot(Ts, 48, 48, Ys, 0, 0, 16, rr, c4, acc);
        *reinterpret_cast<float4 *>(Ts + (48 + rr) * kLd + 4 * c4) = neg4(acc);
    }
    __syncthreads();
}

// Where finish_record keeps its operands and staging (offsets from the
// 1024-aligned shared-memory base; each region must be dead when it is used).
struct FinishSmem {
    uint32_t w;     // 16384: W bf16 MN-major image (B of MMA-NP)
    uint32_t us;    // 16384: U~^T bf16 staging
    uint32_t kh;    // K^ (or a per-channel multiple of it) over the tokens, already in
                    // place: the A operand of MMA-NP
    uint32_t kh_lbo;  // 0: K-major rows i (16 KB); else MN-major token rows, key
                      // blocks kh_lbo bytes apart
    uint32_t kh_scale;  // 0, or fp32 [128]: K^ row i = kh_scale[i] x the operand's row i
    uint32_t pp;    // 8192:  P rows t (A of MMA-NP), already in place
    uint32_t n0;    // 16384: -N staging, key block 0 (after MMA-NP)
    uint32_t n1;    // 16384: -N staging, key block 1 (after MMA-NP)
    uint32_t qp;    // 16384: Q' staging (2 key blocks of 8 KB, after MMA-NP)
};

// The end of both prep kernels, once the W and U~^T MMAs (TMEM columns 0..127
// lanes 0..63, and columns 128..191 lanes 0..127) are committed to bar_wu and the
// K^ operand and P are in shared memory:
//   1. W -> bf16 MN-major image; U~^T -> bf16 rows j of its half, sent to the record;
//   2. MMA-NP: N = K^^T W (M = 128, columns 0..127) and P W (M = 64, columns 128..255);
//   3. -N and Q' = Q~ - P W as record images, sent with bulk stores; then every
//      copy and MMA is drained.
// Q~ of token t comes from qload(t, key block, half warp, raw[4]) (the 4
// 16-byte chunks 4 hl .. 4 hl + 3 of the block, issued before the MMA-NP wait)
// and qconv(t, raw chunk, q8) (8 floats).
// Ends with the CTA's asynchronous work finished (TMEM may be released).
template <typename QLoad, typename QConv>
__device__ __forceinline__ void finish_record(uint8_t *sm, const FinishSmem &f, uint32_t tmem,
                                              uint8_t *rec, uint64_t *bar_wu, uint64_t *bar_np,
                                              uint64_t *bar_ld, uint64_t *bar_fin,
                                              volatile int *abort, const TcParams &p, int code,
                                              QLoad qload, QConv qconv)
{
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int lg = warp & 3, wh = warp >> 2;
    const uint32_t la = tmem + ((uint32_t)(lg * 32) << 16);
    {
        tc::mbar_wait(bar_wu, 0, abort, p.err, code, p.spin);
        tc::tc_fence_after_sync();
        const int row = lg * 32 + lane;
        float w[32];
        if (lg < 2) {  // W: lanes 0..63 are the tokens
            uint8_t *wb = sm + f.w + (uint32_t)wh * 8192;
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
                tc::tmem_ld32_sync(la + 64 * wh + 32 * q2, w);
#pragma unroll
                for (int c16 = 0; c16 < 4; ++c16) {
                    uint32_t u[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) u[e] = pack_bf16x2(w[c16 * 8 + 2 * e], w[c16 * 8 + 2 * e + 1]);
                    *reinterpret_cast<uint4 *>(wb + tc::sw128(row, (q2 * 4 + c16) * 16)) =
                        make_uint4(u[0], u[1], u[2], u[3]);
                }
            }
        }
        // U~^T: lane = value column j, columns 128 + 32 wh.. = tokens
        tc::tmem_ld32_sync(la + 128 + 32 * wh, w);
        uint8_t *ub = sm + f.us + (uint32_t)(row >> 6) * 8192;
#pragma unroll
        for (int c16 = 0; c16 < 4; ++c16) {
            uint32_t u[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) u[e] = pack_bf16x2(w[c16 * 8 + 2 * e], w[c16 * 8 + 2 * e + 1]);
            *reinterpret_cast<uint4 *>(ub + tc::sw128(row & 63, (4 * wh + c16) * 16)) =
                make_uint4(u[0], u[1], u[2], u[3]);
        }
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before_sync();
    __syncthreads();
    tc::tc_fence_after_sync();
    if (tid == 0) {
        tc::bulk_s2g(rec + Record::kU, sm + f.us, 16384);
        tc::bulk_commit();
        const uint32_t wd = tc::smem_u32(sm + f.w);
        const uint32_t kd = tc::smem_u32(sm + f.kh);
        const uint32_t pd = tc::smem_u32(sm + f.pp);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            tc::mma_bf16(tmem,
                         f.kh_lbo ? tc::smem_desc(kd + kk * 2048, f.kh_lbo, 1024)
                                  : tc::smem_desc(kd + kk * 32, 16, 1024),
                         tc::smem_desc(wd + kk * 2048, 8192, 1024),
                         tc::idesc_bf16(128, 128, f.kh_lbo ? 1 : 0, 1), kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            tc::mma_bf16(tmem + 128, tc::smem_desc(pd + kk * 32, 16, 1024),
                         tc::smem_desc(wd + kk * 2048, 8192, 1024), tc::idesc_bf16(64, 128, 0, 1),
                         kk > 0);
        tc::mma_commit(bar_np);
        // the staging below reuses memory that earlier bulk stores read from
        tc::bulk_wait_read_all();
    }
    // Q~ of this thread's token, fetched while MMA-NP runs
    const int t = 16 * lg + (lane & 15), hl = lane >> 4;
    uint4 qraw[4];
    qload(t, wh, hl, qraw);
    {
        tc::mbar_wait(bar_np, 0, abort, p.err, code + 1, p.spin);
        tc::tc_fence_after_sync();
        __syncthreads();
        const int i = lg * 32 + lane;  // N: lane = key channel i, columns i' = 64 wh..
        const float ns = f.kh_scale ? -reinterpret_cast<const float *>(sm + f.kh_scale)[i] : -1.f;
        uint8_t *nb = sm + (wh ? f.n1 : f.n0);
        float w[32];
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
            tc::tmem_ld32_sync(la + 64 * wh + 32 * q2, w);
#pragma unroll
            for (int c16 = 0; c16 < 4; ++c16) {
                uint32_t u[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    u[e] = pack_bf16x2(ns * w[c16 * 8 + 2 * e], ns * w[c16 * 8 + 2 * e + 1]);
                *reinterpret_cast<uint4 *>(nb + tc::sw128(i, (q2 * 4 + c16) * 16)) =
                    make_uint4(u[0], u[1], u[2], u[3]);
            }
        }
        // P W (M = 64): row t in lanes 0..15 of lane group lg, columns split by
        // half warps: this thread has channels 64 wh + 32 hl .. + 31
        tc::tmem_ld16x2_x32_sync(la + 128 + 64 * wh, w);
        uint8_t *qb = sm + f.qp + (uint32_t)wh * 8192;
#pragma unroll
        for (int c16 = 0; c16 < 4; ++c16) {
            const int cb = 4 * hl + c16;  // 16-byte chunk inside the key block
            float q8[8];
            qconv(t, qraw[c16], q8);
            uint32_t u[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                u[e] = pack_bf16x2(q8[2 * e] - w[c16 * 8 + 2 * e], q8[2 * e + 1] - w[c16 * 8 + 2 * e + 1]);
            *reinterpret_cast<uint4 *>(qb + (uint32_t)t * 128 + ((((uint32_t)cb) ^ ((uint32_t)t & 7u)) << 4)) =
                make_uint4(u[0], u[1], u[2], u[3]);
        }
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before_sync();
    __syncthreads();
    if (tid == 0) {
        tc::fence_proxy_async_global();  // Q~ written to the Q' slot by threads, overwritten now
        tc::bulk_s2g(rec + Record::kBk, sm + f.n0, 16384);
        tc::bulk_s2g(rec + Record::kBk + Record::kBlk, sm + f.n1, 16384);
        tc::bulk_s2g(rec + Record::kBk + Record::kOut, sm + f.qp, 8192);
        tc::bulk_s2g(rec + Record::kBk + Record::kBlk + Record::kOut, sm + f.qp + 8192, 8192);
        tc::bulk_commit();
        tc::bulk_wait_read_all();  // the CTA's shared memory must outlive the reads
        // drain (matters only after a wait gave up): the input tiles have
        // landed and every MMA has finished before the memory is released
        tc::mbar_drain(bar_ld, 0, p.err, code + 2, p.spin);
        tc::mma_commit(bar_fin);
        tc::mbar_drain(bar_fin, 0, p.err, code + 2, p.spin);
    }
}

__global__ void __launch_bounds__(kPrep2Threads, 2) tc_prep2_kernel(const __grid_constant__ TcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar_ap = reinterpret_cast<uint64_t *>(sm + Prep2Smem::kBar);
    uint64_t *bar_wu = bar_ap + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_ap + 2);
    volatile int *abort = reinterpret_cast<volatile int *>(bar_ap + 3);
    uint64_t *bar_ld = bar_ap + 4;
    float *tot = reinterpret_cast<float *>(sm + Prep2Smem::kTot);    // [16][128] group totals
    float *cst = reinterpret_cast<float *>(sm + Prep2Smem::kCst);    // [8][128] per channel
    float *sbeta = reinterpret_cast<float *>(sm + Prep2Smem::kB);

    const int c = blockIdx.x, h = blockIdx.y, H = p.H;
    ChunkLoc loc;
    if (!locate_chunk(p, c, loc)) return;  // uniform over the CTA: nothing allocated yet
    const int t0 = loc.t0, L = loc.L;
    const int tid = threadIdx.x, warp = tid >> 5;
    // 16-byte granules: channel octet `oc` (8 channels = one 16-byte swizzle
    // chunk of a bf16 row) x token group `tg` (4 consecutive tokens)
    const int oc = tid & 15, tg = tid >> 4;
    const int c0 = 8 * oc;
    const uint32_t kb = (uint32_t)(oc >> 3);   // K-block / MN atom
    const uint32_t ck = (uint32_t)(oc & 7);    // chunk inside the 128-byte row

    // The chunk's q, k, v and log_alpha arrive as ten TMA tiles (64 tokens x
    // 128 bytes, 128-byte swizzle): q, k, v as [channel block of 64][64 tokens]
    // [128 B], log_alpha as [block of 32]. q, k and log_alpha land in operand
    // buffers that step 1 fills only after every thread holds its inputs in
    // registers; v lands where it stays, as the A operand of U~^T (the solve's
    // beta is folded into T instead).
    uint8_t *in_q = sm + Prep2Smem::kAop, *in_k = sm + Prep2Smem::kAop + 16384;
    uint8_t *in_v = sm + Prep2Smem::kBV, *in_la = sm + Prep2Smem::kBop;
    if (tid == 0) {
        tc::mbar_init(bar_ap, 1);
        tc::mbar_init(bar_wu, 1);
        tc::mbar_init(bar_ld, 1);
        tc::mbar_init(bar_ld + 1, 1);  // bar_fin
        tc::mbar_init(bar_ld + 2, 1);  // bar_np
        *abort = 0;
        tc::fence_mbar_init();
        tc::mbar_arrive_expect_tx(bar_ld, 10 * 8192);
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            tc::tma_load_3d(in_q + b * 8192, &p.tm_q, 64 * b, h, t0, bar_ld);
            tc::tma_load_3d(in_k + b * 8192, &p.tm_k, 64 * b, h, t0, bar_ld);
            tc::tma_load_3d(in_v + b * 8192, &p.tm_v, 64 * b, h, t0, bar_ld);
        }
#pragma unroll
        for (int b = 0; b < 4; ++b)
            tc::tma_load_3d(in_la + b * 8192, &p.tm_la, 32 * b, h, t0, bar_ld);
    }
    if (warp == 0) { tc::tmem_alloc(tmem_slot, 256); tc::tmem_relinquish(); }
    if (tid < C) sbeta[tid] = tid < L ? p.beta[(size_t)(t0 + tid) * H + h] : 0.f;

    // ---- 1. loads and the cumulative log-decay
    uint4 qv[4], kv[4];
    float g[4][8];
    __syncthreads();  // the barriers are initialised
    tc::mbar_wait(bar_ld, 0, abort, p.err, 10, p.spin);
    // rows of the v tile past the chunk's end (the next sequence, or past the
    // tensor) must not reach the U~ product: zero them (tail chunks only)
    for (int i = tid; i < 2 * (C - L) * 8; i += kPrep2Threads) {
        const int b = i / ((C - L) * 8), rem = i % ((C - L) * 8);
        *reinterpret_cast<uint4 *>(in_v + b * 8192 + (L + (rem >> 3)) * 128 + (rem & 7) * 16) =
            make_uint4(0, 0, 0, 0);
    }
    {
        float run[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) run[j] = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int r = tg * 4 + e;
            uint4 q4 = make_uint4(0, 0, 0, 0), k4 = q4;
            float4 la0 = make_float4(0.f, 0.f, 0.f, 0.f), la1 = la0;
            if (r < L) {  // rows past the chunk's end hold the next sequence (or zero)
                const uint32_t qo = kb * 8192 + r * 128 + ((ck ^ (uint32_t)(r & 7)) << 4);
                q4 = *reinterpret_cast<const uint4 *>(in_q + qo);
                k4 = *reinterpret_cast<const uint4 *>(in_k + qo);
                const uint32_t lb = (uint32_t)(oc >> 2) * 8192 + r * 128, j0 = (uint32_t)(oc & 3) * 2;
                la0 = *reinterpret_cast<const float4 *>(in_la + lb + ((j0 ^ (uint32_t)(r & 7)) << 4));
                la1 = *reinterpret_cast<const float4 *>(in_la + lb + (((j0 + 1) ^ (uint32_t)(r & 7)) << 4));
            }
            qv[e] = q4; kv[e] = k4;
            run[0] += la0.x; run[1] += la0.y; run[2] += la0.z; run[3] += la0.w;
            run[4] += la1.x; run[5] += la1.y; run[6] += la1.z; run[7] += la1.w;
#pragma unroll
            for (int j = 0; j < 8; ++j) g[e][j] = run[j];
        }
        *reinterpret_cast<float4 *>(tot + tg * D + 4 * oc) = make_float4(run[0], run[1], run[2], run[3]);
        *reinterpret_cast<float4 *>(tot + tg * D + 64 + 4 * oc) = make_float4(run[4], run[5], run[6], run[7]);
    }
    __syncthreads();
    if (tid < D) {
        // exclusive prefix over the 16 token groups of channel `tid`, plus the
        // per-channel constants of the factorised exponentials; rows of tot and
        // cst keep channel 8 o + 4 u + e at 64 u + 4 o + e, so that the 16
        // octets of a warp read each half of their 8 channels as one
        // contiguous 256-byte line
        const int pos = ((tid >> 2) & 1) * 64 + (tid >> 3) * 4 + (tid & 3);
        float run = 0.f, g15 = 0.f, g31 = 0.f;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            if (q == 4) g15 = run;
            if (q == 8) g31 = run;
            const float v = tot[q * D + pos];
            tot[q * D + pos] = run;
            run += v;
        }
        const float gC = run;
        cst[0 * D + pos] = g15;
        cst[1 * D + pos] = g31;
        cst[2 * D + pos] = gC;
        cst[3 * D + pos] = __expf(-g15);
        cst[4 * D + pos] = __expf(-g31);
        cst[5 * D + pos] = __expf(g15 - gC);
        cst[6 * D + pos] = __expf(g31 - gC);
        reinterpret_cast<float *>(sm + Prep2Smem::kF)[tid] = __expf(gC - g31);
        reinterpret_cast<float *>(p.rec + ((size_t)c * H + h) * Record::kBytes + Record::kG)[tid] =
            __expf(gC);
    }
    // Multiplicative factors are exact while e^{g} cannot underflow; otherwise
    // take every factor as a direct exponential of its difference.
    // (cst rows are permuted; threads 0..127 cover every channel either way)
    const bool fast = __syncthreads_and(tid >= D || cst[2 * D + tid] > -80.f);

    uint8_t *rec = p.rec + ((size_t)c * H + h) * Record::kBytes;
    {
        const float4 lo = *reinterpret_cast<const float4 *>(tot + tg * D + 4 * oc);
        const float4 hi = *reinterpret_cast<const float4 *>(tot + tg * D + 64 + 4 * oc);
        const float go[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
#pragma unroll
            for (int e = 0; e < 4; ++e) g[e][j] += go[j];
        }
    }
    bool clamped = false;
    auto cexp = [&](float x) { if (x > 80.f) { clamped = true; x = 80.f; } return __expf(x); };
    auto ld8 = [&](int row, float *a) {  // 8 per-channel constants of this octet
        const float4 x = *reinterpret_cast<const float4 *>(cst + row * D + 4 * oc);
        const float4 y = *reinterpret_cast<const float4 *>(cst + row * D + 64 + 4 * oc);
        a[0] = x.x; a[1] = x.y; a[2] = x.z; a[3] = x.w; a[4] = y.x; a[5] = y.y; a[6] = y.z; a[7] = y.w;
    };
    const bool first_half = tg < 8;
    uint32_t khp[8][2];  // K^ of this thread's 4 tokens as bf16 pairs, per channel
    float kh_even[8];
    // Products that only feed bf16 operands are formed in packed bf16 (two per
    // instruction): the factor is rounded to bf16 once, the product once more.
    auto to2 = [](const float *a, __nv_bfloat162 *b2) {
#pragma unroll
        for (int j = 0; j < 4; ++j) b2[j] = __floats2bfloat162_rn(a[2 * j], a[2 * j + 1]);
    };
    auto mul4 = [](const uint4 &x, const __nv_bfloat162 *f) {
        const __nv_bfloat162 *x2 = reinterpret_cast<const __nv_bfloat162 *>(&x);
        uint4 r;
        __nv_bfloat162 *r2 = reinterpret_cast<__nv_bfloat162 *>(&r);
#pragma unroll
        for (int j = 0; j < 4; ++j) r2[j] = __hmul2(x2[j], f[j]);
        return r;
    };
    // g_C of this thread's channels, once for its 4 tokens; the fast form's
    // reference-token factors (first half: e^{-g_15}, e^{g_15 - g_C},
    // e^{g_31 - g_C}; second half: e^{-g_31}, e^{g_31 - g_C}) are read from
    // shared memory per token, which keeps the loop inside the register
    // budget of two CTAs per SM without spilling
    float cC[8];
    ld8(2, cC);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int r = tg * 4 + e;
        const uint32_t sw = ((ck ^ (uint32_t)(r & 7)) << 4);  // swizzled chunk offset
        const float *ge = g[e];
        const uint4 qe = qv[e], ke = kv[e];
        float E[8], Hh[8];
        __nv_bfloat162 f2[4];
#pragma unroll
        for (int j = 0; j < 8; ++j) { E[j] = __expf(ge[j]); Hh[j] = __expf(cC[j] - ge[j]); }
        // Q~ = e^{g} q into the Q' slot of the record (read back for Q' = Q~ - P W),
        // and K~ = e^{g} k, the B operand of W = [T Diag(beta); P] K~
        to2(E, f2);
        *reinterpret_cast<uint4 *>(rec + Record::kBk + kb * Record::kBlk + Record::kOut + r * 128 +
                                   sw) = mul4(qe, f2);
        *reinterpret_cast<uint4 *>(sm + Prep2Smem::kBK + kb * 8192 + r * 128 + sw) = mul4(ke, f2);
        {   // K^ = e^{g_C - g} k, paired over consecutive tokens for the transposed image
            const __nv_bfloat162 *k2 = reinterpret_cast<const __nv_bfloat162 *>(&ke);
            float kh[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                kh[2 * j] = Hh[2 * j] * __low2float(k2[j]);
                kh[2 * j + 1] = Hh[2 * j + 1] * __high2float(k2[j]);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (e & 1) khp[j][e >> 1] = pack_bf16x2(kh_even[j], kh[j]);
                else kh_even[j] = kh[j];
            }
        }
        // factors for the A/P contraction: row factor (k and q rows) and the
        // column factor(s) (k rows of the B operand)
        float ref[8];
        if (first_half) {
            float c0f[8], c1f[8];
            if (fast) {
                float cx[8], cy[8], cz[8];
                ld8(3, cx); ld8(5, cy); ld8(6, cz);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    E[j] *= cx[j];            // e^{g_r - g_15}
                    c0f[j] = Hh[j] * cy[j];   // e^{g_15 - g_r}
                    c1f[j] = Hh[j] * cz[j];   // e^{g_31 - g_r}
                }
            } else {
                ld8(0, ref);
#pragma unroll
                for (int j = 0; j < 8; ++j) { E[j] = cexp(ge[j] - ref[j]); c0f[j] = cexp(ref[j] - ge[j]); }
                ld8(1, ref);
#pragma unroll
                for (int j = 0; j < 8; ++j) c1f[j] = cexp(ref[j] - ge[j]);
            }
            to2(c0f, f2);
            *reinterpret_cast<uint4 *>(sm + Prep2Smem::kBop + kb * 12288 + r * 128 + sw) = mul4(ke, f2);
            to2(c1f, f2);
            *reinterpret_cast<uint4 *>(sm + Prep2Smem::kBop + kb * 12288 + (32 + r) * 128 + sw) = mul4(ke, f2);
            to2(E, f2);
            *reinterpret_cast<uint4 *>(sm + Prep2Smem::kAop + kb * 16384 + r * 128 + sw) = mul4(ke, f2);
            *reinterpret_cast<uint4 *>(sm + Prep2Smem::kAop + kb * 16384 + (32 + r) * 128 + sw) = mul4(qe, f2);
        } else {
            if (fast) {
                float cx[8], cy[8];
                ld8(4, cx); ld8(6, cy);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    E[j] *= cx[j];            // e^{g_r - g_31}
                    Hh[j] *= cy[j];           // e^{g_31 - g_r}
                }
            } else {
                ld8(1, ref);
#pragma unroll
                for (int j = 0; j < 8; ++j) { E[j] = cexp(ge[j] - ref[j]); Hh[j] = cexp(ref[j] - ge[j]); }
            }
            to2(Hh, f2);
            *reinterpret_cast<uint4 *>(sm + Prep2Smem::kBop + kb * 12288 + (32 + r) * 128 + sw) = mul4(ke, f2);
            to2(E, f2);
            *reinterpret_cast<uint4 *>(sm + Prep2Smem::kAop + kb * 16384 + (32 + r) * 128 + sw) = mul4(ke, f2);
            *reinterpret_cast<uint4 *>(sm + Prep2Smem::kAop + kb * 16384 + (64 + r) * 128 + sw) = mul4(qe, f2);
        }
    }
    // K^ as rows i (channels) over the tokens. The lane 16 apart holds the
    // same 8 channels for the next 4 tokens: the pair swaps halves so that each
    // lane has 4 channels x 8 tokens, one 16-byte chunk of each channel row.
    {
        const bool odd_tg = tg & 1;
        const uint32_t w8 = (uint32_t)tg >> 1;  // 8-token group: chunk of the row
#pragma unroll
        for (int j = 0; j < 4; ++j) {  // channels j (kept by even lanes) and 4 + j (odd)
            const uint32_t k0 = odd_tg ? khp[4 + j][0] : khp[j][0];
            const uint32_t k1 = odd_tg ? khp[4 + j][1] : khp[j][1];
            const uint32_t r0 = __shfl_xor_sync(0xffffffffu, odd_tg ? khp[j][0] : khp[4 + j][0], 16);
            const uint32_t r1 = __shfl_xor_sync(0xffffffffu, odd_tg ? khp[j][1] : khp[4 + j][1], 16);
            const uint32_t i = (uint32_t)(c0 + (odd_tg ? 4 + j : j));
            const uint4 v = odd_tg ? make_uint4(r0, r1, k0, k1) : make_uint4(k0, k1, r0, r1);
            *reinterpret_cast<uint4 *>(rec + Record::kBt + i * 128 + ((w8 ^ (i & 7u)) << 4)) = v;
        }
    }
    // A chunk whose decay inside half a chunk exceeds the factorised range is
    // recomputed exactly by the fixup kernel.
    if (__syncthreads_or(clamped) && tid == 0) p.fix_list[atomicAdd(p.fix_count, 1)] = c * H + h;
    tc::fence_proxy_async_smem();
    tc::tc_fence_before_sync();
    __syncthreads();
    tc::tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    // ---- 2. MMA-AP
    if (tid == 0) {
        const uint32_t a0 = tc::smem_u32(sm + Prep2Smem::kAop);
        const uint32_t b0 = tc::smem_u32(sm + Prep2Smem::kBop);
        const uint32_t id = tc::idesc_bf16(128, 96, 0, 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint64_t a = tc::smem_desc(a0 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
            const uint64_t b = tc::smem_desc(b0 + (kk >> 2) * 12288 + (kk & 3) * 32, 16, 1024);
            tc::mma_bf16(tmem, a, b, id, kk > 0);
        }
        tc::mma_commit(bar_ap);
    }
    float *As = reinterpret_cast<float *>(sm + Prep2Smem::kA);   // A[r][s], stride kLd
    float *Ts = reinterpret_cast<float *>(sm + Prep2Smem::kT);   // T[r][s], stride kLd
    {
        // every warp reads its 32 TMEM lanes; warps 0-3 take the first 32 of the
        // row's 64 relevant columns, warps 4-7 the other 32
        tc::mbar_wait(bar_ap, 0, abort, p.err, 11, p.spin);
        tc::tc_fence_after_sync();
        const int t = (warp & 3) * 32 + (tid & 31);  // accumulator row
        const int sh = (warp >> 2) * 32;             // first s of this thread
        const uint32_t col0 = (t < 64 ? 0u : 32u) + (uint32_t)sh;
        float d[32];
        tc::tmem_ld32_sync(tmem + ((uint32_t)((warp & 3) * 32) << 16) + col0, d);
        const bool is_k = (t & 32) == 0;             // rows 0-31, 64-95 come from k
        const int r = t < 64 ? (t & 31) : 32 + (t & 31);
        const int lim = (t < 64) ? 32 : 64;          // first-half rows see only s < 32
        if (is_k) {
            const float b = sbeta[r];
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
                float v[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int s2 = sh + e + q;
                    v[q] = (s2 < lim && s2 < r) ? b * d[e + q] : 0.f;
                }
                *reinterpret_cast<float4 *>(As + r * kLd + sh + e) = make_float4(v[0], v[1], v[2], v[3]);
            }
        } else {
            uint8_t *prow = sm + Prep2Smem::kP;  // P stays: the record's and MMA-NP's operand
#pragma unroll
            for (int c16 = 0; c16 < 4; ++c16) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int s0 = sh + c16 * 8 + 2 * e;
                    w[e] = pack_bf16x2((s0 < lim && s0 <= r) ? d[c16 * 8 + 2 * e] : 0.f,
                                       (s0 + 1 < lim && s0 + 1 <= r) ? d[c16 * 8 + 2 * e + 1] : 0.f);
                }
                *reinterpret_cast<uint4 *>(prow + tc::sw128(r, (sh / 8 + c16) * 16)) =
                    make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before_sync();
    __syncthreads();
    if (tid == 0) {
        tc::bulk_s2g(rec + Record::kBt + Record::kOut, sm + Prep2Smem::kP, 8192);
        tc::bulk_commit();
    }

    // ---- 3. T = (I + A)^{-1} by 16x16 blocks (rows 64..127 of the W operand
    // [T; P] hold P: they only feed accumulator rows nobody reads)
    invert_unit_lower64(As, Ts, tid);
    {   // [T Diag(beta); P] operand rows 0..63 (K-major, element (r, s) = T[r][s] beta_s,
        // zero above the diagonal)
        const int r = tid >> 2, s0 = (tid & 3) * 16;
        uint8_t *tt = sm + Prep2Smem::kTt;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            // 8 entries of row r as two float4 reads (entries above the
            // diagonal hold the inverse's scratch and are not selected)
            const int sb0 = s0 + h2 * 8;
            const float4 t0 = *reinterpret_cast<const float4 *>(Ts + r * kLd + sb0);
            const float4 t1 = *reinterpret_cast<const float4 *>(Ts + r * kLd + sb0 + 4);
            const float4 b0 = *reinterpret_cast<const float4 *>(sbeta + sb0);
            const float4 b1 = *reinterpret_cast<const float4 *>(sbeta + sb0 + 4);
            const float t8[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
            const float b8[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
            float v8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int sa = sb0 + e;
                v8[e] = (sa < r ? t8[e] : (sa == r ? 1.f : 0.f)) * b8[e];
            }
            *reinterpret_cast<uint4 *>(tt + tc::sw128(r, sb0 * 2)) =
                make_uint4(pack_bf16x2(v8[0], v8[1]), pack_bf16x2(v8[2], v8[3]),
                           pack_bf16x2(v8[4], v8[5]), pack_bf16x2(v8[6], v8[7]));
        }
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before_sync();
    __syncthreads();
    tc::tc_fence_after_sync();

    // ---- 4. W = [T Diag(beta); P] . K~ and U~^T = V^T . (T Diag(beta))^T
    if (tid == 0) {
        const uint32_t bk = tc::smem_u32(sm + Prep2Smem::kBK);  // 2 MN atoms (channels)
        const uint32_t bv = tc::smem_u32(sm + Prep2Smem::kBV);
        const uint32_t tt = tc::smem_u32(sm + Prep2Smem::kTt);
        const uint32_t idw = tc::idesc_bf16(128, 128, 0, 1);  // rows: tokens (64 used)
        const uint32_t idu = tc::idesc_bf16(128, 64, 1, 0);   // rows: value columns
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            tc::mma_bf16(tmem, tc::smem_desc(tt + kk * 32, 16, 1024),
                         tc::smem_desc(bk + kk * 2048, 8192, 1024), idw, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            tc::mma_bf16(tmem + 128, tc::smem_desc(bv + kk * 2048, 8192, 1024),
                         tc::smem_desc(tt + kk * 32, 16, 1024), idu, kk > 0);
        tc::mma_commit(bar_wu);
    }
    FinishSmem fs;
    fs.w = Prep2Smem::kW; fs.us = Prep2Smem::kUs; fs.pp = Prep2Smem::kP;
    // K^ = e^{g_C - g_31} (k e^{g_31 - g}): the B operand's reference-31 rows times a
    // per-channel factor, which scales the rows of N = K^^T W
    fs.kh = Prep2Smem::kKh; fs.kh_lbo = 12288; fs.kh_scale = Prep2Smem::kF;
    fs.n0 = Prep2Smem::kN0; fs.n1 = Prep2Smem::kN1; fs.qp = Prep2Smem::kQp;
    // Q~ of row t: written by step 1 into the record's Q' slot (read back from L2)
    auto qload = [&](int t, int kb2, int hl, uint4 *raw) {
        const uint8_t *row = rec + Record::kBk + kb2 * Record::kBlk + Record::kOut + t * 128;
#pragma unroll
        for (int c16 = 0; c16 < 4; ++c16)
            raw[c16] = *reinterpret_cast<const uint4 *>(
                row + ((((uint32_t)(4 * hl + c16)) ^ ((uint32_t)t & 7u)) << 4));
    };
    auto qconv = [&](int, const uint4 &x, float *q8) {
        const __nv_bfloat162 *x2 = reinterpret_cast<const __nv_bfloat162 *>(&x);
#pragma unroll
        for (int e = 0; e < 4; ++e) { q8[2 * e] = __low2float(x2[e]); q8[2 * e + 1] = __high2float(x2[e]); }
    };
    finish_record(sm, fs, tmem, rec, bar_wu, bar_ld + 2, bar_ld, bar_ld + 1, abort, p, 12, qload,
                  qconv);
    if (warp == 0) {
        __syncwarp();
        tc::tc_fence_after_sync();
        tc::tmem_dealloc(tmem, 256);
    }
}

// ------------------------------------------------------------------- GDN prep
// Gate shared by all channels (one log-decay per token and head, the gated
// DeltaNet case of the rule). With g_r the chunk's inclusive cumulative
// log-decay, every decay factor of A and P is e^{g_r - g_s} <= 1 (s <= r) and
// comes out of the channel contraction, so
//     A_rs = beta_r e^{g_r - g_s} (K K^T)_rs  (s < r),   P_rs = e^{g_r - g_s} (Q K^T)_rs  (s <= r)
// come from one MMA on the raw bf16 tiles, D (128x64) = [K; Q] . K^T, scaled in
// the epilogue: no reference tokens and no fixup. The diagonal scalings of the
// solve fold into T: W = (T Diag(beta e^g)) K and U~^T = V^T (T Diag(beta))^T.
// The record is the one the carry kernel reads for per-channel gates, with
// gamma = e^{g_C} in every channel. One CTA per (chunk, head), 256 threads.
constexpr int kGdnThreads = 256;

struct GdnSmem {
    static constexpr uint32_t kQK = 0;        // 32768: [K; Q] bf16, K-major SW128, 2 K-blocks x 128 rows
    static constexpr uint32_t kV = 32768;     // 16384: V bf16, [channel block][64 tokens][128 B] SW128
    static constexpr uint32_t kA = 49152;     // fp32 A [64][kLd]
    static constexpr uint32_t kT = 66560;     // fp32 T [64][kLd]
    static constexpr uint32_t kY = 83968;     // fp32 3 x [16][16] block products
    static constexpr uint32_t kTw = 87040;    // 16384: [T Diag(beta e^g); 0] bf16, K-major rows r
    static constexpr uint32_t kTu = 103424;   // 8192:  T Diag(beta) bf16, K-major rows r
    static constexpr uint32_t kG = 111616;    // fp32 g [64], beta [64]
    static constexpr uint32_t kBar = 112128;  // barriers + tmem slot + flags
    static constexpr uint32_t kE = kBar + 64; // fp32 e^{g} [64], e^{g_C - g} [64]
    static constexpr uint32_t kBytes = kE + 512 + 1024;
    // Later tenants (each region is dead by then):
    static constexpr uint32_t kP = kTw + 8192;  // 8192:  P, from the A/P read-out to MMA-NP
    static constexpr uint32_t kKhT = 49152;     // 16384: K^ rows i, after the T images
    static constexpr uint32_t kW = 65536;       // 16384: W bf16 image, after MMA-WU
};
static_assert(GdnSmem::kA == GdnSmem::kV + 16384 && GdnSmem::kT == GdnSmem::kA + 64 * kLd * 4 &&
              GdnSmem::kY == GdnSmem::kT + 64 * kLd * 4 && GdnSmem::kTw >= GdnSmem::kY + 3072 &&
              GdnSmem::kTw % 1024 == 0 && GdnSmem::kTu % 1024 == 0 &&
              GdnSmem::kG == GdnSmem::kTu + 8192, "GDN prep layout");

__global__ void __launch_bounds__(kGdnThreads, 2) tc_gdn_prep_kernel(const __grid_constant__ TcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar_ap = reinterpret_cast<uint64_t *>(sm + GdnSmem::kBar);
    uint64_t *bar_wu = bar_ap + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_ap + 2);
    volatile int *abort = reinterpret_cast<volatile int *>(bar_ap + 3);
    uint64_t *bar_ld = bar_ap + 4;
    float *sg = reinterpret_cast<float *>(sm + GdnSmem::kG);
    float *sbeta = sg + C;
    float *seg = reinterpret_cast<float *>(sm + GdnSmem::kE);  // e^{g_t}
    float *segk = seg + C;                                       // e^{g_C - g_t}

    const int c = blockIdx.x, h = blockIdx.y, H = p.H;
    ChunkLoc loc;
    if (!locate_chunk(p, c, loc)) return;  // uniform over the CTA: nothing allocated yet
    const int t0 = loc.t0, L = loc.L;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // ---- 1. k, q, v straight into their operand layouts: six TMA tiles of 64
    // channels x 64 tokens (the 128-byte swizzle is the operand swizzle)
    if (tid == 0) {
        tc::mbar_init(bar_ap, 1);
        tc::mbar_init(bar_wu, 1);
        tc::mbar_init(bar_ld, 1);
        tc::mbar_init(bar_ld + 1, 1);  // bar_fin
        tc::mbar_init(bar_ld + 2, 1);  // bar_np
        *abort = 0;
        tc::fence_mbar_init();
        tc::mbar_arrive_expect_tx(bar_ld, 6 * 8192);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
            tc::tma_load_3d(sm + GdnSmem::kQK + kb * 16384, &p.tm_k, 64 * kb, h, t0, bar_ld);
            tc::tma_load_3d(sm + GdnSmem::kQK + kb * 16384 + 8192, &p.tm_q, 64 * kb, h, t0, bar_ld);
            tc::tma_load_3d(sm + GdnSmem::kV + kb * 8192, &p.tm_v, 64 * kb, h, t0, bar_ld);
        }
    }
    if (warp == 0) { tc::tmem_alloc(tmem_slot, 256); tc::tmem_relinquish(); }
    if (warp == 1) {
        // inclusive cumulative log-decay of the 64 tokens, two per lane
        const int r0 = 2 * lane, r1 = r0 + 1;
        const float a0 = r0 < L ? p.log_alpha[(size_t)(t0 + r0) * H + h] : 0.f;
        const float a1 = r1 < L ? p.log_alpha[(size_t)(t0 + r1) * H + h] : 0.f;
        float run = a0 + a1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, run, off);
            if (lane >= off) run += y;
        }
        sg[r1] = run;
        sg[r0] = run - a1;
        // the exponentials every later step needs, once per token
        const float gC = __shfl_sync(0xffffffffu, run, 31);
        seg[r0] = __expf(run - a1);
        seg[r1] = __expf(run);
        segk[r0] = __expf(gC - (run - a1));
        segk[r1] = __expf(gC - run);
    } else if (warp == 2) {
        for (int r = lane; r < C; r += 32) sbeta[r] = r < L ? p.beta[(size_t)(t0 + r) * H + h] : 0.f;
    }
    // rows past the chunk's end (the next sequence, or past the tensor) read zero
    __syncthreads();  // the barriers are initialised
    tc::mbar_wait(bar_ld, 0, abort, p.err, 20, p.spin);
    for (int i = tid; i < 6 * (C - L) * 8; i += kGdnThreads) {
        const int tile = i / ((C - L) * 8), rem = i % ((C - L) * 8);
        const int r = L + (rem >> 3);
        uint8_t *base = tile < 4 ? sm + GdnSmem::kQK + (tile >> 1) * 16384 + (tile & 1) * 8192
                                 : sm + GdnSmem::kV + (tile - 4) * 8192;
        *reinterpret_cast<uint4 *>(base + r * 128 + (rem & 7) * 16) = make_uint4(0, 0, 0, 0);
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before_sync();
    __syncthreads();
    tc::tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    // ---- 2. D (128x64) = [K; Q] . K^T: rows 0..63 K K^T, rows 64..127 Q K^T
    if (tid == 0) {
        const uint32_t a0 = tc::smem_u32(sm + GdnSmem::kQK);
        const uint32_t id = tc::idesc_bf16(128, 64, 0, 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint64_t d = tc::smem_desc(a0 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
            tc::mma_bf16(tmem, d, d, id, kk > 0);  // B = the K rows (the first 64) of A
        }
        tc::mma_commit(bar_ap);
    }
    // ---- 3. gamma, while the MMA runs
    uint8_t *rec = p.rec + ((size_t)c * H + h) * Record::kBytes;
    const float gC = sg[C - 1];
    if (tid < D) reinterpret_cast<float *>(rec + Record::kG)[tid] = __expf(gC);

    // ---- 4. A (fp32, strictly lower, beta-scaled) and P (record) from D
    float *As = reinterpret_cast<float *>(sm + GdnSmem::kA);
    float *Ts = reinterpret_cast<float *>(sm + GdnSmem::kT);
    float *Ys = reinterpret_cast<float *>(sm + GdnSmem::kY);
    {
        tc::mbar_wait(bar_ap, 0, abort, p.err, 21, p.spin);
        tc::tc_fence_after_sync();
        const int t = (warp & 3) * 32 + lane;  // accumulator row
        const int sh = (warp >> 2) * 32;       // first column s of this thread
        float d[32];
        tc::tmem_ld32_sync(tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)sh, d);
        if (t < C) {
            const int r = t;
            const float gr = sg[r], b = sbeta[r];
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
                float v[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int s2 = sh + e + q;
                    v[q] = s2 < r ? b * __expf(gr - sg[s2]) * d[e + q] : 0.f;
                }
                *reinterpret_cast<float4 *>(As + r * kLd + sh + e) = make_float4(v[0], v[1], v[2], v[3]);
            }
        } else {
            const int r = t - C;
            const float gr = sg[r];
            uint8_t *prow = sm + GdnSmem::kP;  // P stays: the record's and MMA-NP's operand
#pragma unroll
            for (int c16 = 0; c16 < 4; ++c16) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int s0 = sh + c16 * 8 + 2 * e;
                    w[e] = pack_bf16x2(s0 <= r ? __expf(gr - sg[s0]) * d[c16 * 8 + 2 * e] : 0.f,
                                       s0 + 1 <= r ? __expf(gr - sg[s0 + 1]) * d[c16 * 8 + 2 * e + 1] : 0.f);
                }
                *reinterpret_cast<uint4 *>(prow + tc::sw128(r, (sh / 8 + c16) * 16)) =
                    make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before_sync();
    __syncthreads();
    if (tid == 0) {
        tc::bulk_s2g(rec + Record::kBt + Record::kOut, sm + GdnSmem::kP, 8192);
        tc::bulk_commit();
    }

    // ---- 5. T = (I + A)^{-1}, then the two scaled T images (rows 64..127 of
    // the W operand's A hold P: they only feed accumulator rows nobody reads)
    invert_unit_lower64_by_distance(As, Ts, Ys, tid);
    {
        const int r = tid >> 2, s0 = (tid & 3) * 16;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int sb0 = s0 + h2 * 8;
            // 8 entries of row r as float4 reads (entries above the diagonal hold
            // the inverse's scratch and are not selected)
            const float4 t0 = *reinterpret_cast<const float4 *>(Ts + r * kLd + sb0);
            const float4 t1 = *reinterpret_cast<const float4 *>(Ts + r * kLd + sb0 + 4);
            const float4 b0 = *reinterpret_cast<const float4 *>(sbeta + sb0);
            const float4 b1 = *reinterpret_cast<const float4 *>(sbeta + sb0 + 4);
            const float4 e0 = *reinterpret_cast<const float4 *>(seg + sb0);
            const float4 e1 = *reinterpret_cast<const float4 *>(seg + sb0 + 4);
            const float t8[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
            const float b8[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
            const float e8[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
            uint32_t ww[4], wu[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int sa = sb0 + 2 * e, sb2 = sa + 1;
                const float ta = sa < r ? t8[2 * e] : (sa == r ? 1.f : 0.f);
                const float tb = sb2 < r ? t8[2 * e + 1] : (sb2 == r ? 1.f : 0.f);
                const float ba = b8[2 * e] * ta, bb = b8[2 * e + 1] * tb;
                wu[e] = pack_bf16x2(ba, bb);
                ww[e] = pack_bf16x2(ba * e8[2 * e], bb * e8[2 * e + 1]);
            }
            const uint32_t off = tc::sw128(r, sb0 * 2);
            *reinterpret_cast<uint4 *>(sm + GdnSmem::kTw + off) = make_uint4(ww[0], ww[1], ww[2], ww[3]);
            *reinterpret_cast<uint4 *>(sm + GdnSmem::kTu + off) = make_uint4(wu[0], wu[1], wu[2], wu[3]);
        }
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before_sync();
    __syncthreads();
    tc::tc_fence_after_sync();

    // ---- 6. W = [T Diag(beta e^g); 0] . K and U~^T = V^T . (T Diag(beta))^T
    if (tid == 0) {
        const uint32_t kq = tc::smem_u32(sm + GdnSmem::kQK);  // K rows as MN-major B: atoms 16 KB apart
        const uint32_t vv = tc::smem_u32(sm + GdnSmem::kV);
        const uint32_t tw = tc::smem_u32(sm + GdnSmem::kTw);
        const uint32_t tu = tc::smem_u32(sm + GdnSmem::kTu);
        const uint32_t idw = tc::idesc_bf16(128, 128, 0, 1);
        const uint32_t idu = tc::idesc_bf16(128, 64, 1, 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            tc::mma_bf16(tmem, tc::smem_desc(tw + kk * 32, 16, 1024),
                         tc::smem_desc(kq + kk * 2048, 16384, 1024), idw, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            tc::mma_bf16(tmem + 128, tc::smem_desc(vv + kk * 2048, 8192, 1024),
                         tc::smem_desc(tu + kk * 32, 16, 1024), idu, kk > 0);
        tc::mma_commit(bar_wu);
    }
    // K^ = e^{g_C - g_t} k_t as rows i over the tokens (the record's image and
    // MMA-NP's A operand), from the raw k tile while the MMAs run: thread ->
    // channel i, 8 tokens of chunk cq; a warp reads one tile row per token
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int gi = tid + kGdnThreads * j;
        const int cq = gi >> 7, i = gi & 127;
        const uint32_t kb = (uint32_t)(i >> 6), ib = 2u * (uint32_t)(i & 63);
        float kh[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int t = 8 * cq + e;
            const __nv_bfloat16 x = *reinterpret_cast<const __nv_bfloat16 *>(
                sm + GdnSmem::kQK + kb * 16384 + tc::sw128((uint32_t)t, ib));
            kh[e] = segk[t] * __bfloat162float(x);
        }
        *reinterpret_cast<uint4 *>(sm + GdnSmem::kKhT + tc::sw128((uint32_t)i, 16u * (uint32_t)cq)) =
            make_uint4(pack_bf16x2(kh[0], kh[1]), pack_bf16x2(kh[2], kh[3]),
                       pack_bf16x2(kh[4], kh[5]), pack_bf16x2(kh[6], kh[7]));
    }
    tc::fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
        tc::bulk_s2g(rec + Record::kBt, sm + GdnSmem::kKhT, 16384);
        tc::bulk_commit();
    }
    FinishSmem fs;
    fs.w = GdnSmem::kW; fs.us = GdnSmem::kV; fs.pp = GdnSmem::kP;
    fs.kh = GdnSmem::kKhT; fs.kh_lbo = 0; fs.kh_scale = 0;
    fs.n0 = GdnSmem::kKhT; fs.n1 = GdnSmem::kW; fs.qp = GdnSmem::kTw;
    // Q~ of row t: e^{g_t} times the raw q tile (rows 64.. of the [K; Q] buffer)
    auto qload = [&](int t, int kb2, int hl, uint4 *raw) {
        const uint8_t *row = sm + GdnSmem::kQK + kb2 * 16384 + (64 + t) * 128;
#pragma unroll
        for (int c16 = 0; c16 < 4; ++c16)
            raw[c16] = *reinterpret_cast<const uint4 *>(
                row + ((((uint32_t)(4 * hl + c16)) ^ ((uint32_t)t & 7u)) << 4));
    };
    auto qconv = [&](int t, const uint4 &x, float *q8) {
        const __nv_bfloat162 *x2 = reinterpret_cast<const __nv_bfloat162 *>(&x);
        const float et = seg[t];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            q8[2 * e] = et * __low2float(x2[e]);
            q8[2 * e + 1] = et * __high2float(x2[e]);
        }
    };
    finish_record(sm, fs, tmem, rec, bar_wu, bar_ld + 2, bar_ld, bar_ld + 1, abort, p, 22, qload,
                  qconv);
    if (warp == 0) {
        __syncwarp();
        tc::tc_fence_after_sync();
        tc::tmem_dealloc(tmem, 256);
    }
}

// ------------------------------------------------------------------- carry
// The state slice is carried transposed, S^T (64 value columns x 128 key
// channels). With N = K^^T W and Q' = Q~ - P W precomputed per chunk, one
// chunk step is a single product with the slice's 64 value columns on the M
// side:
//     D = U~^T . [K^ | P^T]  +  S^T . [-N^T | Q'^T]       (64 x 192)
// whose columns 0..127 are the state increment and columns 128..191 the
// output, since U = U~ - W S gives
//     S_next^T = S^T Diag(gamma) + D[:, :128],   O^T = scale * D[:, 128:].
// The U~ part does not depend on S, so it is issued as soon as the record has
// landed ("early", 4 K-steps over the tokens); the S part (8 K-steps over the
// keys) follows the moment the state warps have written bf16 S^T. D is
// double-buffered in TMEM, and S^T in shared memory, so the early group of
// chunk c+1 and the state update of chunk c overlap.
// An M = 64 accumulator keeps row m in TMEM lane 32*(m/16) + m%16; warp w reads
// rows 16*(w%4) .. +15 with the 16x32bx2 shape, lanes 0-15 and 16-31 splitting
// the columns. Warps 0-7 own the state: thread (w, l) keeps S^T row
// 16*(w%4) + l%16, key channels 64*(w/4) + 32*(l/16) .. +31, in fp32 registers,
// and stores output tokens 32*(w/4) + 16*(l/16) .. +15 of that value column.
// Warp 8 streams the records into a two-stage ring with bulk copies; warp 9
// issues the MMAs. Per chunk the state warps and the MMA warp meet once at a
// named barrier (S^T of the chunk complete), also after a wait has given up,
// so their generations never mix.
constexpr int kCarryThreads = 320;
constexpr int kCarrySync = 288;      // state warps + the MMA warp
constexpr uint32_t kTmemCols = 512;  // D[0]: [0,192), D[1]: [256,448)

enum { kErrFull = 1, kErrEmpty, kErrD, kErrUnused, kErrUnused2, kErrDrain };

__device__ __forceinline__ void named_bar(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__global__ void __launch_bounds__(kCarryThreads, 1) tc_carry_kernel(TcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + CarrySmem::kBar);
    uint64_t *full = bars + 0;     // [2] record landed
    uint64_t *empty = bars + 2;    // [2] 8 state warps + the MMA commit
    uint64_t *d_done = bars + 4;   // chunk's MMAs completed (one phase per chunk)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 5);
    volatile int *abort = reinterpret_cast<volatile int *>(bars + 6);
    uint64_t *drain = bars + 7;    // all MMAs of the CTA completed

    // The CTA's job: (sequence, head, half), a range of the sequence's chunks,
    // where its state starts and ends, and whether it writes outputs.
    //  pass 0 (no split): one CTA per (sequence, head, half), sequences longest
    //    first; the whole sequence from S0 to S_final, with outputs.
    //  pass 1 of a split into P segments: per (sequence, head), segment 0 from
    //    S0 with outputs (its end state kept), and for every later segment p the
    //    state from a zero start and the transition (the product of the chunk
    //    steps' linear parts, carried like a state that starts at the identity
    //    and has no U~ term), both without outputs: 2 + 4 (P - 1) CTAs.
    //  pass 2: every segment p >= 1 again from its true entry state (the end
    //    state of segment p - 1, combined in between), with outputs; the last
    //    segment writes S_final: 2 (P - 1) CTAs.
    const int H = p.H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int half, h, n, seg = 0;
    const float *S_in;
    float *S_out;
    bool outputs = true, transition = false;
    const size_t blk = (size_t)D * D;
    auto seg_block = [&](int kind, int sp, int sn, int sh) {
        return p.seg + ((((size_t)kind * p.nseg + sp) * p.N + sn) * H + sh) * blk;
    };
    if (p.pass == 0) {
        half = blockIdx.x % kSlices;
        h = (blockIdx.x / kSlices) % H;
        n = p.order[blockIdx.x / (kSlices * H)];
        S_in = p.S0 ? p.S0 + ((size_t)n * H + h) * blk : nullptr;
        S_out = p.S_final ? p.S_final + ((size_t)n * H + h) * blk : nullptr;
    } else if (p.pass == 1) {
        const int Q = 2 + 4 * (p.nseg - 1), q = blockIdx.x % Q, u = blockIdx.x / Q;
        h = u % H;
        n = p.order[u / H];
        if (q < 2) {
            half = q;
            S_in = p.S0 ? p.S0 + ((size_t)n * H + h) * blk : nullptr;
            S_out = seg_block(2, 0, n, h);
        } else {
            const int r = q - 2;
            seg = 1 + r / 4;
            half = r & 1;
            transition = (r >> 1) & 1;
            outputs = false;
            S_in = nullptr;
            S_out = seg_block(transition ? 1 : 0, seg, n, h);
        }
    } else {
        const int Q = 2 * (p.nseg - 1), q = blockIdx.x % Q, u = blockIdx.x / Q;
        h = u % H;
        n = p.order[u / H];
        seg = 1 + q / 2;
        half = q & 1;
        S_in = seg_block(2, seg - 1, n, h);
        S_out = (seg == p.nseg - 1 && p.S_final) ? p.S_final + ((size_t)n * H + h) * blk : nullptr;
    }

    if (threadIdx.x == 0) {
        tc::mbar_init(&full[0], 1); tc::mbar_init(&full[1], 1);
        tc::mbar_init(&empty[0], 9); tc::mbar_init(&empty[1], 9);
        tc::mbar_init(d_done, 1);
        tc::mbar_init(drain, 1);
        *abort = 0;
        tc::fence_mbar_init();
    }
    if (warp == 0) { tc::tmem_alloc(tmem_slot, kTmemCols); tc::tmem_relinquish(); }
    tc::tc_fence_before_sync();
    __syncthreads();
    tc::tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    const int te = p.seq_start[n + 1];
    int c0 = p.chunk_off[n], nc = p.chunk_off[n + 1] - c0;
    if (p.pass != 0) {  // this segment's chunks: [nc p / P, nc (p + 1) / P)
        const int b0 = (int)((long long)nc * seg / p.nseg);
        const int b1 = (int)((long long)nc * (seg + 1) / p.nseg);
        c0 += b0;
        nc = b1 - b0;
    }
    // first token of the CTA's first chunk
    const int ts = p.seq_start[n] + (c0 - p.chunk_off[n]) * C;
    constexpr uint32_t kStageBytes = 49152 + 24576 + 8192 + 512;

    if (warp == 8) {
        // ---------------- producer: one record per chunk into the two-stage ring
        if (lane == 0) {
            // Records of the chunks kAhead ahead are prefetched into L2, so that
            // a stage's copy, issued as soon as the stage is released (about one
            // chunk step before the MMAs need it), reads L2 rather than DRAM.
            constexpr int kAhead = 4;
            auto prefetch = [&](int lc) {
                const uint8_t *rec = p.rec + ((size_t)(c0 + lc) * H + h) * Record::kBytes;
                tc::bulk_prefetch_l2(rec, Record::kU);  // both B ranges
                tc::bulk_prefetch_l2(rec + Record::kU + half * 8192, 8192);
                tc::bulk_prefetch_l2(rec + Record::kG, 512);
            };
            for (int lc = 2; lc < nc && lc < 2 + kAhead && !p.starve; ++lc) prefetch(lc);
            int issued = 0;
            for (int lc = 0; lc < nc && !p.starve; ++lc) {
                const int st = lc & 1;
                if (lc + 2 + kAhead < nc) prefetch(lc + 2 + kAhead);
                if (lc >= 2 && !tc::mbar_wait(&empty[st], ((lc >> 1) - 1) & 1, abort, p.err,
                                              kErrEmpty, p.spin))
                    break;
                if (*abort) break;
                const uint8_t *rec = p.rec + ((size_t)(c0 + lc) * H + h) * Record::kBytes;
                uint8_t *sb = sm + st * CarrySmem::kStage;
                tc::mbar_arrive_expect_tx(&full[st], kStageBytes);
                tc::bulk_g2s(sb + CarrySmem::kBk, rec + Record::kBk, 49152, &full[st]);
                tc::bulk_g2s(sb + CarrySmem::kBt, rec + Record::kBt, 24576, &full[st]);
                tc::bulk_g2s(sb + CarrySmem::kU, rec + Record::kU + half * 8192, 8192, &full[st]);
                tc::bulk_g2s(sb + CarrySmem::kG, rec + Record::kG, 512, &full[st]);
                issued = lc + 1;
            }
            // every issued copy has landed before the CTA may exit (also after
            // an abort: the copies write this CTA's shared memory)
            for (int lc = (issued > 2 ? issued - 2 : 0); lc < issued; ++lc)
                tc::mbar_drain(&full[lc & 1], (lc >> 1) & 1, p.err, kErrFull, p.spin);
        }
    } else if (warp == 9) {
        // ---------------- MMA issue
        // the transition needs only the state columns and no U~ term
        const uint32_t id = tc::idesc_bf16(64, transition ? 128 : 192, 0, 0);
        const uint32_t a_s0 = tc::smem_u32(sm + CarrySmem::kSt);
        bool issued = false;
        for (int lc = 0; lc < nc; ++lc) {
            const int st = lc & 1;
            const uint32_t sb = tc::smem_u32(sm + st * CarrySmem::kStage);
            const uint32_t d = tmem + (uint32_t)st * 256;
            // after an abort no MMA is issued; the barrier is still met
            bool go = false;
            if (lane == 0) {
                go = tc::mbar_wait(&full[st], (lc >> 1) & 1, abort, p.err, kErrFull, p.spin) &&
                     !*abort;
                if (go && !transition) {  // early: D = U~^T . [K^ | P^T]
                    issued = true;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::mma_bf16(d, tc::smem_desc(sb + CarrySmem::kU + kk * 32, 16, 1024),
                                     tc::smem_desc(sb + CarrySmem::kBt + kk * 32, 16, 1024), id,
                                     kk > 0);
                }
            }
            __syncwarp();
            named_bar(1, kCarrySync);  // S^T of this chunk complete
            if (lane == 0 && go && !*abort) {
                issued = true;
                tc::tc_fence_after_sync();
                const uint32_t a_s = a_s0 + (uint32_t)st * 16384;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_bf16(d, tc::smem_desc(a_s + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                                 tc::smem_desc(sb + CarrySmem::kBk + (kk >> 2) * Record::kBlk +
                                               (kk & 3) * 32, 16, 1024),
                                 id, (transition && kk == 0) ? 0u : 1u);
                tc::mma_commit(d_done);
                tc::mma_commit(&empty[st]);
            }
            __syncwarp();
        }
        // every MMA this thread issued has finished before TMEM is released
        if (lane == 0 && issued) {
            tc::mma_commit(drain);
            tc::mbar_drain(drain, 0, p.err, kErrDrain, p.spin);
        }
        __syncwarp();
    } else {
        // ---------------- state owners
        const int lg = warp & 3, wh = warp >> 2, hl = lane >> 4;
        const int cr = 16 * lg + (lane & 15);  // S^T row: value column inside the slice
        const int kc0 = 64 * wh + 32 * hl;     // first key channel of this thread
        const uint32_t lane_base = tmem + ((uint32_t)(lg * 32) << 16);
        float S[32];
        const size_t sbase = (size_t)kc0 * D + half * kSlice + cr;  // inside a (sequence, head) block
        if (transition) {  // the identity: S^T row (half * 64 + cr) is that unit vector
#pragma unroll
            for (int j = 0; j < 32; ++j) S[j] = (kc0 + j == half * kSlice + cr) ? 1.f : 0.f;
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) S[j] = S_in ? S_in[sbase + (size_t)j * D] : 0.f;
        }
        // bf16 S^T row cr, channels kc0..kc0+31: 4 of the row's 8 swizzled
        // 16-byte chunks in K-block wh of buffer `buf`
        auto store_st = [&](int buf) {
            uint8_t *base = sm + CarrySmem::kSt + buf * 16384 + wh * 8192;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) w[e] = pack_bf16x2(S[8 * q + 2 * e], S[8 * q + 2 * e + 1]);
                *reinterpret_cast<uint4 *>(base + tc::sw128(cr, (4 * hl + q) * 16)) =
                    make_uint4(w[0], w[1], w[2], w[3]);
            }
        };
        // store_o sends the warp's 16 value columns x 32 tokens of chunk lc
        // through a 1 KB staging tile (token rows of 32 bytes, value pairs
        // packed with one shuffle), then to o with two 16-byte stores per lane.
        uint8_t *os = sm + CarrySmem::kOs + warp * 1024;
        float ov[16];
        auto store_o = [&](int lc) {
            const bool odd = lane & 1;
            const int l15 = lane & 15;
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
                // even lane: token j, columns (l15, l15+1); odd lane: token j+1, (l15-1, l15)
                const float x = __shfl_xor_sync(0xffffffffu, odd ? ov[j] : ov[j + 1], 1);
                const int row = 16 * hl + j + (odd ? 1 : 0);
                const uint32_t w = odd ? pack_bf16x2(p.scale * x, p.scale * ov[j + 1])
                                       : pack_bf16x2(p.scale * ov[j], p.scale * x);
                *reinterpret_cast<uint32_t *>(os + row * 32 + (l15 & ~1) * 2) = w;
            }
            __syncwarp();
            const int t0 = ts + lc * C;
            const int L = min(C, te - t0);
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int k = lane + 32 * i;           // 16-byte piece: token row k/2, half k&1
                const int tok = 32 * wh + (k >> 1);
                if (tok < L)
                    *reinterpret_cast<uint4 *>(p.o + ((size_t)(t0 + tok) * H + h) * D + half * kSlice +
                                               16 * lg + 8 * (k & 1)) =
                        *reinterpret_cast<const uint4 *>(os + k * 16);
            }
            __syncwarp();
        };
        if (nc > 0) {
            store_st(0);
            tc::fence_proxy_async_smem();
            tc::tc_fence_before_sync();
            named_bar(1, kCarrySync);  // S^T of chunk 0 complete
        }
        for (int lc = 0; lc < nc; ++lc) {
            const int st = lc & 1;
            const uint8_t *sb = sm + st * CarrySmem::kStage;
            float g[32];
            tc::mbar_wait(&full[st], (lc >> 1) & 1, abort, p.err, kErrFull, p.spin);
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                const float4 x = *reinterpret_cast<const float4 *>(sb + CarrySmem::kG + (kc0 + j) * 4);
                g[j] = x.x; g[j + 1] = x.y; g[j + 2] = x.z; g[j + 3] = x.w;
            }
            // this warp has read its piece of the stage (gamma); the MMA
            // warp's commit covers the operands
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&empty[st]);
            tc::mbar_wait(d_done, lc & 1, abort, p.err, kErrD, p.spin);
            tc::tc_fence_after_sync();
            {
                float ku[32];
                tc::tmem_ld16x2_x32_x16_sync(lane_base + (uint32_t)st * 256 + 64 * wh, ku,
                                             lane_base + (uint32_t)st * 256 + 128 + 32 * wh, ov);
#pragma unroll
                for (int j = 0; j < 32; ++j) S[j] = g[j] * S[j] + ku[j];
            }
            if (lc + 1 < nc) {
                store_st((lc + 1) & 1);
                tc::fence_proxy_async_smem();
                tc::tc_fence_before_sync();
                named_bar(1, kCarrySync);  // S^T of chunk lc+1 complete
            }
            if (outputs) store_o(lc);
        }
        if (S_out) {
#pragma unroll
            for (int j = 0; j < 32; ++j) S_out[sbase + (size_t)j * D] = S[j];
        }
    }
    tc::tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------- combine
// Between the two passes of a time split: the true end state of every segment
// but the last, S_end(p) = Phi_p S_end(p - 1) + S0_p for p = 1 .. P - 2, in
// fp32 (Phi_p: segment p's transition, S0_p: its state from a zero start).
// One CTA per (sequence, head, 16 value columns); sequential over p.
constexpr int kCombThreads = 256;
constexpr int kCombCols = 16;

__global__ void __launch_bounds__(kCombThreads) tc_combine_kernel(TcParams p)
{
    __shared__ float sS[D][kCombCols];
    const int H = p.H, tiles = D / kCombCols;
    const int tile = blockIdx.x % tiles, u = blockIdx.x / tiles;
    const int h = u % H, n = u / H;
    const int tid = threadIdx.x, i = tid >> 1, c8 = (tid & 1) * 8, col = tile * kCombCols + c8;
    auto block = [&](int kind, int sp) {
        return p.seg + ((((size_t)kind * p.nseg + sp) * p.N + n) * H + h) * (size_t)D * D;
    };
    {
        const float *s0 = block(2, 0) + (size_t)i * D + col;
#pragma unroll
        for (int e = 0; e < 8; ++e) sS[i][c8 + e] = s0[e];
    }
    __syncthreads();
    for (int sp = 1; sp + 1 < p.nseg; ++sp) {
        const float *phi = block(1, sp) + (size_t)i * D;
        const float *z = block(0, sp) + (size_t)i * D + col;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = z[e];
        for (int m = 0; m < D; m += 4) {
            const float4 f = *reinterpret_cast<const float4 *>(phi + m);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                acc[e] += f.x * sS[m][c8 + e] + f.y * sS[m + 1][c8 + e] + f.z * sS[m + 2][c8 + e] +
                          f.w * sS[m + 3][c8 + e];
        }
        __syncthreads();
        float *out = block(2, sp) + (size_t)i * D + col;
#pragma unroll
        for (int e = 0; e < 8; ++e) { sS[i][c8 + e] = acc[e]; out[e] = acc[e]; }
        __syncthreads();
    }
}

constexpr size_t kPrepSmem = sizeof(float) * (4 * C * DP + C * D + 2 * C * (C + 1) + C);
static_assert(kPrepSmem <= 227 * 1024, "fixup shared memory");
constexpr int kFixupBlocks = 148;

}  // namespace

// cuTensorMapEncodeTiled, looked up once through the runtime (no link to the
// driver library).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// [tokens, H, 128] (bf16 or fp32) as a {128, H, tokens} tensor with boxes of
// 128 bytes of channels x 1 head x 64 tokens in the 128-byte swizzle;
// out-of-range tokens read zero.
bool encode_token_map(CUtensorMap *tm, const void *base, bool fp32, int H, long long tokens)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t es = fp32 ? 4 : 2;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)tokens};
    cuuint64_t strides[2] = {(cuuint64_t)D * es, (cuuint64_t)H * D * es};
    cuuint32_t box[3] = {(cuuint32_t)(128 / es), 1, (cuuint32_t)C};
    cuuint32_t estride[3] = {1, 1, 1};
    return enc(tm, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
               const_cast<void *>(base), dims, strides, box, estride,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

bool tc_supported(const Problem &p)
{
    return p.dtype == KDA_DTYPE_BF16 && p.dk == 128 && p.dv == 128;
}

int tc_auto_segments(const Problem &p)
{
    // Split the sequential phase in time only when few (sequence, head) chains
    // leave most SMs idle: the first pass needs 2 + 4 (P - 1) one-SM CTAs per
    // chain and the two passes together take about 2/P of the unsplit time, so
    // P >= 3 within one wave of 148 SMs, and segments of at least 16 chunks.
    const long long chains = (long long)p.N * p.H;
    if (chains <= 0 || p.max_chunks <= 0) return 1;
    const long long per_seq = (long long)p.max_chunks / p.N;
    long long P = (148 / chains - 2) / 4 + 1;
    P = P < per_seq / 16 ? P : per_seq / 16;
    if (P > kMaxSegments) P = kMaxSegments;
    return P >= 3 ? (int)P : 1;
}

WorkspaceLayout tc_workspace_layout(const Problem &p)
{
    WorkspaceLayout l;
    // header (status word, fixup count), plan arrays and the fixup list
    l.plan_bytes = align_up(kWsHeader + sizeof(int32_t) * (plan_ints(p.N) +
                                                           (size_t)p.max_chunks * p.H), 1024);
    l.chunk_bytes = (size_t)Record::kBytes * (size_t)p.H * (size_t)p.max_chunks;
    if (p.nseg > 1)  // the time split's segment states
        l.chunk_bytes += 3 * (size_t)p.nseg * p.N * p.H * D * D * sizeof(float);
    l.total = l.plan_bytes + l.chunk_bytes;
    return l;
}

cudaError_t launch_tc_prefill(const Problem &pb, void *workspace, int phases, cudaStream_t st)
{
    const WorkspaceLayout lay = tc_workspace_layout(pb);
    TcParams p;
    p.q = static_cast<const __nv_bfloat16 *>(pb.q);
    p.k = static_cast<const __nv_bfloat16 *>(pb.k);
    p.v = static_cast<const __nv_bfloat16 *>(pb.v);
    p.log_alpha = pb.log_alpha; p.beta = pb.beta; p.S0 = pb.S0;
    p.N = pb.N; p.H = pb.H; p.scale = pb.scale;
    p.o = static_cast<__nv_bfloat16 *>(pb.o); p.S_final = pb.S_final;
    Plan plan;
    p.err = static_cast<int32_t *>(workspace);
    p.fix_count = p.err + 1;
    plan.seq_start = reinterpret_cast<int32_t *>(static_cast<char *>(workspace) + kWsHeader);
    plan.chunk_off = plan.seq_start + (pb.N + 1);
    plan.order = plan.chunk_off + (pb.N + 1);
    p.seq_start = plan.seq_start; p.chunk_off = plan.chunk_off; p.order = plan.order;
    p.fix_list = plan.order + pb.N;
    p.rec = static_cast<uint8_t *>(workspace) + lay.plan_bytes;
    const DebugKnobs dbg = debug_knobs();
    p.spin = dbg.wait_limit ? dbg.wait_limit : tc::kSpinLimit;
    p.starve = dbg.starve_carry;
    p.nseg = pb.nseg > 1 ? pb.nseg : 1;
    p.pass = 0;
    p.T_uniform = pb.cu_seqlens ? 0 : pb.T;
    p.seg = reinterpret_cast<float *>(p.rec + (size_t)Record::kBytes * pb.H * pb.max_chunks);

    cudaError_t e = cudaSuccess;
    if (phases & kPhasePrepare) {
        e = launch_plan(pb, plan, st);
        if (e != cudaSuccess) return e;
        e = cudaMemsetAsync(p.err, 0, 2 * sizeof(int), st);
        if (e != cudaSuccess) return e;
        if (pb.max_chunks > 0 &&
            (!encode_token_map(&p.tm_q, pb.q, false, pb.H, pb.total_tokens) ||
             !encode_token_map(&p.tm_k, pb.k, false, pb.H, pb.total_tokens) ||
             !encode_token_map(&p.tm_v, pb.v, false, pb.H, pb.total_tokens) ||
             (pb.gate_per_channel &&
              !encode_token_map(&p.tm_la, pb.log_alpha, true, pb.H, pb.total_tokens))))
            return cudaErrorInvalidValue;
        if (pb.max_chunks > 0 && !pb.gate_per_channel) {
            e = cudaFuncSetAttribute(tc_gdn_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)GdnSmem::kBytes);
            if (e != cudaSuccess) return e;
            tc_gdn_prep_kernel<<<dim3(pb.max_chunks, pb.H), kGdnThreads, GdnSmem::kBytes, st>>>(p);
            note_launch();
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        } else if (pb.max_chunks > 0) {
            e = cudaFuncSetAttribute(tc_prep2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)Prep2Smem::kBytes);
            if (e != cudaSuccess) return e;
            tc_prep2_kernel<<<dim3(pb.max_chunks, pb.H), kPrep2Threads, Prep2Smem::kBytes, st>>>(p);
            note_launch();
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
            e = cudaFuncSetAttribute(tc_prep_fixup_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPrepSmem);
            if (e != cudaSuccess) return e;
            tc_prep_fixup_kernel<<<kFixupBlocks, kPrepThreads, kPrepSmem, st>>>(p);
            note_launch();
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
    }
    if (phases & kPhaseCarry) {
        e = cudaFuncSetAttribute(tc_carry_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)CarrySmem::kBytes);
        if (e != cudaSuccess) return e;
        const unsigned chains = (unsigned)(pb.N * pb.H);
        if (p.nseg == 1) {
            tc_carry_kernel<<<chains * kSlices, kCarryThreads, CarrySmem::kBytes, st>>>(p);
            note_launch();
            e = cudaGetLastError();
        } else {
            p.pass = 1;
            tc_carry_kernel<<<chains * (2 + 4 * (p.nseg - 1)), kCarryThreads, CarrySmem::kBytes,
                              st>>>(p);
            note_launch();
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
            if (p.nseg > 2) {
                tc_combine_kernel<<<chains * (D / kCombCols), kCombThreads, 0, st>>>(p);
                note_launch();
                e = cudaGetLastError();
                if (e != cudaSuccess) return e;
            }
            p.pass = 2;
            tc_carry_kernel<<<chains * 2 * (p.nseg - 1), kCarryThreads, CarrySmem::kBytes, st>>>(p);
            note_launch();
            e = cudaGetLastError();
        }
    }
    return e;
}

}  // namespace kda
