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
//    order. Warp 4 streams each record into a two-stage shared-memory ring
//    with bulk async copies; warp 5 issues the tcgen05 MMAs; warps 0-3 own the
//    128 rows of the state slice (fp32, in registers), read the accumulators
//    out of TMEM and write the bf16 operands the next MMA needs:
//        MMA1: D1 = [W; Q~] (128x128) . S (128x64)        -> WS rows, Q~S rows
//        U    = U~ - WS                                    (warps 0-1)
//        MMA2: D2 = K^^T (128x64) . U (64x64)              -> state increment
//              D1 += [0; P] (128x64) . U                   -> Q~S + PU
//        S    = gamma * S + D2 (warps 0-3); o = scale * D1 rows 64..127 (warps 2-3)
//    The state never leaves the SM between chunks; S_final is written once.
#include "kda_internal.cuh"
#include "tc_primitives.cuh"

namespace kda {
namespace {

constexpr int C = kChunk;   // 64 tokens per chunk
constexpr int D = 128;      // dk = dv
constexpr int kSlice = 64;  // value columns per carry CTA
constexpr int kSlices = D / kSlice;

// Workspace record per (chunk, head), bytes. Every piece is a verbatim image of
// a shared-memory operand so the carry kernel can bulk-copy it.
struct Record {
    static constexpr uint32_t kA1 = 0;        // [W; Q~] 128x128 bf16, K-major, SW128, 2 K-blocks
    static constexpr uint32_t kKh = 32768;    // K^^T 128x64 bf16, MN-major, SW128, 2 MN-blocks
    static constexpr uint32_t kP = 49152;     // P 64x64 bf16, K-major, SW128
    static constexpr uint32_t kG = 57344;     // gamma fp32 [128]
    static constexpr uint32_t kU = 57856;     // U~ fp32 [2 halves][64 rows][64 cols], 16B-chunk swizzled
    static constexpr uint32_t kBytes = 90624;
};
static_assert(Record::kU + kSlices * C * kSlice * 4 == Record::kBytes, "record size");

// Shared-memory layout of the carry kernel (offsets from a 1024-aligned base).
struct CarrySmem {
    static constexpr uint32_t kA1 = 0;         // 32768
    static constexpr uint32_t kKh = 32768;     // 16384
    static constexpr uint32_t kA2b = 49152;    // 16384: rows 0..63 zero, rows 64..127 = P
    static constexpr uint32_t kU = 65536;      // 16384
    static constexpr uint32_t kG = 81920;      // 512
    static constexpr uint32_t kStage = 83968;  // stage stride (1024-aligned)
    static constexpr uint32_t kB1 = 2 * kStage;        // S (bf16, 128x64, MN-major)
    static constexpr uint32_t kB2 = kB1 + 16384;       // U (bf16, 64x64, MN-major)
    static constexpr uint32_t kBar = kB2 + 8192;       // mbarriers
    static constexpr uint32_t kBytes = kBar + 256 + 1024;  // + alignment slack
};

__device__ __forceinline__ uint32_t u_swz(uint32_t r, uint32_t jj)
{
    // byte offset of U~[r][jj] inside one 64x64 fp32 half: 16-byte chunks XORed by row
    return r * 256u + ((((jj >> 2) ^ (r & 15u)) << 4) | ((jj & 3u) << 2));
}

struct TcParams {
    const __nv_bfloat16 *q, *k, *v;
    const float *log_alpha, *beta, *S0;
    int N, H;
    float scale;
    __nv_bfloat16 *o;
    float *S_final;
    const int32_t *seq_start, *chunk_off;
    uint8_t *rec;  // records
    int *err;      // device error word
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

// ------------------------------------------------------------------- prep (v1)
// fp32 CUDA-core prep: exact per-term gate exponents for A and P, forward
// substitution for W and U~, then the record image.
constexpr int kPrepThreads = 256;

__global__ void __launch_bounds__(kPrepThreads, 1) tc_prep_kernel(TcParams p)
{
    constexpr int DP = D + 1;
    extern __shared__ float smem[];
    float *sk = smem;               // [C][DP]
    float *sq = sk + C * DP;        // [C][DP]
    float *sg = sq + C * DP;        // [C][DP]
    float *sv = sg + C * DP;        // [C][D]
    float *sA = sv + C * D;         // [C][C+1]
    float *sb = sA + C * (C + 1);   // [C]

    const int c = blockIdx.x, h = blockIdx.y, H = p.H;
    const int n = find_seq(p.chunk_off, p.N, c);
    if (n < 0) return;
    const int t0 = p.seq_start[n] + (c - p.chunk_off[n]) * C;
    const int L = min(C, p.seq_start[n + 1] - t0);
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
    __nv_bfloat16 *a1 = reinterpret_cast<__nv_bfloat16 *>(rec + Record::kA1);
    __nv_bfloat16 *kh = reinterpret_cast<__nv_bfloat16 *>(rec + Record::kKh);
    __nv_bfloat16 *pp = reinterpret_cast<__nv_bfloat16 *>(rec + Record::kP);
    float *gg = reinterpret_cast<float *>(rec + Record::kG);
    uint8_t *uu = rec + Record::kU;

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
            pp[tc::sw128(r, 2 * s) / 2] = __float2bfloat16_rn(pqk);
        }
    }
    // Q~ (rows 64..127 of A1), K^ (MN-major image) and gamma.
    for (int idx = tid; idx < C * D; idx += kPrepThreads) {
        const int r = idx / D, i = idx % D;
        const float g = sg[r * DP + i], gC = sg[(C - 1) * DP + i];
        const uint32_t kb = (uint32_t)(i >> 6) * 16384u;
        a1[(kb + tc::sw128(64 + r, 2 * (i & 63))) / 2] = __float2bfloat16_rn(expf(g) * sq[r * DP + i]);
        kh[((uint32_t)(i >> 6) * 8192u + tc::sw128(r, 2 * (i & 63))) / 2] =
            __float2bfloat16_rn(expf(gC - g) * sk[r * DP + i]);
    }
    for (int i = tid; i < D; i += kPrepThreads) gg[i] = expf(sg[(C - 1) * DP + i]);
    __syncthreads();
    for (int idx = tid; idx < C * D; idx += kPrepThreads) {
        const int r = idx / D, i = idx % D;
        sk[r * DP + i] *= sb[r] * expf(sg[r * DP + i]);
        sv[r * D + i] *= sb[r];
    }
    __syncthreads();
    for (int col = tid; col < 2 * D; col += kPrepThreads) {
        float *x = col < D ? sk + col : sv + (col - D);
        const int stride = col < D ? DP : D;
        for (int r = 1; r < C; ++r) {
            float acc = x[r * stride];
            for (int s = 0; s < r; ++s) acc -= sA[r * (C + 1) + s] * x[s * stride];
            x[r * stride] = acc;
        }
    }
    __syncthreads();
    for (int idx = tid; idx < C * D; idx += kPrepThreads) {
        const int r = idx / D, i = idx % D;
        const uint32_t kb = (uint32_t)(i >> 6) * 16384u;
        a1[(kb + tc::sw128(r, 2 * (i & 63))) / 2] = __float2bfloat16_rn(sk[r * DP + i]);
        const int half = i >> 6, jj = i & 63;
        *reinterpret_cast<float *>(uu + half * 16384 + u_swz(r, jj)) = sv[r * D + i];
    }
}

// ------------------------------------------------------------------- carry
constexpr int kCarryThreads = 192;  // warps 0-3 epilogue, 4 producer, 5 MMA
constexpr uint32_t kTmemCols = 128; // D1: columns [0,64), D2: [64,128)

enum { kErrFull = 1, kErrEmpty, kErrD1, kErrU, kErrD2, kErrS };

__global__ void __launch_bounds__(kCarryThreads, 1) tc_carry_kernel(TcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + CarrySmem::kBar);
    uint64_t *full = bars + 0;   // [2]
    uint64_t *empty = bars + 2;  // [2]
    uint64_t *d1_done = bars + 4;
    uint64_t *u_ready = bars + 5;
    uint64_t *d2_done = bars + 6;
    uint64_t *s_ready = bars + 7;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 8);
    volatile int *abort = reinterpret_cast<volatile int *>(bars + 9);

    const int n = blockIdx.x, h = blockIdx.y, half = blockIdx.z, H = p.H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        tc::mbar_init(&full[0], 1); tc::mbar_init(&full[1], 1);
        tc::mbar_init(&empty[0], 4); tc::mbar_init(&empty[1], 4);
        tc::mbar_init(d1_done, 1); tc::mbar_init(u_ready, 2);
        tc::mbar_init(d2_done, 1); tc::mbar_init(s_ready, 4);
        *abort = 0;
        tc::fence_mbar_init();
    }
    // rows 0..63 of the [0; P] operand stay zero
    for (int s = 0; s < 2; ++s) {
        uint4 *z = reinterpret_cast<uint4 *>(sm + s * CarrySmem::kStage + CarrySmem::kA2b);
        for (int i = threadIdx.x; i < 8192 / 16; i += kCarryThreads) z[i] = make_uint4(0, 0, 0, 0);
    }
    if (warp == 5) { tc::tmem_alloc(tmem_slot, kTmemCols); tc::tmem_relinquish(); }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before_sync();
    __syncthreads();
    tc::tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    const int ts = p.seq_start[n], te = p.seq_start[n + 1];
    const int c0 = p.chunk_off[n], nc = p.chunk_off[n + 1] - c0;

    if (warp == 4) {
        // ---------------- producer: one record per chunk into the two-stage ring
        if (lane == 0) {
            for (int lc = 0; lc < nc; ++lc) {
                const int st = lc & 1;
                if (lc >= 2) tc::mbar_wait(&empty[st], ((lc >> 1) - 1) & 1, abort, p.err, kErrEmpty);
                const uint8_t *rec = p.rec + ((size_t)(c0 + lc) * H + h) * Record::kBytes;
                uint8_t *sb = sm + st * CarrySmem::kStage;
                tc::mbar_arrive_expect_tx(&full[st], 32768 + 16384 + 8192 + 512 + 16384);
                tc::bulk_g2s(sb + CarrySmem::kA1, rec + Record::kA1, 32768, &full[st]);
                tc::bulk_g2s(sb + CarrySmem::kKh, rec + Record::kKh, 16384, &full[st]);
                tc::bulk_g2s(sb + CarrySmem::kA2b + 8192, rec + Record::kP, 8192, &full[st]);
                tc::bulk_g2s(sb + CarrySmem::kG, rec + Record::kG, 512, &full[st]);
                tc::bulk_g2s(sb + CarrySmem::kU, rec + Record::kU + half * 16384, 16384, &full[st]);
            }
            // every issued copy has landed before the CTA may exit
            for (int lc = (nc > 2 ? nc - 2 : 0); lc < nc; ++lc)
                tc::mbar_wait(&full[lc & 1], (lc >> 1) & 1, abort, p.err, kErrFull);
        }
    } else if (warp == 5) {
        // ---------------- MMA issuer
        if (lane == 0) {
            const uint32_t id1 = tc::idesc_bf16(128, 64, 0, 1);   // [W;Q~] K-major . S MN-major
            const uint32_t id2a = tc::idesc_bf16(128, 64, 1, 1);  // K^^T MN-major . U MN-major
            const uint32_t id2b = tc::idesc_bf16(128, 64, 0, 1);  // [0;P] K-major . U MN-major
            const uint32_t b1 = tc::smem_u32(sm + CarrySmem::kB1);
            const uint32_t b2 = tc::smem_u32(sm + CarrySmem::kB2);
            for (int lc = 0; lc < nc; ++lc) {
                const int st = lc & 1;
                const uint32_t sb = tc::smem_u32(sm + st * CarrySmem::kStage);
                tc::mbar_wait(&full[st], (lc >> 1) & 1, abort, p.err, kErrFull);
                tc::mbar_wait(s_ready, lc & 1, abort, p.err, kErrS);
                tc::tc_fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t a = tc::smem_desc(sb + CarrySmem::kA1 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                    const uint64_t b = tc::smem_desc(b1 + kk * 2048, 8192, 1024);
                    tc::mma_bf16(tmem + 0, a, b, id1, kk > 0);
                }
                tc::mma_commit(d1_done);
                tc::mbar_wait(u_ready, lc & 1, abort, p.err, kErrU);
                tc::tc_fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t a = tc::smem_desc(sb + CarrySmem::kKh + kk * 2048, 8192, 1024);
                    const uint64_t b = tc::smem_desc(b2 + kk * 2048, 8192, 1024);
                    tc::mma_bf16(tmem + 64, a, b, id2a, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t a = tc::smem_desc(sb + CarrySmem::kA2b + kk * 32, 16, 1024);
                    const uint64_t b = tc::smem_desc(b2 + kk * 2048, 8192, 1024);
                    tc::mma_bf16(tmem + 0, a, b, id2b, 1);
                }
                tc::mma_commit(d2_done);
            }
        }
    } else {
        // ---------------- epilogue: thread t owns row t of the state slice
        const int t = threadIdx.x;  // 0..127
        const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
        float S[kSlice];
        const size_t sbase = (((size_t)n * H + h) * D + t) * D + half * kSlice;
#pragma unroll
        for (int j = 0; j < kSlice; j += 4) {
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (p.S0) x = *reinterpret_cast<const float4 *>(p.S0 + sbase + j);
            S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
        }
        uint8_t *b1row = sm + CarrySmem::kB1;
        auto store_row_bf16 = [&](uint8_t *base, int row, const float *vals) {
#pragma unroll
            for (int c16 = 0; c16 < 8; ++c16) {
                __nv_bfloat162 w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    w[e] = __floats2bfloat162_rn(vals[c16 * 8 + 2 * e], vals[c16 * 8 + 2 * e + 1]);
                *reinterpret_cast<uint4 *>(base + tc::sw128(row, c16 * 16)) =
                    *reinterpret_cast<uint4 *>(w);
            }
        };
        store_row_bf16(b1row, t, S);
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(s_ready);

        for (int lc = 0; lc < nc; ++lc) {
            const int st = lc & 1;
            uint8_t *sb = sm + st * CarrySmem::kStage;
            const int t0 = ts + lc * C;
            const int L = min(C, te - t0);
            tc::mbar_wait(&full[st], (lc >> 1) & 1, abort, p.err, kErrFull);
            if (warp < 2) {
                tc::mbar_wait(d1_done, lc & 1, abort, p.err, kErrD1);
                tc::tc_fence_after_sync();
                float U[kSlice];
                tc::tmem_ld32_sync(lane_addr + 0, U);
                tc::tmem_ld32_sync(lane_addr + 32, U + 32);
#pragma unroll
                for (int j = 0; j < kSlice; j += 4) {
                    const float4 ut = *reinterpret_cast<const float4 *>(
                        sb + CarrySmem::kU + u_swz(t, j));
                    U[j] = ut.x - U[j];
                    U[j + 1] = ut.y - U[j + 1];
                    U[j + 2] = ut.z - U[j + 2];
                    U[j + 3] = ut.w - U[j + 3];
                }
                store_row_bf16(sm + CarrySmem::kB2, t, U);
                tc::fence_proxy_async_smem();
                tc::tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(u_ready);
            }
            tc::mbar_wait(d2_done, lc & 1, abort, p.err, kErrD2);
            tc::tc_fence_after_sync();
            const float gamma = reinterpret_cast<const float *>(sb + CarrySmem::kG)[t];
            {
                float ku[kSlice];
                tc::tmem_ld32_sync(lane_addr + 64, ku);
                tc::tmem_ld32_sync(lane_addr + 96, ku + 32);
#pragma unroll
                for (int j = 0; j < kSlice; ++j) S[j] = gamma * S[j] + ku[j];
            }
            store_row_bf16(b1row, t, S);
            if (warp >= 2) {
                const int r = t - 64;
                __nv_bfloat16 *orow = p.o + ((size_t)(t0 + r) * H + h) * D + half * kSlice;
                float ov[kSlice];
                tc::tmem_ld32_sync(lane_addr + 0, ov);
                tc::tmem_ld32_sync(lane_addr + 32, ov + 32);
                if (r < L) {
#pragma unroll
                    for (int j = 0; j < kSlice; j += 8) {
                        __nv_bfloat162 w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            w[e] = __floats2bfloat162_rn(p.scale * ov[j + 2 * e],
                                                         p.scale * ov[j + 2 * e + 1]);
                        *reinterpret_cast<uint4 *>(orow + j) = *reinterpret_cast<uint4 *>(w);
                    }
                }
            }
            tc::fence_proxy_async_smem();
            tc::tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) { tc::mbar_arrive(s_ready); tc::mbar_arrive(&empty[st]); }
        }
        if (p.S_final) {
#pragma unroll
            for (int j = 0; j < kSlice; j += 4)
                *reinterpret_cast<float4 *>(p.S_final + sbase + j) =
                    make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    }
    tc::tc_fence_before_sync();
    __syncthreads();
    if (warp == 5) {
        tc::tc_fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

constexpr size_t kPrepSmem = sizeof(float) * (3 * C * (D + 1) + C * D + C * (C + 1) + C);

}  // namespace

bool tc_supported(const Problem &p)
{
    return p.dtype == KDA_DTYPE_BF16 && p.dk == 128 && p.dv == 128;
}

WorkspaceLayout tc_workspace_layout(const Problem &p)
{
    WorkspaceLayout l;
    // plan arrays + the device error word
    l.plan_bytes = align_up(sizeof(int32_t) * (2 * (size_t)(p.N + 1) + 1), 1024);
    l.chunk_bytes = (size_t)Record::kBytes * (size_t)p.H * (size_t)p.max_chunks;
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
    plan.seq_start = static_cast<int32_t *>(workspace);
    plan.chunk_off = plan.seq_start + (pb.N + 1);
    p.seq_start = plan.seq_start; p.chunk_off = plan.chunk_off;
    p.err = plan.chunk_off + (pb.N + 1);
    p.rec = static_cast<uint8_t *>(workspace) + lay.plan_bytes;

    cudaError_t e = cudaSuccess;
    if (phases & kPhasePrepare) {
        e = launch_plan(pb, plan, st);
        if (e != cudaSuccess) return e;
        e = cudaMemsetAsync(p.err, 0, sizeof(int), st);
        if (e != cudaSuccess) return e;
        if (pb.max_chunks > 0) {
            e = cudaFuncSetAttribute(tc_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kPrepSmem);
            if (e != cudaSuccess) return e;
            tc_prep_kernel<<<dim3(pb.max_chunks, pb.H), kPrepThreads, kPrepSmem, st>>>(p);
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
    }
    if (phases & kPhaseCarry) {
        e = cudaFuncSetAttribute(tc_carry_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)CarrySmem::kBytes);
        if (e != cudaSuccess) return e;
        tc_carry_kernel<<<dim3(pb.N, pb.H, kSlices), kCarryThreads, CarrySmem::kBytes, st>>>(p);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace kda
