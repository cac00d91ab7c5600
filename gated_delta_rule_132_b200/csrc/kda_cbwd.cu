// kda_cbwd.cu — chunk-parallel backward of the prefill on CUDA cores (fp32).
//
// Launch sequence: the plan, then five kernels whose bodies are in
// kda_cbwd_body.cuh, where the derivation is written out: the per-chunk
// records (all chunks in parallel), the forward chunk walk that keeps each
// chunk's entry state and U, the reverse chunk walk that keeps each chunk's
// end gradient and dU (and returns dS0), and two chunk-parallel kernels for
// the token gradients. The walks are the only sequential part: one CTA per
// (sequence, head, 32 value columns), one step per 64-token chunk.
#include "kda_cbwd_body.cuh"
#include "kda_internal.cuh"

namespace kda {
namespace {

using namespace cbwd;

struct DevX {
    __device__ int tid() const { return threadIdx.x; }
    __device__ int block() const { return blockIdx.x; }
    __device__ int block_y() const { return blockIdx.y; }
    __device__ void sync() { __syncthreads(); }
    // 16-byte asynchronous copy global -> shared (both 16-byte aligned), in
    // this thread's current group
    __device__ void cp16(void *dst, const void *src)
    {
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                     ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src) : "memory");
    }
    __device__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
    // wait until at most `pending` of this thread's committed groups are in flight
    __device__ void cp_wait(int pending)
    {
        if (pending <= 0) asm volatile("cp.async.wait_group 0;" ::: "memory");
        else if (pending == 1) asm volatile("cp.async.wait_group 1;" ::: "memory");
        else asm volatile("cp.async.wait_group 2;" ::: "memory");
    }
};

template <int D, typename TIn>
__global__ void __launch_bounds__(NT, 1) cb_prep_kernel(CbParams p, float *rec)
{
    extern __shared__ float smem[];
    DevX x;
    prep<D, TIn>(p, x, smem, rec);
}

template <int D>
__global__ void __launch_bounds__(NT, 1) cb_fwd_carry_kernel(CbParams p)
{
    extern __shared__ float smem[];
    DevX x;
    fwd_carry<D>(p, x, smem);
}

template <int D, typename TIn>
__global__ void __launch_bounds__(NT, 1) cb_bwd_carry_kernel(CbParams p)
{
    extern __shared__ float smem[];
    DevX x;
    bwd_carry<D, TIn>(p, x, smem);
}

template <int D, typename TIn>
__global__ void __launch_bounds__(NT, 1) cb_grad_a_kernel(CbParams p)
{
    extern __shared__ float smem[];
    DevX x;
    grad_a<D, TIn>(p, x, smem);
}

template <int D, typename TIn>
__global__ void __launch_bounds__(NT, 1) cb_grad_b_kernel(CbParams p)
{
    extern __shared__ float smem[];
    DevX x;
    grad_b<D, TIn>(p, x, smem);
}

// Byte offsets of the workspace regions: header and plan, then per (chunk,
// head) the record, the entry state and chunk-end gradient, U and dU, and
// grad_a's products.
struct CbRegions {
    size_t rec, Sst, dSst, Ust, dUst, scr, total;
};

CbRegions cb_regions(const Problem &pb)
{
    const size_t D = (size_t)pb.dk, units = (size_t)pb.max_chunks * pb.H;
    CbRegions g;
    g.rec = kWsHeader + align_up(sizeof(int32_t) * plan_ints(pb.N), 256);
    g.Sst = g.rec + align_up(sizeof(float) * units * (4 * C * D + C * C + D), 256);
    g.dSst = g.Sst + align_up(sizeof(float) * units * D * D, 256);
    g.Ust = g.dSst + align_up(sizeof(float) * units * D * D, 256);
    g.dUst = g.Ust + align_up(sizeof(float) * units * C * D, 256);
    g.scr = g.dUst + align_up(sizeof(float) * units * C * D, 256);
    g.total = g.scr + align_up(sizeof(float) * units * (3 * C * D + C * C + D), 256);
    return g;
}

template <int D, typename TIn>
cudaError_t launch_cb_d(const CbParams &p, float *rec, int max_chunks, cudaStream_t st)
{
    auto k0 = cb_prep_kernel<D, TIn>;
    auto k1 = cb_fwd_carry_kernel<D>;
    auto k2 = cb_bwd_carry_kernel<D, TIn>;
    auto k3 = cb_grad_a_kernel<D, TIn>;
    auto k4 = cb_grad_b_kernel<D, TIn>;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k0, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)prep_smem<D>())) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fwd_carry_smem<D>())) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bwd_carry_smem<D>())) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)grad_a_smem<D>())) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(k4, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)grad_b_smem<D>())) != cudaSuccess) return e;
    const unsigned walks = (unsigned)p.N * p.H * (D / WV);
    if (max_chunks > 0) {
        k0<<<dim3(max_chunks, p.H), NT, prep_smem<D>(), st>>>(p, rec);
        note_launch();
    }
    if (walks > 0) {
        k1<<<walks, NT, fwd_carry_smem<D>(), st>>>(p);
        note_launch();
        k2<<<walks, NT, bwd_carry_smem<D>(), st>>>(p);
        note_launch();
    }
    if (max_chunks > 0) {
        k3<<<dim3(max_chunks, p.H), NT, grad_a_smem<D>(), st>>>(p);
        note_launch();
        k4<<<dim3(max_chunks, p.H), NT, grad_b_smem<D>(), st>>>(p);
        note_launch();
    }
    return cudaGetLastError();
}

}  // namespace

size_t cbwd_workspace_bytes(const Problem &pb) { return cb_regions(pb).total; }

cudaError_t launch_backward_chunked(const Problem &pb, const void *dO, const float *dS_final,
                                    float *gq, float *gk, float *gv, float *gla, float *gbeta,
                                    float *gS0, void *workspace, cudaStream_t st)
{
    const CbRegions g = cb_regions(pb);
    char *ws = static_cast<char *>(workspace);
    Plan plan;
    plan.seq_start = reinterpret_cast<int32_t *>(ws + kWsHeader);
    plan.chunk_off = plan.seq_start + (pb.N + 1);
    plan.order = plan.chunk_off + (pb.N + 1);
    cudaError_t e = launch_plan(pb, plan, st);
    if (e != cudaSuccess) return e;
    float *rec = reinterpret_cast<float *>(ws + g.rec);
    CbParams p;
    p.q = pb.q; p.k = pb.k; p.v = pb.v; p.dO = dO;
    p.log_alpha = pb.log_alpha; p.beta = pb.beta; p.S0 = pb.S0; p.dS_final = dS_final;
    p.N = pb.N; p.H = pb.H; p.gate_per_channel = pb.gate_per_channel; p.scale = pb.scale;
    p.seq_start = plan.seq_start;
    p.chunk_off = plan.chunk_off;
    p.order = plan.order;
    p.rec = rec;
    p.Sst = reinterpret_cast<float *>(ws + g.Sst);
    p.dSst = reinterpret_cast<float *>(ws + g.dSst);
    p.Ust = reinterpret_cast<float *>(ws + g.Ust);
    p.dUst = reinterpret_cast<float *>(ws + g.dUst);
    p.scr = reinterpret_cast<float *>(ws + g.scr);
    p.gq = gq; p.gk = gk; p.gv = gv; p.gla = gla; p.gbeta = gbeta; p.gS0 = gS0;
    const bool bf = pb.dtype == KDA_DTYPE_BF16;
    switch (pb.dk) {
    case 32: return bf ? launch_cb_d<32, __nv_bfloat16>(p, rec, pb.max_chunks, st)
                       : launch_cb_d<32, float>(p, rec, pb.max_chunks, st);
    case 64: return bf ? launch_cb_d<64, __nv_bfloat16>(p, rec, pb.max_chunks, st)
                       : launch_cb_d<64, float>(p, rec, pb.max_chunks, st);
    case 128: return bf ? launch_cb_d<128, __nv_bfloat16>(p, rec, pb.max_chunks, st)
                        : launch_cb_d<128, float>(p, rec, pb.max_chunks, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace kda
