// kda_noalloc.cu — kda_chunk_fwd for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: a plugin whose host application owns all
// device memory and hands out none, or code running where an allocation's
// implicit device synchronisation is not allowed. kda_chunk_fwd_noalloc serves
// them: it runs the same prefill as kda_chunk_fwd_ex, but its workspace is a
// fixed array in the library's own device memory instead of a caller buffer.
//
// The array is a file-scope __device__ variable of KDA_NOALLOC_SCRATCH_BYTES.
// Every GPU that loads the library holds it until the process exits. Host code
// cannot pass the variable's name to a kernel (on the host the name is only a
// stand-in, not a device address), so the first call on each device looks up
// the device address with cudaGetSymbolAddress, with that device current, and
// caches it together with the device's current context; a later call on that
// device reuses the address while the context is the same and looks it up
// again after the context changed (for example after cudaDeviceReset, which
// reloads the module and may move the array).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "kda_internal.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices];     // device address of g_noalloc_scratch, per device
CUcontext g_scratch_ctx[kMaxDevices];  // the context that address belongs to

// cuCtxGetCurrent through the runtime's driver entry point (no link to libcuda).
PFN_cuCtxGetCurrent_v4000 ctx_getter()
{
    static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    });
    return fn;
}

// Device address of the scratch array on the current device (looked up once
// per device and context).
cudaError_t scratch_on_current_device(void **out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    PFN_cuCtxGetCurrent_v4000 get_ctx = ctx_getter();
    if (!get_ctx) return cudaErrorInvalidDevice;
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS) return cudaErrorInvalidDevice;
    if (ctx == nullptr) {
        // no context yet on this thread: selecting the device initialises its
        // primary context and makes it current
        e = cudaSetDevice(dev);
        if (e != cudaSuccess) return e;
        if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorInvalidDevice;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_ptr[dev] == nullptr || g_scratch_ctx[dev] != ctx) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
        g_scratch_ctx[dev] = ctx;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" kda_status_t kda_chunk_fwd_noalloc(
    const void *q, const void *k, const void *v, kda_dtype_t dt, const float *log_alpha,
    const float *beta, const float *S0, const int32_t *cu_seqlens, int n_seqs, int B, int T,
    int H, int dk, int dv, float scale, void *o, float *S_final, int algo, void *stream)
{
    // The size limit is checked on the host before any CUDA call.
    const size_t need = kda_chunk_fwd_workspace_size_ex(B, T, H, dk, dv,
                                                        cu_seqlens ? n_seqs : 0, dt, algo);
    if (need == 0)  // invalid sizes, dtype or algo: rejected on the host, nothing launched
        return kda_chunk_fwd_ex(q, k, v, dt, log_alpha, beta, S0, cu_seqlens, n_seqs, B, T, H,
                                dk, dv, scale, o, S_final, nullptr, 0, algo, stream);
    if (need > (size_t)KDA_NOALLOC_SCRATCH_BYTES) return KDA_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (scratch_on_current_device(&scratch) != cudaSuccess) return KDA_ERR_CUDA;
    return kda_chunk_fwd_ex(q, k, v, dt, log_alpha, beta, S0, cu_seqlens, n_seqs, B, T, H,
                            dk, dv, scale, o, S_final, scratch, KDA_NOALLOC_SCRATCH_BYTES, algo,
                            stream);
}
