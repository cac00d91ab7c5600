// kda_tc.cu — tcgen05 tensor-core prefill (bf16, dk = dv = 128).
#include "kda_internal.cuh"

namespace kda {

bool tc_supported(const Problem &) { return false; }

WorkspaceLayout tc_workspace_layout(const Problem &p) { return simt_workspace_layout(p); }

cudaError_t launch_tc_prefill(const Problem &, void *, int, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace kda
