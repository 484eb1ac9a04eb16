// monarch_sm100.cuh -- entry points of the sm_100a tensor-core kernel family.
#pragma once

#include "monarch_common.cuh"

namespace monarch {

// True when the tensor-core kernels handle this call.
bool sm100_supports(const Problem &p, monarch_dtype dtype);
// Workspace of the tensor-core path (overflow set if it does not fit in size_t).
size_t sm100_workspace_bytes(const Problem &p, bool &overflow);
// Enqueue the forward pass; `status` is the device status word for bounded
// waits, `stall` the fault-injection hook (see monarch_debug_inject_stall).
cudaError_t sm100_forward(const Problem &p, const void *q, const void *k, const void *v,
                          void *out, void *workspace, int *status, long long wait_limit,
                          int stall, cudaStream_t stream);

}  // namespace monarch
