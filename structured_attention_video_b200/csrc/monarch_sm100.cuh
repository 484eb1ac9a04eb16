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

// The backward of the L-step and the output on the tensor cores: bfloat16,
// d = 128, [B][H][N][d], self-attention, query-row tiles, one iteration.
bool sm100_backward_supports(const Problem &p, monarch_dtype dtype);
// Its workspace: the forward's tensor-core intermediates and the row statistics.
size_t sm100_backward_workspace_bytes(const Problem &p, bool &overflow);
// Runs the forward's q̄, R-step (R in two bfloat16 parts) and the L-step's row
// statistics on the tensor cores, then delta = dy.y (as sum L dP), the gradients
// dKtil, dZ, dH (float32, [BH][t][b2][b1] rows) and the L-step's part of dq
// (float32 [BH][N][d]).
cudaError_t sm100_backward_lstep(const Problem &p, const void *q, const void *k, const void *v,
                                 const void *dy, void *workspace, float *delta, float *dkt,
                                 float *dz, float *dh, float *dql, int *status,
                                 long long wait_limit, cudaStream_t stream);

}  // namespace monarch
