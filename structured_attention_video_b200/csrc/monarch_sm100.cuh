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

// The backward pass on the tensor cores: bfloat16, d = 128, [B][H][N][d],
// self-attention, query-row tiles, one iteration.
bool sm100_backward_supports(const Problem &p, monarch_dtype dtype);
// Its workspace: the forward's tensor-core intermediates, the row statistics and
// the intermediate gradients.
size_t sm100_backward_workspace_bytes(const Problem &p, bool &overflow);
// The forward's q̄, R-step (R in two bfloat16 parts) and L-step row statistics on
// the tensor cores; then the L-step side (delta as sum L dP, dKtil, dZ, dH, the
// L-step's part of dq) and the R-step side (dk, dv, the partial sums of dq̄), and
// dq = dq_L + dq̄ / |T_g|.  dq, dk, dv: bfloat16 [B][H][N][d].
cudaError_t sm100_backward(const Problem &p, const void *q, const void *k, const void *v,
                           const void *dy, void *dq, void *dk, void *dv, void *workspace,
                           int *status, long long wait_limit, cudaStream_t stream);

}  // namespace monarch
