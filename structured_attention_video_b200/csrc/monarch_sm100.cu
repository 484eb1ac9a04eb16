// monarch_sm100.cu -- sm_100a tensor-core kernels (tcgen05 / TMEM / TMA).
#include "monarch_sm100.cuh"

namespace monarch {

bool sm100_supports(const Problem &, monarch_dtype) { return false; }

size_t sm100_workspace_bytes(const Problem &, bool &overflow) {
    overflow = false;
    return 0;
}

cudaError_t sm100_forward(const Problem &, const void *, const void *, const void *, void *,
                          void *, int *, long long, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace monarch
