// monarch_noalloc.cu -- monarch_attn_fwd_noalloc: the forward pass for callers
// that may not allocate device memory.  Its scratch space is the file-scope
// static device array below; nothing here allocates.
#include "monarch_common.cuh"

namespace monarch {
namespace {

// Scratch of the no-allocation entry point: MONARCH_NOALLOC_SCRATCH_BYTES on
// every device that loads this module, kept until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MONARCH_NOALLOC_SCRATCH_BYTES];

SymbolAddressCache g_scratch_cache;

// In host code g_noalloc_scratch names a host-side stand-in, not device
// memory: the kernels must receive the device address, looked up once per
// CUDA context (with that context current) and cached under its id.
cudaError_t scratch_on_current_device(void **out) {
    return g_scratch_cache.lookup(g_noalloc_scratch, out);
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace
}  // namespace monarch

using namespace monarch;

extern "C" monarch_status monarch_attn_fwd_noalloc(const void *q, const void *k, const void *v,
                                                   void *out, int B, int H, int f, int h, int w,
                                                   int d, int b1, int b2, int tiles, int iters,
                                                   monarch_dtype dtype, monarch_stream_t stream) {
    if (!q || !k || !v || !out) return MONARCH_ERR_INVALID_ARG;
    Problem p;
    monarch_status st = validate_shape(B, H, f, h, w, d, b1, b2, tiles, iters, dtype, &p);
    if (st != MONARCH_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return MONARCH_ERR_ALIGN;
    bool overflow = false;
    const size_t need = generic_workspace_bytes(p, overflow);
    if (overflow || need > MONARCH_NOALLOC_SCRATCH_BYTES) return MONARCH_ERR_SCRATCH_LIMIT;
    void *scratch = nullptr;
    if (scratch_on_current_device(&scratch) != cudaSuccess) return MONARCH_ERR_CUDA;
    // every scratch region is written before it is read: no clearing needed
    const cudaError_t e = generic_forward(p, dtype, q, k, v, out,
                                          generic_workspace_carve(p, scratch),
                                          (cudaStream_t)stream);
    return e == cudaSuccess ? MONARCH_OK : MONARCH_ERR_CUDA;
}
