// tc_selftest.cu -- test-only checks of the sm_100a building blocks used by the
// tensor-core kernels: TMA tile loads with the 128-byte swizzle, tcgen05.mma
// with both operands in shared memory (K-major) and with A in tensor memory and
// B MN-major, TMEM loads/stores, and the bounded mbarrier wait.
#include "../../structured_attention_video_b200/csrc/tc_primitives.cuh"

#include <cuda.h>

using namespace monarch;
using namespace monarch::tc;

namespace {

// D[128 x N] = A[128 x 128] B[N x 128]^T    (both K-major, SS)
// E[128 x 128] = bf16(D) B                  (A = bf16(D) from TMEM, B MN-major, TS)
template <int N>
__global__ void __launch_bounds__(128, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            float *dout, float *eout, int *status) {
    extern __shared__ uint8_t raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    constexpr uint32_t kA = 0, kB = 32768, kPanelB = N * 128, kBar = kB + 2 * kPanelB;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + kBar);
    uint32_t *slot = reinterpret_cast<uint32_t *>(bar + 4);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bar + 5);
    const int warp = threadIdx.x >> 5, r = threadIdx.x;
    if (threadIdx.x == 0) {
        for (int i = 0; i < 3; i++) mbar_init(bar + i, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    const WaitCtx w{1LL << 22, status, abort_flag};
    if (threadIdx.x == 0) {
        mbar_expect_tx(bar, 32768 + 2 * kPanelB);
        for (int pn = 0; pn < 2; pn++) {
            tma_load_2d(sm + kA + pn * 16384, &tmA, pn * 64, 0, bar);
            tma_load_2d(sm + kB + pn * kPanelB, &tmB, pn * 64, 0, bar);
        }
        if (wait_phase(bar, 0, w)) {
            tc_fence_after();
            for (int kk = 0; kk < 8; kk++) {
                const uint32_t ao = (kk >> 2) * 16384 + (kk & 3) * 32;
                const uint32_t bo = (kk >> 2) * kPanelB + (kk & 3) * 32;
                mma_ss(tmem, smem_desc_sw128(smem_u32(sm + kA) + ao, 16, 1024),
                       smem_desc_sw128(smem_u32(sm + kB) + bo, 16, 1024),
                       idesc_bf16(128, N, 0, 0), kk > 0);
            }
            mma_commit(bar + 1);
        }
    }
    __syncwarp();
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    bool ok = __all_sync(0xffffffffu, wait_phase(bar + 1, 0, w));
    if (ok) {
        tc_fence_after();
        for (int c = 0; c < N / 16; c++) {
            uint32_t v[16];
            tmem_ld16(tmem + lane_off + c * 16, v);
            tmem_wait_ld();
            uint32_t pk[8];
            for (int k = 0; k < 16; k++) dout[r * N + c * 16 + k] = __uint_as_float(v[k]);
            for (int k = 0; k < 8; k++)
                pk[k] = pack_bf16(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1]));
            tmem_st8(tmem + lane_off + 256 + c * 8, pk);
        }
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && ok) {
        tc_fence_after();
        for (int kk = 0; kk < N / 16; kk++)
            mma_ts(tmem + 128, tmem + 256 + kk * 8,
                   smem_desc_sw128(smem_u32(sm + kB) + kk * 2048, kPanelB, 1024),
                   idesc_bf16(128, 128, 0, 1), kk > 0);
        mma_commit(bar + 2);
    }
    __syncwarp();
    ok = ok && __all_sync(0xffffffffu, wait_phase(bar + 2, 0, w));
    if (ok) {
        tc_fence_after();
        for (int c = 0; c < 4; c++) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_off + 128 + c * 32, v);
            tmem_wait_ld();
            for (int k = 0; k < 32; k++) eout[r * 128 + c * 32 + k] = __uint_as_float(v[k]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// A barrier nobody arrives on: the bounded wait must give up and report.
__global__ void wait_kernel(int *status, long long limit, int *result) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const WaitCtx w{limit, status, &abort_flag};
    const bool ok = wait_phase(&bar, 0, w);
    if (threadIdx.x == 0) result[0] = ok ? 1 : 0;
}

// exp2_poly_x2 on n values (pairs of consecutive entries), next to the MUFU ex2.
__global__ void exp2_kernel(const float *x, float *poly, float *mufu, int n) {
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i + 1 >= n + 1) return;
    const float a = x[i], b = i + 1 < n ? x[i + 1] : 0.f;
    float lo, hi;
    f2_unpack(exp2_poly_x2(f2_pack(a, b)), lo, hi);
    poly[i] = lo;
    mufu[i] = fast_exp2(a);
    if (i + 1 < n) {
        poly[i + 1] = hi;
        mufu[i + 1] = fast_exp2(b);
    }
}

typedef CUresult (*EncodeFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                             const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                             const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                             CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool map2d(CUtensorMap *m, const void *base, uint64_t rows, uint32_t box_rows) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess || !fn)
        return false;
    cuuint64_t dims[2] = {128, rows}, strides[1] = {256};
    cuuint32_t box[2] = {64, box_rows}, estr[2] = {1, 1};
    return ((EncodeFn)fn)(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int N>
int run_gemm(const void *a, const void *b, float *d, float *e, int *status) {
    CUtensorMap ma, mb;
    if (!map2d(&ma, a, 128, 128) || !map2d(&mb, b, N, N)) return -1;
    const int smem = 32768 + 2 * N * 128 + 64 + 1024;
    if (cudaFuncSetAttribute(gemm_kernel<N>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
        return -2;
    gemm_kernel<N><<<1, 128, smem>>>(ma, mb, d, e, status);
    return (int)cudaDeviceSynchronize();
}

}  // namespace

extern "C" __attribute__((visibility("default"))) int selftest_gemm(const void *a, const void *b,
                                                                  int n, float *d, float *e,
                                                                  int *status) {
    switch (n) {
        case 64: return run_gemm<64>(a, b, d, e, status);
        case 80: return run_gemm<80>(a, b, d, e, status);
        case 128: return run_gemm<128>(a, b, d, e, status);
    }
    return -3;
}

extern "C" __attribute__((visibility("default"))) int selftest_wait(int *status, long long limit,
                                                                  int *result) {
    wait_kernel<<<1, 32>>>(status, limit, result);
    return (int)cudaDeviceSynchronize();
}

extern "C" __attribute__((visibility("default"))) int selftest_exp2(const float *x, float *poly,
                                                                  float *mufu, int n) {
    exp2_kernel<<<(n / 2 + 128) / 128, 128>>>(x, poly, mufu, n);
    return (int)cudaDeviceSynchronize();
}
