// monarch_common.cuh -- index arithmetic, problem description and the device
// status word shared by the kernels of the Monarch attention library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <mutex>
#include <utility>
#include <vector>

#include "../../include/monarch_attn.h"

namespace monarch {

// Token n = u*b2 + v (block row u, column v); the Monarch permutation P sends
// it to v*b1 + u (explainer page, "Monarch矩阵" section: a fixed permutation
// between the two block-diagonal factors).
__host__ __device__ __forceinline__ int block_row(int64_t n, int b2) { return (int)(n / b2); }
__host__ __device__ __forceinline__ int block_col(int64_t n, int b2) { return (int)(n % b2); }
__host__ __device__ __forceinline__ int64_t shuffle(int u, int v, int b1) {
    return (int64_t)v * b1 + u;
}

// Tiled Monarch ("创新二：平铺Monarch参数化", Fig. 2): block rows split into t
// contiguous tiles T_g = [floor(g*b1/t), floor((g+1)*b1/t)).
__host__ __device__ __forceinline__ int tile_begin(int g, int b1, int tiles) {
    return (int)(((int64_t)g * b1) / tiles);
}
__host__ __device__ __forceinline__ int tile_max_rows(int b1, int tiles) {
    return (b1 + tiles - 1) / tiles;
}

// Everything a kernel needs to know about one call.
struct Problem {
    int B, H, BH;        // batch, heads, B*H
    int N, d;            // tokens per head, head dim
    int b1, b2, tiles;   // Monarch blocks and tiles
    int iters;
    float scale;         // 1/sqrt(d)
    // the (head, tile) units this call computes, unit = (b*H + h)*tiles + g:
    // [unit_begin, unit_end); every unit is independent from the aggregated
    // query to its output rows (all of them by default)
    int unit_begin, unit_end;
    // keys and values: Nk = b1k * b2 tokens in b1k blocks (Nk = N, b1k = b1 for
    // self-attention over one clip; more when the queries of a chunk of frames
    // also attend to a cache of earlier frames)
    int Nk, b1k;
    // layout of q, k, v and the output: kLayoutBHND or kLayoutBNHD (below)
    int layout;
    // which axis the tiles split (the tiled parameterisation does not fix it):
    // 0, the query rows u of every block (tile g owns R_{u',g} and the rows
    // u in T_g); 1, the key columns v' of every block (key tile g' owns the
    // columns [floor(g' b2/t), floor((g'+1) b2/t)), R_{u',g'} is a softmax over
    // them, and every query row's L runs over the b1k*t (block, key tile)
    // super-keys).  With key tiles the units are still (head, g') for the
    // aggregated queries and the R-step; the L-step runs per head.
    int key_tiles;
    __host__ __device__ int head_begin() const { return unit_begin / tiles; }
    __host__ __device__ int head_end() const { return (unit_end + tiles - 1) / tiles; }
};

// Query rows that unit g aggregates and whose output it writes: the rows of
// tile g, or all b1 rows with key tiles.
__host__ __device__ __forceinline__ int unit_row_begin(const Problem &p, int g) {
    return p.key_tiles ? 0 : tile_begin(g, p.b1, p.tiles);
}
__host__ __device__ __forceinline__ int unit_row_end(const Problem &p, int g) {
    return p.key_tiles ? p.b1 : tile_begin(g + 1, p.b1, p.tiles);
}
// Key columns of block u' that the R-step of tile g takes its softmax over:
// all b2, or the key tile's own with key tiles.
__host__ __device__ __forceinline__ int unit_col_begin(const Problem &p, int g) {
    return p.key_tiles ? tile_begin(g, p.b2, p.tiles) : 0;
}
__host__ __device__ __forceinline__ int unit_col_end(const Problem &p, int g) {
    return p.key_tiles ? tile_begin(g + 1, p.b2, p.tiles) : p.b2;
}

// Layouts of the inputs and the output: [B][H][N][d] (the tokens of a head are
// contiguous rows) or [B][N][H][d] (the heads of a token are contiguous).
// Element j of token n of head bh = b*H + h sits at
//   head_base(p, bh, n_tokens) + n * tok_stride(p) + j.
// Every intermediate in the workspace keeps its own [B*H]-major layout.
constexpr int kLayoutBHND = 0, kLayoutBNHD = 1;
__host__ __device__ __forceinline__ int64_t tok_stride(const Problem &p) {
    return p.layout == kLayoutBNHD ? (int64_t)p.H * p.d : (int64_t)p.d;
}
__host__ __device__ __forceinline__ int64_t head_base(const Problem &p, int bh, int ntok) {
    return p.layout == kLayoutBNHD
               ? ((int64_t)(bh / p.H) * ntok * p.H + bh % p.H) * p.d
               : (int64_t)bh * ntok * p.d;
}

// Kernels that can give up a bounded wait receive a pointer to the device
// status word of the library (one int per device, read and cleared by
// monarch_last_device_status) and record MONARCH_ERR_TIMEOUT there.
constexpr long long kDefaultWaitLimit = 1LL << 22;

__device__ __forceinline__ void record_status(int *status, int code) {
    atomicCAS(status, 0, code);
}

// Kernel families, for the optional per-kernel timing of monarch_profile_*.
enum KernelId {
    K_QBAR_MEAN = 0,      // S1, generic
    K_RSTEP = 1,          // S2, generic
    K_LSTEP = 2,          // S3, generic
    K_QBAR_WEIGHTED = 3,  // S4, generic
    K_TC_QBAR = 4,        // S1, tensor-core path
    K_TC_RSTEP = 5,       // S2, tensor-core path
    K_TC_LSTEP = 6,       // S3, tensor-core path
    K_TC_LSTAT = 7,       // S3 row statistics of the iterations before the last (tensor-core)
    K_TC_QAGG = 8,        // S4 re-aggregated queries (tensor-core)
    K_BWD_L = 9,          // backward of the L-step and the output (generic)
    K_BWD_R = 10,         // backward of the R-step and the aggregation (generic)
    K_TC_BWD_DELTA = 11,  // tensor-core backward: delta = sum L dP per query row
    K_TC_BWD_DKZ = 12,    // tensor-core backward: dKtil, dZ, dH per key row
    K_TC_BWD_DQ = 13,     // tensor-core backward: dq through the L-step
    K_TC_BWD_R = 14,      // tensor-core backward: dk, dv and s*da per block
    K_TC_BWD_DQBAR = 15,  // tensor-core backward: dq̄ partial sums and the final dq
    K_COUNT = 16
};

// Brackets one kernel launch with CUDA events while profiling is enabled.
class ProfileScope {
  public:
    ProfileScope(KernelId id, cudaStream_t stream);
    ~ProfileScope();

  private:
    KernelId id_;
    cudaStream_t stream_;
    void *start_ = nullptr;
};

// Device addresses of module-scope __device__ variables are valid only in the
// CUDA context that loaded the module: a cache of such an address must be keyed
// by the context, not by the device ordinal (a primary context that was reset,
// or a context the caller created and made current, loads the module again at
// another address).  current_context_id() gives the id of the context current
// on the calling thread (CUDA never reuses an id within a process).
bool current_context_id(unsigned long long *id);

// The device address of one module-scope symbol, looked up with
// cudaGetSymbolAddress once per context (with that context current) and cached
// under the context id.  lookup() must run in the translation unit that
// defines the symbol.  Nothing here allocates device memory.
class SymbolAddressCache {
  public:
    template <typename T> cudaError_t lookup(const T &symbol, void **out) {
        unsigned long long ctx = 0;
        bool have_ctx = current_context_id(&ctx);
        if (have_ctx) {
            std::lock_guard<std::mutex> lock(mu_);
            for (const auto &e : entries_)
                if (e.first == ctx) {
                    *out = e.second;
                    return cudaSuccess;
                }
        }
        void *ptr = nullptr;
        cudaError_t err = cudaGetSymbolAddress(&ptr, symbol);   // creates the context if needed
        if (err != cudaSuccess) return err;
        if (!have_ctx) have_ctx = current_context_id(&ctx);
        if (have_ctx) {
            std::lock_guard<std::mutex> lock(mu_);
            entries_.emplace_back(ctx, ptr);
        }
        *out = ptr;
        return cudaSuccess;
    }

  private:
    std::mutex mu_;
    std::vector<std::pair<unsigned long long, void *>> entries_;
};

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Host-side argument validation shared by the entry points; fills *p on success.
monarch_status validate_shape(int B, int H, int f, int h, int w, int d, int b1, int b2, int tiles,
                              int iters, monarch_dtype dtype, Problem *p);

// Generic (SIMT) path: float32 intermediates.
struct GenericWorkspace {
    float *qbar;   // iters == 1: [BH][t][b2][d];  iters > 1: [BH][t][b2][b1k][d]
    float *ktil;   // [BH][t][b2][b1k][d]  Ktil[g][v][u'] = sum_v' R_{u',g}[v,v'] k_(u',v')
    float *z;      // [BH][t][b2][b1k][d]  Z[g][v][u']    = sum_v' R_{u',g}[v,v'] v_(u',v')
    float *hent;   // [BH][t][b2][b1k]     entropy of R_{u',g}[v,:]
    float *lse;    // [BH][N]              row log-sum-exp of the L-step (iters > 1)
};

size_t generic_workspace_bytes(const Problem &p, bool &overflow);
GenericWorkspace generic_workspace_carve(const Problem &p, void *base);
// S1 and the first R-step only (qbar, Ktil, Z, H into the workspace), for the
// backward pass of one iteration.
cudaError_t generic_rstep_only(const Problem &p, monarch_dtype dtype, const void *q,
                               const void *k, const void *v, const GenericWorkspace &ws,
                               cudaStream_t stream);

// Backward pass of one iteration (float32 intermediates after the forward's).
struct BwdWorkspace {
    float *lse, *delta;   // [BH][N]  per query row: L-step log-sum-exp, dy.y
    float *dql;           // [BH][N][d]  the L-step's part of dq
    float *dkt, *dz;      // [BH][t][b2][b1k][d]  dKtil, dZ
    float *dh;            // [BH][t][b2][b1k]     dH
    float *lsea, *ea, *rho;   // [BH][t][b2][b1k]  per R row: lse(a), E_R[a], sum R dR
    float *dqbar;         // [BH][t][b2][d]
};
size_t backward_workspace_bytes(const Problem &p, monarch_dtype dtype, bool &overflow);
// status/wait_limit: the device status word and the poll limit of the bounded
// waits (the tensor-core L-step side runs when `status` is given and it applies)
cudaError_t generic_backward(const Problem &p, monarch_dtype dtype, const void *q, const void *k,
                             const void *v, const void *dy, void *dq, void *dk, void *dv,
                             void *workspace, int *status, long long wait_limit,
                             cudaStream_t stream);
cudaError_t generic_forward(const Problem &p, monarch_dtype dtype, const void *q, const void *k,
                            const void *v, void *out, const GenericWorkspace &ws,
                            cudaStream_t stream);

cudaError_t index_maps_device(int N, int b1, int b2, int tiles, int32_t *u_of_n,
                              int32_t *v_of_n, int32_t *perm, int32_t *tile_lo,
                              cudaStream_t stream);

}  // namespace monarch
