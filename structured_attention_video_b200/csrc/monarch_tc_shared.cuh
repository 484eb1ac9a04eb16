// monarch_tc_shared.cuh -- what the tensor-core family's forward
// (monarch_sm100.cu) and backward (monarch_bwd_sm100.cu) translation units share:
// tile constants, the TMA loads of the L-step's operands, the workspace of the
// forward's intermediates and the host functions that enqueue its kernels.
#pragma once

#include "monarch_common.cuh"
#include "tc_primitives.cuh"

#include <cuda.h>

namespace monarch {
namespace tcs {

using namespace tc;

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kD = 128;                        // head dimension of this path
constexpr uint32_t kPanel = 128 * 128;         // 128 rows x 64 bf16 (128 B), SW128
constexpr uint32_t kTile = 2 * kPanel;         // 128 rows x 128 bf16
constexpr int kMaxSmem = 232448;               // sm_100 opt-in dynamic shared memory
constexpr long long kCleanupPolls = 1LL << 22;

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Warp-uniform bounded wait: all 32 lanes take the same decision.
__device__ __forceinline__ bool wait_warp(uint64_t *bar, uint32_t parity, const WaitCtx &w) {
    bool ok = wait_phase(bar, parity, w);
    return __all_sync(0xffffffffu, ok);
}

// Key rows per (q̄ row, head) slab of Ktil, Z and the entropy panels: b1k, or
// with key-column tiles b1k rounded up to 64, so that the t key tiles of one
// column v (q̄ rows v*t + g') form one run of t*slab keys in which every 64-key
// half (one gather box with key-column tiles) lies inside one tile.  The rows
// past b1k of each tile hold Ktil = Z = 0 and an entropy of -1e30
// (tc_keypad_kernel): their L-step logits are -1e30 and their probabilities
// exactly 0; a problem's first half always holds real keys, so the running
// maximum starts on one.
__host__ __device__ __forceinline__ int key_slab(const Problem &p) {
    return p.key_tiles ? (p.b1k + 63) / 64 * 64 : p.b1k;
}

// Ktil and Z are stored [bh][u'][panel][r][64] (r = q̄ row, t*b2 of them; panel =
// 64-column half of d = 128): the R-step's natural order.  Flat key row
// z = (bh*t*b2 + r)*slab + u' (the order the L-step walks) addresses panel pn of
// (bh, u', r) through the 5-D map (x, r, panel, u', bh).
__device__ __forceinline__ void kz_coords(const Problem &p, int z, int &r, int &u, int &bh) {
    const int slab = key_slab(p), rows = p.tiles * p.b2;
    const int rid = z / slab;
    u = z % slab;
    r = rid % rows;
    bh = rid / rows;
}

// One 128-row tile of query rows (u, v), u = u0 .. u0 + 127 at column v of head bh,
// through the 5-D query map: (x, v, u, head, batch), or (x, head, v, u, batch) for
// [B][N][H][d] (the map's dimensions run in order of increasing stride); rows past
// b1 read zeros.
__device__ __forceinline__ void ls_load_q(void *dst, const CUtensorMap *map, int x, int v, int u0,
                                          int bh, const Problem &p, uint64_t *bar) {
    const int hh = bh % p.H, bb = bh / p.H;
    if (p.layout == kLayoutBNHD)
        tma_load_5d(dst, map, x, hh, v, u0, bb, bar);
    else
        tma_load_5d(dst, map, x, v, u0, hh, bb, bar);
}

// Panel pn of the 128 key rows z .. z + 127 (flat, see kz_coords) of Ktil or Z:
// 128 blocks u' of one q̄ row r (blocks past the slab read zeros), or with
// key-column tiles two boxes of 64, each inside one key tile (a 64-row box
// lands 8 KB on, where the 128-byte swizzle pattern repeats).
__device__ __forceinline__ void ls_load_kz(void *dst, const CUtensorMap *map, int pn, int z,
                                           const Problem &p, uint64_t *bar) {
    int r, u, bh;
    kz_coords(p, z, r, u, bh);
    tma_load_5d(dst, map, 0, r, pn, u, bh, bar);
    if (p.key_tiles) {
        kz_coords(p, z + 64, r, u, bh);
        tma_load_5d(static_cast<uint8_t *>(dst) + 64 * 128, map, 0, r, pn, u, bh, bar);
    }
}

enum LsMode { kLsOut = 0, kLsStat = 1, kLsAgg = 2 };

struct TcWorkspace {
    __nv_bfloat16 *qbar, *ktil, *z;
    uint4 *hx;            // [BH][t][b2][b1] rows of 32 bytes
    __nv_bfloat16 *qblk;  // iters > 1: aggregated queries per block [BH][b1][mpad][d]
    uint4 *lam;           // iters > 1: log-sum-exp panels [BH][N] rows of 32 bytes
};

// Key rows of Ktil, Z and the entropy panels over all heads and q̄ rows.
inline size_t key_rows(const Problem &p) { return (size_t)p.BH * p.tiles * p.b2 * key_slab(p); }

TcWorkspace carve(const Problem &p, void *base);
size_t al256(size_t x);
int b2_padded(int b2);
int qbar_tiles(const Problem &p);
int sm_count();
uint32_t rstep_smem(int b2p, int nmt, int hdirect, int pack = 1);
bool make_map(CUtensorMap *m, const void *base, int rank, const uint64_t *dims,
              const uint64_t *strides, const uint32_t *box,
              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B);
// Keys or values (4-D, box of `rows` tokens) and queries (5-D gather of one column
// v over 128 block rows) in the call's layout.
bool map_keys(CUtensorMap *m, const void *base, const Problem &p, uint32_t rows);
bool map_queries(CUtensorMap *m, const void *base, const Problem &p);
// The forward's kernels: S1, the R-step (qblk: per-block aggregated queries; split:
// R in two bfloat16 parts), the L-step in one of its modes.
cudaError_t run_qbar(const Problem &p, const void *q, const TcWorkspace &ws, cudaStream_t stream);
cudaError_t run_rstep(const Problem &p, const TcWorkspace &ws, const void *k, const void *v,
                      int qblk, float c_log2, int *status, long long wait_limit, int stall,
                      cudaStream_t stream, int split = 0);
cudaError_t run_lstep(const Problem &p, const TcWorkspace &ws, const void *q, void *out, int mode,
                      float c_log2, int *status, long long wait_limit, int stall,
                      cudaStream_t stream);

template <typename K>
cudaError_t set_smem(K kernel, uint32_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace tcs
}  // namespace monarch
