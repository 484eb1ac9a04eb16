// monarch_sm100.cu -- sm_100a tensor-core kernels of the Monarch attention
// forward pass (bfloat16 inputs, d = 128, one alternating iteration).
//
// Steps (MonarchAttention as the MonarchRT pages describe it: explainer page,
// "Monarch矩阵" section and Fig. 3; tiles from "创新二：平铺Monarch参数化", Fig. 2;
// the entropy term after the VMonarch abstract's online entropy):
//   S1 tc_qbar_kernel   qbar[g][v] = mean_{u in T_g} q_(u,v) -> bf16, rows
//                       r = g*b2 + v of a [t*b2 padded to 128] x d tile stack
//   S2 tc_rstep_kernel  per block u' and 128-row tile of qbar:
//                         S = qbar K_u'^T                  (tcgen05, SMEM x SMEM)
//                         R = rowsoftmax(s S), H = entropy (float32, per thread row)
//                         [Z | Ktil] = R [V_u' | K_u']     (tcgen05, R from TMEM)
//                       Z and Ktil leave through TMA stores whose 4-D tensor map
//                       folds the Monarch permutation: row (g, v) of block u'
//                       lands at [bh][g*b2+v][u'] (rows past t*b2 are clipped).
//   S3 tc_lstep_kernel  per (bh, g, v) and pair of 128-query tiles: the queries
//                       (u, v), u in T_g, come through a 3-D tensor map that
//                       strides over b2 (P^T folded into the load); online
//                       softmax over the b1 blocks with logits s q.Ktil + H,
//                       O accumulated in TMEM, rows written back strided.
// The entropy enters the L-step's logit MMA: the R-step stores, per key row of
// Ktil, a 16-column bfloat16 panel [H'_hi, H'_lo, 0, ...] with H' = H / (s ln 2)
// (split in two bfloat16 parts that sum to H' within 2^-16 relative), and the
// L-step adds one K-step of an all-ones query panel times that panel, so S
// arrives in TMEM as (s q.Ktil + H) / (s ln 2) with no per-element entropy work.
// Warp roles (384 threads): warp 0 TMA producer (in the L-step: queries, Ktil
// and entropies; warp 2 produces Z), warp 1 MMA issuer and TMEM owner, warps
// 4-7 and 8-11 the two softmax (L-step) or the softmax and epilogue (R-step)
// warpgroups; the remaining warps idle.  Every wait on another role is
// a bounded mbarrier wait (tc_primitives.cuh): on time-out the kernel records
// MONARCH_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and returns.
#include "monarch_sm100.cuh"
#include "tc_primitives.cuh"

#include <mutex>

namespace monarch {
namespace {

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

// =====================================================================
// S1: aggregated queries
// =====================================================================
__global__ void __launch_bounds__(128) tc_qbar_kernel(const __nv_bfloat16 *__restrict__ q,
                                                      __nv_bfloat16 *__restrict__ qbar, Problem p,
                                                      int mpad) {
    const int row_elems = p.b2 * kD;
    const int nchunk = (row_elems / 8 + 127) / 128;
    const int chunk = blockIdx.x % nchunk;
    // every tile of the heads that the unit range touches (the R-step reads all
    // of a head's aggregated rows, padding included)
    const int bhg = blockIdx.x / nchunk + p.head_begin() * p.tiles;
    const int g = bhg % p.tiles, bh = bhg / p.tiles;
    const int col = (chunk * 128 + threadIdx.x) * 8;
    const int u0 = tile_begin(g, p.b1, p.tiles), u1 = tile_begin(g + 1, p.b1, p.tiles);
    if (col < row_elems) {
        const uint4 *src = reinterpret_cast<const uint4 *>(q + (int64_t)bh * p.N * kD +
                                                           (int64_t)u0 * row_elems + col);
        const int64_t stride = row_elems / 8;
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; i++) acc[i] = 0.f;
        int u = u0;
        // eight independent 16-byte loads in flight per thread: the grid has only
        // B*H*t*ceil(b2*d/1024) blocks, too few warps to cover the memory latency
        for (; u + 8 <= u1; u += 8) {
            uint4 x[8];
#pragma unroll
            for (int k = 0; k < 8; k++) x[k] = __ldg(src + k * stride);
            src += 8 * stride;
#pragma unroll
            for (int k = 0; k < 8; k++) {
                const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&x[k]);
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    float2 f = __bfloat1622float2(h[i]);
                    acc[2 * i] += f.x;
                    acc[2 * i + 1] += f.y;
                }
            }
        }
        for (; u < u1; u++) {
            uint4 x = __ldg(src);
            src += stride;
            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&x);
#pragma unroll
            for (int i = 0; i < 4; i++) {
                float2 f = __bfloat1622float2(h[i]);
                acc[2 * i] += f.x;
                acc[2 * i + 1] += f.y;
            }
        }
        const float inv = 1.f / (float)(u1 - u0);
        uint4 o;
        uint32_t *ow = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
        for (int i = 0; i < 4; i++) ow[i] = pack_bf16(acc[2 * i] * inv, acc[2 * i + 1] * inv);
        *reinterpret_cast<uint4 *>(qbar + ((int64_t)bh * mpad + (int64_t)g * p.b2) * kD + col) = o;
    }
    if (g == 0) {   // zero the padding rows [t*b2, mpad) of this head
        const int64_t pad = (int64_t)(mpad - p.tiles * p.b2) * kD;
        __nv_bfloat16 *base = qbar + ((int64_t)bh * mpad + (int64_t)p.tiles * p.b2) * kD;
        for (int64_t e = col; e < pad; e += (int64_t)nchunk * 128 * 8)
            *reinterpret_cast<uint4 *>(base + e) = make_uint4(0, 0, 0, 0);
    }
}

// =====================================================================
// S3: L-step with the output (persistent: each CTA walks a strided list of
// (bh, g, v, query-pair) problems, two 128-query tiles per problem)
//
// 16 warps.  Warps 0-3 and 4-7: the softmax warpgroups of query tiles 0 and 1
// (one query row per thread); warps 8-11: the epilogue warpgroup (O / l to
// bfloat16 rows of Y, off the softmax warps' chain); warp 12: the TMA producer
// of Ktil and its entropy panel; warp 13: the MMA issuer; warp 14: the
// producer of Z; warp 15: the producer of the query tiles.  setmaxnreg moves registers from the
// producer and epilogue warpgroups to the softmax warpgroups.
// Tensor memory: S_0 | S_1 | O_0 | O_1 (128 columns each); P_t overwrites the
// first 64 columns of S_t as packed bfloat16 pairs.
// =====================================================================
namespace ls {
constexpr int kThreads = 512;
constexpr int kSoftmaxRegs = 176, kEpilogueRegs = 96, kProducerRegs = 64;
static_assert(2 * kSoftmaxRegs + kEpilogueRegs + kProducerRegs == 4 * (65536 / kThreads),
              "the warpgroups' registers must add up to the launch's 128 per thread");
// one pair of every kPolyEvery takes its exponentials on the FMA pipe (0: none).
// Measured at 720p: the softmax is bound by issue slots, not by the MUFU, so the
// polynomial's extra instructions cost more than the exponentials it moves
// (1.30 ms per step with a quarter on the polynomial, 1.25 ms with none).
constexpr int kPolyEvery = 0;
constexpr uint32_t kQ = 0;                          // query tiles 0, 1
constexpr uint32_t kK = 2 * kTile;                  // Ktil stages 0, 1
constexpr uint32_t kZ = kK + 2 * kTile;             // Z stages 0, 1
constexpr uint32_t kHx = kZ + 2 * kTile;            // entropy panels (128 x 32 B) of the Ktil stages
constexpr uint32_t kPanelHx = 128 * 32;
constexpr uint32_t kQx = kHx + 2 * kPanelHx;        // the all-ones query panel
constexpr uint32_t kL = kQx + kPanelHx;             // row sums [problem parity][tile][128]
constexpr uint32_t kStg = kL + 2048;                // epilogue: 4 warps x 32 rows x 128 B
constexpr uint32_t kBar = kStg + 4 * 4096;
constexpr uint32_t kSmem = kBar + 512;              // the base is 1024-aligned (checked)
static_assert(kSmem <= (uint32_t)kMaxSmem, "L-step shared memory");
}  // namespace ls

struct LsArgs {
    Problem p;
    int nchunks;    // key chunks of 128 blocks
    int npairs;     // pairs of 128-query tiles per (g, v)
    int nprob;      // problems of the unit range: units * b2 * npairs
    int prob0;      // first problem: unit_begin * b2 * npairs
    float c_log2;   // (1/sqrt(d)) * log2(e)
    __nv_bfloat16 *out;
    int *status;
    long long limit;
    int stall;      // test hook: the MMA warp first waits on a barrier nothing completes
};

struct LsProblem {
    int bh, g, v, u_start, u1, key_row0;
};

__device__ __forceinline__ LsProblem ls_problem(const LsArgs &a, int unit) {
    const Problem &p = a.p;
    LsProblem q;
    unit += a.prob0;
    const int pair = unit % a.npairs;
    unit /= a.npairs;
    q.v = unit % p.b2;
    unit /= p.b2;
    q.g = unit % p.tiles;
    q.bh = unit / p.tiles;
    q.u1 = tile_begin(q.g + 1, p.b1, p.tiles);
    q.u_start = tile_begin(q.g, p.b1, p.tiles) + 256 * pair;
    q.key_row0 = ((q.bh * p.tiles + q.g) * p.b2 + q.v) * p.b1;
    return q;
}

__global__ void __launch_bounds__(ls::kThreads, 1)
tc_lstep_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmZ, const __grid_constant__ CUtensorMap tmHx,
                LsArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // the SW128 operand tiles need a 1024-byte aligned base; the layout leaves no
    // room to align by hand, so a misaligned base is reported, not worked around
    if ((smem_u32(smem_raw) & 1023u) != 0) {
        if (threadIdx.x == 0) record_status(a.status, MONARCH_ERR_CUDA);
        return;
    }
    uint8_t *sm = smem_raw;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + ls::kBar);
    uint64_t *q_full = bars + 0;     // [2 tiles]
    uint64_t *q_empty = bars + 2;    // [2 tiles]: the tile's last S MMA of a problem done
    uint64_t *k_full = bars + 4;     // [2 stages]: Ktil and its entropy panel
    uint64_t *k_empty = bars + 6;    // [2 stages]: both S MMAs of the chunk done
    uint64_t *z_full = bars + 8;     // [2 stages]
    uint64_t *z_empty = bars + 10;   // [2 stages]: both PV MMAs of the chunk done
    uint64_t *s_full = bars + 16;    // [2 tiles]
    uint64_t *p_full = bars + 18;    // [2 tiles], one arrival per softmax warp
    uint64_t *o_full = bars + 20;    // [2 tiles]: the last PV MMA of a problem done
    uint64_t *o_free = bars + 22;    // [2 tiles], one arrival per epilogue warp: O_t read
    uint64_t *l_full = bars + 24;    // [2 tiles], one arrival per softmax warp: row sums written
    uint64_t *mma_done = bars + 26;
    uint64_t *stall_bar = bars + 27;   // never completed (fault-injection hook)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 28);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 29);
    float *lsum = reinterpret_cast<float *>(sm + ls::kL);   // [2][2][128]

    const Problem &p = a.p;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nmine = a.nprob > (int)blockIdx.x
                          ? (a.nprob - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int nch = a.nchunks;

    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; t++) {
            mbar_init(q_full + t, 1);
            mbar_init(q_empty + t, 1);
            mbar_init(k_full + t, 1);
            mbar_init(k_empty + t, 1);
            mbar_init(z_full + t, 1);
            mbar_init(z_empty + t, 1);
            mbar_init(s_full + t, 1);
            mbar_init(p_full + t, 4);   // one arrival per softmax warp
            mbar_init(o_full + t, 1);
            mbar_init(o_free + t, 4);   // one arrival per epilogue warp
            mbar_init(l_full + t, 4);   // one arrival per softmax warp
        }
        mbar_init(mma_done, 1);
        mbar_init(stall_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // the all-ones query panel (every bfloat16 = 1.0, so its swizzle is moot):
    // the entropy K-step adds 1 * H'_hi + 1 * H'_lo (the panel's other columns are 0)
    for (int i = threadIdx.x; i < (int)(ls::kPanelHx / 16); i += blockDim.x)
        reinterpret_cast<uint4 *>(sm + ls::kQx)[i] =
            make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    fence_proxy_async_smem();   // generic writes -> the tensor cores' async proxy
    if (warp == 13) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtx w{a.limit, a.status, abort_flag};

    if (warp >= 12) {
        regs_dec<ls::kProducerRegs>();
        if (warp == 12) {
            // ---------------- producer of Ktil and its entropy panel: per chunk as
            // soon as the S MMAs of two chunks back are done (never behind a query
            // load, which has its own warp)
            int issued[2] = {0, 0};
            bool ok = true;
            for (int pi = 0; ok && pi < nmine; pi++) {
                const LsProblem pr = ls_problem(a, blockIdx.x + pi * gridDim.x);
                for (int j = 0; j < nch; j++) {
                    const int jc = pi * nch + j, sk = jc & 1;
                    if (jc >= 2 && !wait_warp(k_empty + sk, ((jc >> 1) - 1) & 1, w)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        // keys past b1 in the ragged last chunk belong to the next
                        // row (or are zero-filled past the array): masked later
                        mbar_expect_tx(k_full + sk, kTile + ls::kPanelHx);
                        for (int pn = 0; pn < 2; pn++)
                            tma_load_2d(sm + ls::kK + sk * kTile + pn * kPanel, &tmK, pn * 64,
                                        pr.key_row0 + j * 128, k_full + sk);
                        tma_load_2d(sm + ls::kHx + sk * ls::kPanelHx, &tmHx, 0,
                                    pr.key_row0 + j * 128, k_full + sk);
                    }
                    issued[sk]++;
                }
            }
            if (lane == 0)   // every issued copy lands before the CTA may exit
                for (int s = 0; s < 2; s++)
                    if (issued[s] > 0) wait_phase_cleanup(k_full + s, (issued[s] - 1) & 1, kCleanupPolls);
        } else if (warp == 15) {
            // ---------------- query producer: each query tile reloads as soon as its
            // own last S MMA of the previous problem is done; the next problem's
            // rows (a strided gather) are prefetched into L2 a whole problem ahead
            int qloads = 0;
            bool ok = true;
            for (int pi = 0; ok && pi < nmine; pi++) {
                const LsProblem pr = ls_problem(a, blockIdx.x + pi * gridDim.x);
                for (int t = 0; t < 2; t++) {
                    if (pi > 0 && !wait_warp(q_empty + t, (pi - 1) & 1, w)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        mbar_expect_tx(q_full + t, kTile);
                        for (int pn = 0; pn < 2; pn++)
                            tma_load_3d(sm + ls::kQ + t * kTile + pn * kPanel, &tmQ, pn * 64, pr.v,
                                        pr.bh * p.b1 + pr.u_start + t * 128, q_full + t);
                    }
                }
                if (!ok) break;
                qloads++;
                if (lane == 0 && pi + 1 < nmine) {
                    const LsProblem nx = ls_problem(a, blockIdx.x + (pi + 1) * gridDim.x);
                    for (int t = 0; t < 2; t++)
                        for (int pn = 0; pn < 2; pn++)
                            tma_prefetch_3d(&tmQ, pn * 64, nx.v, nx.bh * p.b1 + nx.u_start + t * 128);
                }
            }
            if (lane == 0)
                for (int t = 0; t < 2; t++)
                    if (qloads > 0) wait_phase_cleanup(q_full + t, (qloads - 1) & 1, kCleanupPolls);
        } else if (warp == 14) {
            // ---------------- Z producer: its own warp, so that a Ktil load never
            // queues behind the wait for a Z stage (released one PV later than Ktil)
            int issued_z[2] = {0, 0};
            bool ok = true;
            for (int pi = 0; ok && pi < nmine; pi++) {
                const LsProblem pr = ls_problem(a, blockIdx.x + pi * gridDim.x);
                for (int j = 0; j < nch; j++) {
                    const int jc = pi * nch + j, st = jc & 1;
                    if (jc >= 2 && !wait_warp(z_empty + st, ((jc >> 1) - 1) & 1, w)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        mbar_expect_tx(z_full + st, kTile);
                        for (int pn = 0; pn < 2; pn++)
                            tma_load_2d(sm + ls::kZ + st * kTile + pn * kPanel, &tmZ, pn * 64,
                                        pr.key_row0 + j * 128, z_full + st);
                    }
                    issued_z[st]++;
                }
            }
            if (lane == 0)
                for (int s = 0; s < 2; s++)
                    if (issued_z[s] > 0)
                        wait_phase_cleanup(z_full + s, (issued_z[s] - 1) & 1, kCleanupPolls);
        } else if (warp == 13) {
            // ---------------- MMA issuer.  Order: S_0 and S_1 of the first chunk, then
            // per chunk PV_0, S_0 of the next chunk, PV_1, S_1 of the next chunk, so
            // that a tile's chain never waits on the other tile's softmax.  S_t of
            // the next chunk overwrites the columns that PV_t reads as P: tcgen05
            // MMAs issued by one thread execute in issue order, so it follows PV_t
            // without a wait, and its commit (s_full) also covers PV_t, which orders
            // the softmax's rescale of O_t after PV_t.
            constexpr uint32_t idS = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idO = idesc_bf16(128, 128, 0, 1);
            const uint64_t dQ = smem_desc_sw128(smem_u32(sm + ls::kQ), 16, 1024);
            const uint64_t dK = smem_desc_sw128(smem_u32(sm + ls::kK), 16, 1024);
            const uint64_t dZ = smem_desc_sw128(smem_u32(sm + ls::kZ), kPanel, 1024);
            const uint64_t dQx = smem_desc_sw32(smem_u32(sm + ls::kQx));
            const uint64_t dHx = smem_desc_sw32(smem_u32(sm + ls::kHx));
            constexpr uint32_t kTileDesc = kTile >> 4, kHxDesc = ls::kPanelHx >> 4;
            const int total = nmine * nch;
            // fault injection: a wait that can only give up (bounded, then abort)
            bool ok = !a.stall || spin_warp(stall_bar, 0, w);
            auto issue_s = [&](int t, int jc) -> bool {
                const int sk = jc & 1;
                if (jc % nch == 0 && !spin_warp(q_full + t, (jc / nch) & 1, w)) return false;
                if (t == 0 && !spin_warp(k_full + sk, (jc >> 1) & 1, w)) return false;
                tc_fence_after();
                mma8_ss_k128(tmem + t * 128, dQ + t * kTileDesc, dK + sk * kTileDesc, idS, 0u);
                mma1_ss_acc(tmem + t * 128, dQx, dHx + sk * kHxDesc, idS);   // + H'
                mma_commit_warp(s_full + t);
                if (t == 1) mma_commit_warp(k_empty + sk);
                if (jc % nch == nch - 1) mma_commit_warp(q_empty + t);   // tile t no longer read
                return true;
            };
            auto issue_pv = [&](int t, int jc) -> bool {
                const int st = jc & 1, j = jc % nch;
                if (t == 0 && !spin_warp(z_full + st, (jc >> 1) & 1, w)) return false;
                if (!spin_warp(p_full + t, jc & 1, w)) return false;
                // the first PV of a problem overwrites O_t: the epilogue of the
                // previous problem must have read it
                if (j == 0 && jc >= nch && !spin_warp(o_free + t, ((jc / nch) - 1) & 1, w))
                    return false;
                tc_fence_after();
                mma8_ts_mn128(tmem + 256 + t * 128, tmem + t * 128, dZ + st * kTileDesc, idO,
                              j > 0 ? 1u : 0u);
                if (t == 1) mma_commit_warp(z_empty + st);
                if (j == nch - 1) mma_commit_warp(o_full + t);
                return true;
            };
            if (ok && total > 0) ok = issue_s(0, 0) && issue_s(1, 0);
            for (int jc = 0; ok && jc < total; jc++) {
                const bool more = jc + 1 < total;
                ok = issue_pv(0, jc) && (!more || issue_s(0, jc + 1)) && issue_pv(1, jc) &&
                     (!more || issue_s(1, jc + 1));
            }
            mma_commit_warp(mma_done);
            wait_phase_cleanup(mma_done, 0, kCleanupPolls);
        }
    } else if (warp >= 8) {
        // ---------------- epilogue warpgroup: per problem and tile, O_t / l to
        // bfloat16; each thread writes its own output row as sixteen 16-byte stores
        regs_dec<ls::kEpilogueRegs>();
        const int wq = warp & 3;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        bool ok = true;
        for (int pi = 0; ok && pi < nmine; pi++) {
            const LsProblem pr = ls_problem(a, blockIdx.x + pi * gridDim.x);
            for (int t = 0; t < 2; t++) {
                if (!wait_warp(o_full + t, pi & 1, w) || !wait_warp(l_full + t, pi & 1, w)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float inv_l = 1.f / lsum[((pi & 1) * 2 + t) * 128 + wq * 32 + lane];
                // O_t leaves tensor memory 32 columns at a time, straight into
                // bfloat16 pairs; once all of it is in registers the next
                // problem's first PV may overwrite it, and only then do the
                // global stores run
                uint32_t pk[64];
#pragma unroll
                for (int c = 0; c < 4; c++) {
                    float o[32];
                    tmem_ld32f(tmem + lane_off + 256 + t * 128 + c * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 16; k++)
                        pk[c * 16 + k] = pack_bf16(o[2 * k] * inv_l, o[2 * k + 1] * inv_l);
                }
                tc_fence_before();
                mbar_arrive_warp(o_free + t);
                // the warp's 32 rows leave through shared memory, half a row (128 B)
                // at a time: each lane writes its own row, then every store
                // instruction covers four whole row halves (eight 16-byte chunks
                // each), instead of 32 scattered 16-byte pieces
                uint8_t *stg = sm + ls::kStg + wq * 4096;
                const int u0w = pr.u_start + t * 128 + wq * 32;
#pragma unroll
                for (int hf = 0; hf < 2; hf++) {
#pragma unroll
                    for (int c = 0; c < 8; c++)   // chunk c at slot (c + row) mod 8: no bank pile-up
                        *reinterpret_cast<uint4 *>(stg + lane * 128 + ((c + lane) & 7) * 16) =
                            make_uint4(pk[hf * 32 + 4 * c], pk[hf * 32 + 4 * c + 1],
                                       pk[hf * 32 + 4 * c + 2], pk[hf * 32 + 4 * c + 3]);
                    __syncwarp();
#pragma unroll
                    for (int rr = 0; rr < 8; rr++) {
                        const int row = rr * 4 + (lane >> 3), c = lane & 7;
                        const uint4 val =
                            *reinterpret_cast<const uint4 *>(stg + row * 128 + ((c + row) & 7) * 16);
                        const int u = u0w + row;
                        if (u < pr.u1)
                            *reinterpret_cast<uint4 *>(
                                a.out + ((int64_t)pr.bh * p.N + (int64_t)u * p.b2 + pr.v) * kD +
                                hf * 64 + c * 8) = val;
                    }
                    __syncwarp();
                }
            }
        }
    } else {
        // ---------------- softmax warpgroups: tile t = 0 (warps 0-3), 1 (warps 4-7)
        regs_inc<ls::kSoftmaxRegs>();
        const int t = warp >> 2;
        const int wq = warp & 3;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const uint32_t tS = tmem + lane_off + t * 128;
        const uint32_t tO = tmem + lane_off + 256 + t * 128;
        const uint64_t c2 = f2_pack(a.c_log2, a.c_log2);
        bool ok = true;
        for (int pi = 0; ok && pi < nmine; pi++) {
            float m_run = -INFINITY, l_run = 0.f;
            for (int j = 0; j < nch; j++) {
                const int jc = pi * nch + j;
                if (!wait_warp(s_full + t, jc & 1, w)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // S = (s q.Ktil + H) / (s ln 2): scaled by c_log2 it is the logit in
                // log2 units, so the maximum is taken on S itself
                float x[128];
#pragma unroll
                for (int c = 0; c < 4; c++) tmem_ld32f(tS + c * 32, &x[c * 32]);
                tmem_wait_ld();
                float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                const int nvalid = p.b1 - j * 128;   // keys of this chunk inside the row
                if (nvalid < 128) {
                    // the ragged last chunk: keys past b1 belong to the next row
                    // (or are zero fill), so mask them by selection
#pragma unroll
                    for (int i = 0; i < 128; i++) x[i] = i < nvalid ? x[i] : -INFINITY;
                }
#pragma unroll
                for (int i = 0; i < 64; i++) mx4[i & 3] = fmax3(mx4[i & 3], x[2 * i], x[2 * i + 1]);
                const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
                // the running maximum moves only when it grows by more than 2^8 in
                // log2 units: the probabilities stay below 256 and O is rescaled rarely
                float alpha = 1.f;
                bool rescale = false;
                if ((mx - m_run) * a.c_log2 > 8.f) {
                    alpha = fast_exp2((m_run - mx) * a.c_log2);
                    m_run = mx;
                    rescale = true;
                }
                const uint64_t nmc2 = f2_pack(-m_run * a.c_log2, -m_run * a.c_log2);
                uint64_t sum2[4] = {0, 0, 0, 0};
#pragma unroll
                for (int h = 0; h < 2; h++) {
                    uint32_t pk[32];
#pragma unroll
                    for (int i = 0; i < 32; i++) {
                        const int e = h * 32 + i;
                        const uint64_t d2 = f2_fma(f2_pack(x[2 * e], x[2 * e + 1]), c2, nmc2);
                        uint64_t e2;
                        constexpr int kEvery = ls::kPolyEvery > 0 ? ls::kPolyEvery : 1;
                        if (ls::kPolyEvery > 0 && (i % kEvery) == kEvery - 1 && nvalid >= 128) {
                            e2 = exp2_poly_x2(d2);
                        } else {
                            float lo, hi;
                            f2_unpack(d2, lo, hi);
                            e2 = f2_pack(fast_exp2(lo), fast_exp2(hi));
                        }
                        sum2[i & 3] = f2_add(sum2[i & 3], e2);
                        float p0, p1;
                        f2_unpack(e2, p0, p1);
                        pk[i] = pack_bf16(p0, p1);
                    }
                    tmem_st32(tS + h * 32, pk);
                }
                float s0, s1;
                f2_unpack(f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3])), s0, s1);
                l_run = l_run * alpha + (s0 + s1);
                if (j > 0 && __any_sync(0xffffffffu, rescale)) {
                    // O_t is complete up to the previous chunk (the commit of this
                    // chunk's S covers the previous PV); scale it in four slices
#pragma unroll
                    for (int c = 0; c < 4; c++) {
                        float o[32];
                        tmem_ld32f(tO + c * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; i++) o[i] *= alpha;
                        tmem_st32f(tO + c * 32, o);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive_warp(p_full + t);
            }
            if (!ok) break;
            // the row sums for the epilogue; slot pi & 1 is rewritten two problems
            // later, when the epilogue has released O_t (o_free) of this problem,
            // which the first PV of the problem after next waits for
            lsum[((pi & 1) * 2 + t) * 128 + wq * 32 + lane] = l_run;
            mbar_arrive_warp(l_full + t);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 13) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// =====================================================================
// S2: R-step
// =====================================================================
struct RsArgs {
    Problem p;
    int nmt;             // 128-row tiles of qbar (t*b2 padded)
    int mpad;            // nmt * 128
    int bpc;             // blocks per CTA (flattened over heads and blocks)
    float c_log2;

    int *status;
    long long limit;
    int stall;           // test hook: the MMA warp first waits on a barrier nothing completes
};

template <int B2P>
struct RsLayout {
    static constexpr uint32_t kStage = 4 * B2P * 128;   // K and V: 2 panels each of B2P x 128 B
    static constexpr uint32_t kVOff = 2 * B2P * 128;    // V inside a stage
    static constexpr uint32_t kPanelKV = B2P * 128;
    __host__ __device__ static uint32_t kv(int nmt) { return (uint32_t)nmt * kTile; }
    __host__ __device__ static uint32_t stg(int nmt) { return kv(nmt) + 2 * kStage; }
    // entropy-panel staging of the softmax warps: 4 warps x 32 rows x 32 B
    __host__ __device__ static uint32_t hstg(int nmt) { return stg(nmt) + 4 * 8192; }
    __host__ __device__ static uint32_t bar(int nmt) { return hstg(nmt) + 4 * 1024; }
    __host__ __device__ static uint32_t smem(int nmt) { return bar(nmt) + 256 + 1024; }
};

template <int B2P>
__global__ void __launch_bounds__(384, 1)
tc_rstep_kernel(const __grid_constant__ CUtensorMap tmQb, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmZs,
                const __grid_constant__ CUtensorMap tmKs, const __grid_constant__ CUtensorMap tmHs,
                RsArgs a) {
    using L = RsLayout<B2P>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    const int nmt = a.nmt;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::bar(nmt));
    uint64_t *q_full = bars + 0;
    uint64_t *q_empty = bars + 1;
    uint64_t *kv_full = bars + 2;    // [2]
    uint64_t *kv_empty = bars + 4;   // [2]
    uint64_t *s_full = bars + 6;     // [2]
    uint64_t *s_free = bars + 8;     // [2]
    uint64_t *p_full = bars + 10;    // [2], one arrival per softmax warp
    uint64_t *o_full = bars + 12;    // [2]: Z part, Ktil part
    uint64_t *o_empty = bars + 14;   // [2], one arrival per epilogue warp
    uint64_t *mma_done = bars + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 17);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 18);
    uint64_t *stall_bar = bars + 19;   // never completed (fault-injection hook)

    const Problem &p = a.p;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // (head, block) items of the heads that the unit range touches
    const int total = p.head_end() * p.b1;
    const int first = p.head_begin() * p.b1 + blockIdx.x * a.bpc;
    const int nblk = min(a.bpc, total - first);
    const int nitems = nblk * nmt;
    const int tb2 = p.tiles * p.b2;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < 2; s++) {
            mbar_init(kv_full + s, 1);
            mbar_init(kv_empty + s, 1);
            mbar_init(s_full + s, 1);
            mbar_init(s_free + s, 1);
            mbar_init(p_full + s, 4);   // one arrival per softmax warp
            mbar_init(o_full + s, 1);
            mbar_init(o_empty + s, 4);   // one arrival per epilogue warp
        }
        mbar_init(mma_done, 1);
        mbar_init(stall_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtx w{a.limit, a.status, abort_flag};

    if (warp == 0) {
        // ---------------- producer: qbar tiles per head, K and V per block
        if (lane == 0) {
            int heads = 0, cur = -1, issued[2] = {0, 0};
            bool ok = true;
            for (int ib = 0; ib < nblk && ok; ib++) {
                const int fb = first + ib, bh = fb / p.b1, up = fb % p.b1;
                if (bh != cur) {
                    if (heads > 0 && !wait_phase(q_empty, (heads - 1) & 1, w)) break;
                    mbar_expect_tx(q_full, nmt * kTile);
                    for (int mt = 0; mt < nmt; mt++)
                        for (int pn = 0; pn < 2; pn++)
                            tma_load_2d(sm + mt * kTile + pn * kPanel, &tmQb, pn * 64,
                                        bh * a.mpad + mt * 128, q_full);
                    heads++;
                    cur = bh;
                }
                const int st = ib & 1;
                if (ib >= 2 && !wait_phase(kv_empty + st, ((ib >> 1) - 1) & 1, w)) break;
                uint8_t *stage = sm + L::kv(nmt) + st * L::kStage;
                mbar_expect_tx(kv_full + st, L::kStage);
                const int row = bh * p.N + up * p.b2;
                for (int pn = 0; pn < 2; pn++) {
                    tma_load_2d(stage + pn * L::kPanelKV, &tmK, pn * 64, row, kv_full + st);
                    tma_load_2d(stage + L::kVOff + pn * L::kPanelKV, &tmV, pn * 64, row,
                                kv_full + st);
                }
                issued[st]++;
            }
            if (heads > 0) wait_phase_cleanup(q_full, (heads - 1) & 1, kCleanupPolls);
            for (int s = 0; s < 2; s++)
                if (issued[s] > 0)
                    wait_phase_cleanup(kv_full + s, (issued[s] - 1) & 1, kCleanupPolls);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer: the whole warp runs the loop, one elected
        // lane issues each MMA (see mma_ss_warp)
        {
            constexpr uint32_t id1 = idesc_bf16(128, B2P, 0, 0);
            constexpr uint32_t id2 = idesc_bf16(128, 128, 0, 1);
            const uint64_t dQ = smem_desc_sw128(smem_u32(sm), 16, 1024);
            const uint64_t dK = smem_desc_sw128(smem_u32(sm + L::kv(nmt)), 16, 1024);
            const uint64_t dV = smem_desc_sw128(smem_u32(sm + L::kv(nmt)), L::kPanelKV, 1024);
            int heads = 0;
            // fault injection: a wait that can only give up (bounded, then abort)
            bool ok = !a.stall || spin_warp(stall_bar, 0, w);
            // S = qbar_mt K_u'^T for item i into S buffer i & 1
            auto gemm1 = [&](int i) -> bool {
                const int ib = i / nmt, mt = i % nmt;
                const int fb = first + ib, bh = fb / p.b1;
                if (mt == 0) {
                    if (ib == 0 || (fb - 1) / p.b1 != bh) {
                        if (!wait_warp(q_full, heads & 1, w)) return false;
                        heads++;
                    }
                    if (!wait_warp(kv_full + (ib & 1), (ib >> 1) & 1, w)) return false;
                }
                if (i >= 2 && !wait_warp(s_free + (i & 1), ((i >> 1) - 1) & 1, w)) return false;
                tc_fence_after();
                const uint64_t a0 = desc_plus(dQ, mt * kTile);
                const uint64_t b0 = desc_plus(dK, (ib & 1) * L::kStage);
#pragma unroll
                for (int kk = 0; kk < 8; kk++)
                    mma_ss_warp(tmem + (i & 1) * 128,
                           desc_plus(a0, (kk >> 2) * kPanel + (kk & 3) * 32),
                           desc_plus(b0, (kk >> 2) * L::kPanelKV + (kk & 3) * 32), id1, kk > 0);
                mma_commit_warp(s_full + (i & 1));
                const bool head_ends = (ib == nblk - 1) || ((fb + 1) / p.b1 != bh);
                if (mt == nmt - 1 && head_ends) mma_commit_warp(q_empty);
                return true;
            };
            if (ok && nitems > 0) ok = gemm1(0);
            for (int i = 0; ok && i < nitems; i++) {
                if (i + 1 < nitems && !gemm1(i + 1)) break;
                const int ib = i / nmt, mt = i % nmt;
                if (!wait_warp(p_full + (i & 1), (i >> 1) & 1, w)) break;
                tc_fence_after();
                const uint32_t pa = tmem + (i & 1) * 128;
                // 0: Z = R V, 1: Ktil = R K
                const uint64_t bz = desc_plus(dV, (ib & 1) * L::kStage + L::kVOff);
                const uint64_t bk = desc_plus(dV, (ib & 1) * L::kStage);
                if (i > 0 && !wait_warp(o_empty + 0, (i - 1) & 1, w)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < B2P / 16; kk++)
                    mma_ts_warp(tmem + 256, pa + kk * 8, desc_plus(bz, kk * 2048), id2, kk > 0 ? 1u : 0u);
                mma_commit_warp(o_full + 0);
                if (i > 0 && !wait_warp(o_empty + 1, (i - 1) & 1, w)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < B2P / 16; kk++)
                    mma_ts_warp(tmem + 384, pa + kk * 8, desc_plus(bk, kk * 2048), id2, kk > 0 ? 1u : 0u);
                mma_commit_warp(o_full + 1);
                mma_commit_warp(s_free + (i & 1));
                if (mt == nmt - 1) mma_commit_warp(kv_empty + (ib & 1));
            }
            mma_commit_warp(mma_done);
            wait_phase_cleanup(mma_done, 0, kCleanupPolls);
        }
    } else if (warp >= 4 && warp < 8) {
        // ---------------- softmax: R rows, entropy, normalised P back to TMEM (bf16)
        const int wq = warp & 3;
        const int r = wq * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        for (int i = 0; i < nitems; i++) {
            const int ib = i / nmt, mt = i % nmt;
            const int fb = first + ib, bh = fb / p.b1, up = fb % p.b1;
            if (!wait_warp(s_full + (i & 1), (i >> 1) & 1, w)) break;
            tc_fence_after();
            const uint32_t tS = tmem + lane_off + (i & 1) * 128;
            // the row's B2P logits: all TMEM loads in flight together, one wait
            float x[B2P];
#pragma unroll
            for (int c = 0; c < B2P / 16; c++) tmem_ld16f(tS + c * 16, &x[c * 16]);
            tmem_wait_ld();
            if (p.b2 < B2P) {   // padded key columns (uniform branch)
                // a large finite logit, not -inf: its probability is exactly 0 and
                // 0 * x stays finite in the entropy sum (no per-column condition)
#pragma unroll
                for (int col = 0; col < B2P; col++) x[col] = col < p.b2 ? x[col] : -1e30f;
            }
            // maximum with four independent chains
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int k = 0; k < B2P / 2; k++) mx4[k & 3] = fmax3(mx4[k & 3], x[2 * k], x[2 * k + 1]);
            const float mxr = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
            // base-2 exponentials of c * (x - max), packed in pairs; the row sum and
            // sum p * x (for the entropy) accumulate in four packed chains each
            const uint64_t c2 = f2_pack(a.c_log2, a.c_log2);
            const uint64_t nm2 = f2_pack(-mxr * a.c_log2, -mxr * a.c_log2);
            uint64_t l2[4] = {0, 0, 0, 0}, e2[4] = {0, 0, 0, 0};
            uint64_t pp[B2P / 2];
#pragma unroll
            for (int k = 0; k < B2P / 2; k++) {
                const uint64_t xs = f2_mul(f2_pack(x[2 * k], x[2 * k + 1]), c2);   // log2 units
                float d0, d1;
                f2_unpack(f2_add(xs, nm2), d0, d1);
                pp[k] = f2_pack(fast_exp2(d0), fast_exp2(d1));
                l2[k & 3] = f2_add(l2[k & 3], pp[k]);
                e2[k & 3] = f2_fma(pp[k], xs, e2[k & 3]);
            }
            float la, lb, ea, eb;
            f2_unpack(f2_add(f2_add(l2[0], l2[1]), f2_add(l2[2], l2[3])), la, lb);
            f2_unpack(f2_add(f2_add(e2[0], e2[1]), f2_add(e2[2], e2[3])), ea, eb);
            const float l = la + lb, inv = 1.f / l;
            const int row = mt * 128 + r;
            // entropy of the row in log2 units, log2(sum 2^x) - E_R[x] = H / ln 2,
            // stored divided by c_log2 = s log2(e) (the L-step's logits are
            // S * c_log2) as a bfloat16 pair hi + lo in the row's entropy panel
            {
                const float hp = (mxr * a.c_log2 + log2f(l) - (ea + eb) * inv) / a.c_log2;
                const __nv_bfloat16 hi = __float2bfloat16_rn(hp);
                const __nv_bfloat16 lo = __float2bfloat16_rn(hp - __bfloat162float(hi));
                const uint32_t pair = (uint32_t)__bfloat16_as_ushort(hi) |
                                      ((uint32_t)__bfloat16_as_ushort(lo) << 16);
                // the warp's 32 panel rows (32 B each) leave in one TMA store, which
                // clips the rows past t*b2; the previous item's store must have
                // finished reading the staging first
                uint8_t *hs = sm + L::hstg(nmt) + wq * 1024;
                if (lane == 0) tma_store_wait_read_all();
                __syncwarp();
                *reinterpret_cast<uint4 *>(hs + lane * 32) = make_uint4(pair, 0u, 0u, 0u);
                *reinterpret_cast<uint4 *>(hs + lane * 32 + 16) = make_uint4(0u, 0u, 0u, 0u);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_4d(&tmHs, hs, 0, up, mt * 128 + wq * 32, bh);
                    tma_store_commit();
                }
            }
            const uint64_t inv2 = f2_pack(inv, inv);
#pragma unroll
            for (int c = 0; c < B2P / 16; c++) {
                uint32_t pk[8];
#pragma unroll
                for (int k = 0; k < 8; k++) {
                    float p0, p1;
                    f2_unpack(f2_mul(pp[c * 8 + k], inv2), p0, p1);
                    pk[k] = pack_bf16(p0, p1);
                }
                tmem_st8(tS + c * 8, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive_warp(p_full + (i & 1));
        }
        if (lane == 0) tma_store_wait_all();   // the entropy stores complete before exit
    } else if (warp >= 8) {
        // ---------------- epilogue: Z and Ktil rows -> bf16 -> staging -> TMA store
        const int wq = warp & 3;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        uint8_t *stg = sm + L::stg(nmt) + wq * 8192;   // 2 panels x 32 rows x 128 B
        bool ok = true;
        for (int i = 0; ok && i < nitems; i++) {
            const int ib = i / nmt, mt = i % nmt;
            const int fb = first + ib, bh = fb / p.b1, up = fb % p.b1;
            for (int part = 0; part < 2; part++) {
                if (!wait_warp(o_full + part, i & 1, w)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t pk[64];
#pragma unroll
                for (int c = 0; c < 4; c++) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_off + 256 + part * 128 + c * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 16; k++)
                        pk[c * 16 + k] =
                            pack_bf16(__uint_as_float(o[2 * k]), __uint_as_float(o[2 * k + 1]));
                }
                tc_fence_before();
                mbar_arrive_warp(o_empty + part);
                // the previous store of this warp must have finished reading staging
                if (lane == 0) tma_store_wait_read_all();
                __syncwarp();
#pragma unroll
                for (int c = 0; c < 16; c++) {   // 16-byte chunk c of the 256-byte row
                    const int pn = c >> 3, pos = (c & 7) ^ (lane & 7);
                    *reinterpret_cast<uint4 *>(stg + pn * 4096 + lane * 128 + pos * 16) =
                        make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    const CUtensorMap *map = part == 0 ? &tmZs : &tmKs;
                    for (int pn = 0; pn < 2; pn++)
                        tma_store_4d(map, stg + pn * 4096, pn * 64, up, mt * 128 + wq * 32, bh);
                    tma_store_commit();
                }
            }
        }
        if (lane == 0) tma_store_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// =====================================================================
// host side
// =====================================================================
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// bf16 tensor map, 128-byte swizzle; dims innermost first, strides in bytes for dims 1..rank-1
bool make_map(CUtensorMap *m, const void *base, int rank, const uint64_t *dims,
              const uint64_t *strides, const uint32_t *box,
              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(base),
              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int b2_padded(int b2) { return (b2 + 15) / 16 * 16; }

int qbar_tiles(const Problem &p) { return (p.tiles * p.b2 + 127) / 128; }
size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

uint32_t rstep_smem(int b2p, int nmt) {
    switch (b2p) {
#define MONARCH_RS_CASE(V) \
    case V: return RsLayout<V>::smem(nmt);
        MONARCH_RS_CASE(16) MONARCH_RS_CASE(32) MONARCH_RS_CASE(48) MONARCH_RS_CASE(64)
        MONARCH_RS_CASE(80) MONARCH_RS_CASE(96) MONARCH_RS_CASE(112) MONARCH_RS_CASE(128)
#undef MONARCH_RS_CASE
    }
    return 0xFFFFFFFFu;
}

struct TcWorkspace {
    __nv_bfloat16 *qbar, *ktil, *z;
    uint4 *hx;   // [BH][t][b2][b1] rows of 32 bytes
};

TcWorkspace carve(const Problem &p, void *base) {
    const size_t mpad = (size_t)qbar_tiles(p) * 128;
    const size_t kz = (size_t)p.BH * p.tiles * p.N * kD * 2;
    char *c = (char *)base;
    TcWorkspace ws;
    ws.qbar = (__nv_bfloat16 *)c;
    c += al256((size_t)p.BH * mpad * kD * 2);
    ws.ktil = (__nv_bfloat16 *)c;
    c += al256(kz);
    ws.z = (__nv_bfloat16 *)c;
    c += al256(kz);
    ws.hx = (uint4 *)c;
    return ws;
}

template <typename K>
cudaError_t set_smem(K kernel, uint32_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int B2P>
cudaError_t launch_rstep(const CUtensorMap *maps, const RsArgs &a, int grid, cudaStream_t s) {
    const uint32_t smem = RsLayout<B2P>::smem(a.nmt);
    cudaError_t e = set_smem(tc_rstep_kernel<B2P>, smem);
    if (e != cudaSuccess) return e;
    tc_rstep_kernel<B2P><<<grid, 384, smem, s>>>(maps[0], maps[1], maps[2], maps[3], maps[4],
                                                   maps[5], a);
    return cudaGetLastError();
}

int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

}  // namespace

bool sm100_supports(const Problem &p, monarch_dtype dtype) {
    if (dtype != MONARCH_BF16 || p.d != kD || p.iters != 1 || p.b2 > 128) return false;
    if (rstep_smem(b2_padded(p.b2), qbar_tiles(p)) > (uint32_t)kMaxSmem) return false;
    // TMA coordinates are 32-bit: every row index must fit
    if ((int64_t)p.BH * p.tiles * p.N + 256 >= (1LL << 31)) return false;
    if ((int64_t)p.BH * qbar_tiles(p) * 128 >= (1LL << 31)) return false;

    if (encode_fn() == nullptr) return false;
    return true;
}

size_t sm100_workspace_bytes(const Problem &p, bool &overflow) {
    overflow = false;
    const size_t mpad = (size_t)qbar_tiles(p) * 128;
    const size_t kz = (size_t)p.BH * p.tiles * p.N * kD * 2;
    const size_t hx = (size_t)p.BH * p.tiles * p.N * 32;
    return al256((size_t)p.BH * mpad * kD * 2) + 2 * al256(kz) + al256(hx);
}

cudaError_t sm100_forward(const Problem &p, const void *q, const void *k, const void *v,
                          void *out, void *workspace, int *status, long long wait_limit,
                          int stall, cudaStream_t stream) {
    const TcWorkspace ws = carve(p, workspace);
    const int nmt = qbar_tiles(p), mpad = nmt * 128, b2p = b2_padded(p.b2);
    const float c_log2 = p.scale * kLog2e;

    // S1
    {
        const int nchunk = (p.b2 * kD / 8 + 127) / 128;
        ProfileScope scope(K_TC_QBAR, stream);
        tc_qbar_kernel<<<(p.head_end() - p.head_begin()) * p.tiles * nchunk, 128, 0, stream>>>(
            (const __nv_bfloat16 *)q, ws.qbar, p, mpad);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    // S2
    {
        CUtensorMap maps[6];
        const uint64_t dq[2] = {(uint64_t)kD, (uint64_t)p.BH * mpad};
        const uint64_t dkv[2] = {(uint64_t)kD, (uint64_t)p.BH * p.N};
        const uint64_t s2[1] = {kD * 2};
        const uint32_t bq[2] = {64, 128};
        const uint32_t bkv[2] = {64, (uint32_t)b2p};
        const uint64_t dst[4] = {(uint64_t)kD, (uint64_t)p.b1, (uint64_t)p.tiles * p.b2,
                                 (uint64_t)p.BH};
        const uint64_t sst[3] = {kD * 2, (uint64_t)p.b1 * kD * 2,
                                 (uint64_t)p.tiles * p.b2 * p.b1 * kD * 2};
        const uint32_t bst[4] = {64, 1, 32, 1};
        if (!make_map(&maps[0], ws.qbar, 2, dq, s2, bq) || !make_map(&maps[1], k, 2, dkv, s2, bkv) ||
            !make_map(&maps[2], v, 2, dkv, s2, bkv) || !make_map(&maps[3], ws.z, 4, dst, sst, bst) ||
            !make_map(&maps[4], ws.ktil, 4, dst, sst, bst))
            return cudaErrorInvalidValue;
        // entropy panels, [bh][t*b2 rows][b1][16], stored 32 rows x 32 B per warp
        const uint64_t dhx[4] = {16, (uint64_t)p.b1, (uint64_t)p.tiles * p.b2, (uint64_t)p.BH};
        const uint64_t shx[3] = {32, (uint64_t)p.b1 * 32, (uint64_t)p.tiles * p.b2 * p.b1 * 32};
        const uint32_t bhx[4] = {16, 1, 32, 1};
        if (!make_map(&maps[5], ws.hx, 4, dhx, shx, bhx, CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
        const int total = (p.head_end() - p.head_begin()) * p.b1;
        const int sms = sm_count();
        const int bpc = (total + sms - 1) / sms;
        const int grid = (total + bpc - 1) / bpc;
        RsArgs a{p, nmt, mpad, bpc, c_log2, status, wait_limit, stall};
        ProfileScope scope(K_TC_RSTEP, stream);
        cudaError_t e = cudaErrorInvalidValue;
        switch (b2p) {
            case 16: e = launch_rstep<16>(maps, a, grid, stream); break;
            case 32: e = launch_rstep<32>(maps, a, grid, stream); break;
            case 48: e = launch_rstep<48>(maps, a, grid, stream); break;
            case 64: e = launch_rstep<64>(maps, a, grid, stream); break;
            case 80: e = launch_rstep<80>(maps, a, grid, stream); break;
            case 96: e = launch_rstep<96>(maps, a, grid, stream); break;
            case 112: e = launch_rstep<112>(maps, a, grid, stream); break;
            case 128: e = launch_rstep<128>(maps, a, grid, stream); break;
        }
        if (e != cudaSuccess) return e;
    }
    // S3
    {
        CUtensorMap maps[4];
        const uint64_t dq[3] = {(uint64_t)kD, (uint64_t)p.b2, (uint64_t)p.BH * p.b1};
        const uint64_t sq[2] = {kD * 2, (uint64_t)p.b2 * kD * 2};
        const uint32_t bq[3] = {64, 1, 128};
        const uint64_t dk[2] = {(uint64_t)kD, (uint64_t)p.BH * p.tiles * p.N};
        const uint64_t sk[1] = {kD * 2};
        const uint32_t bk[2] = {64, 128};
        const uint64_t dh[2] = {16, (uint64_t)p.BH * p.tiles * p.N};
        const uint64_t sh[1] = {32};
        const uint32_t bh[2] = {16, 128};
        if (!make_map(&maps[0], q, 3, dq, sq, bq) || !make_map(&maps[1], ws.ktil, 2, dk, sk, bk) ||
            !make_map(&maps[2], ws.z, 2, dk, sk, bk) ||
            !make_map(&maps[3], ws.hx, 2, dh, sh, bh, CU_TENSOR_MAP_SWIZZLE_32B))
            return cudaErrorInvalidValue;
        const int nq_max = tile_max_rows(p.b1, p.tiles);
        const int npairs = ((nq_max + 127) / 128 + 1) / 2;
        const int nprob = (p.unit_end - p.unit_begin) * p.b2 * npairs;
        LsArgs a{p, (p.b1 + 127) / 128, npairs, nprob, p.unit_begin * p.b2 * npairs, c_log2,
                 (__nv_bfloat16 *)out, status, wait_limit, stall};
        cudaError_t e = set_smem(tc_lstep_kernel, ls::kSmem);
        if (e != cudaSuccess) return e;
        const int grid = nprob < sm_count() ? nprob : sm_count();
        ProfileScope scope(K_TC_LSTEP, stream);
        tc_lstep_kernel<<<grid, ls::kThreads, ls::kSmem, stream>>>(maps[0], maps[1], maps[2],
                                                                   maps[3], a);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace monarch
