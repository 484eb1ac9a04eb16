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
//                       Z and Ktil leave through TMA stores in the R-step's own
//                       order, [bh][u'][panel][g*b2+v][64 columns]: each warp's
//                       32 rows of a 64-column panel are one contiguous 4 KB box
//                       (rows past t*b2 are clipped).  The L-step gathers the
//                       Monarch permutation back: 128 blocks u' of one row (g, v)
//                       per 5-D box.
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
#include "monarch_tc_shared.cuh"
#include "tc_primitives.cuh"

#include <mutex>

namespace monarch {
namespace tcs {

using namespace tc;

// =====================================================================
// S1: aggregated queries
// =====================================================================
// Block: 512 threads = 4 row groups x 128 column threads.  Column thread c owns
// 8 consecutive elements of the flattened (v, d) row; row group r sums a quarter
// of the tile's rows, so four times as many 16-byte loads are in flight as with
// one thread per column (the kernel is bound by memory latency, not bandwidth,
// with B*H*t*ceil(b2*d/1024) blocks).  The four partial sums meet in shared
// memory in a fixed order.
constexpr int kQbarGroups = 4;
__global__ void __launch_bounds__(128 * kQbarGroups, 2) tc_qbar_kernel(
    const __nv_bfloat16 *__restrict__ q, __nv_bfloat16 *__restrict__ qbar, Problem p, int mpad,
    int pack) {
    __shared__ float part[kQbarGroups - 1][8][128];
    const int row_elems = p.b2 * kD;
    const int nchunk = (row_elems / 8 + 127) / 128;
    const int chunk = blockIdx.x % nchunk;
    const int grp = threadIdx.x >> 7, tid = threadIdx.x & 127;
    // every tile of the heads that the unit range touches (the R-step reads all
    // of a head's aggregated rows, padding included)
    // with key-column tiles one block per (head, chunk) aggregates all b1 rows
    // and writes the mean to the t rows v*t + g' of column v
    const int upb = p.key_tiles ? 1 : p.tiles;
    const int bhg = blockIdx.x / nchunk + p.head_begin() * upb;
    const int g = bhg % upb, bh = bhg / upb;
    const int col = (chunk * 128 + tid) * 8;
    const int u0 = unit_row_begin(p, g), u1 = unit_row_end(p, g);
    // rows [r0, r1) of this group: a contiguous quarter of the tile
    const int n = u1 - u0;
    const int r0 = u0 + (grp * n) / kQbarGroups, r1 = u0 + ((grp + 1) * n) / kQbarGroups;
    const bool active = col < row_elems;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; i++) acc[i] = 0.f;
    if (active) {
        // element (u, v, j) of the head: token u*b2 + v; col = v*d + j
        const int64_t ts = tok_stride(p);
        const int64_t stride = p.b2 * ts / 8;   // one block row u, in 16-byte units
        const uint4 *src = reinterpret_cast<const uint4 *>(
            q + head_base(p, bh, p.N) + (int64_t)r0 * p.b2 * ts + (col / kD) * ts + col % kD);
        int u = r0;
        for (; u + 8 <= r1; u += 8) {   // eight independent 16-byte loads in flight
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
        for (; u < r1; u++) {
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
    }
    if (grp > 0) {
#pragma unroll
        for (int i = 0; i < 8; i++) part[grp - 1][i][tid] = acc[i];
    }
    __syncthreads();
    if (grp == 0 && active) {
#pragma unroll
        for (int r = 0; r < kQbarGroups - 1; r++)
#pragma unroll
            for (int i = 0; i < 8; i++) acc[i] += part[r][i][tid];
        const float inv = 1.f / (float)n;
        uint4 o;
        uint32_t *ow = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
        for (int i = 0; i < 4; i++) ow[i] = pack_bf16(acc[2 * i] * inv, acc[2 * i + 1] * inv);
        // the R-step's packed tile (pack > 1) repeats the rows in each segment of
        // 128 / pack rows
        const int pseg = 128 / pack;
        for (int sg = 0; sg < pack; sg++) {
            __nv_bfloat16 *seg = qbar + ((int64_t)bh * mpad + (int64_t)sg * pseg) * kD;
            if (p.key_tiles) {
                const int v = col / kD, j = col % kD;
                for (int gk = 0; gk < p.tiles; gk++)
                    *reinterpret_cast<uint4 *>(seg + ((int64_t)v * p.tiles + gk) * kD + j) = o;
            } else {
                *reinterpret_cast<uint4 *>(seg + (int64_t)g * p.b2 * kD + col) = o;
            }
        }
    }
    if (g == 0 && grp == 0) {
        // zero the padding rows of this head: [t*b2, mpad), or [t*b2, 128 / pack) of
        // every segment of a packed tile
        const int nseg = pack > 1 ? pack : 1;
        const int seglen = pack > 1 ? 128 / pack : mpad;
        for (int sg = 0; sg < nseg; sg++) {
            const int64_t pad = (int64_t)(seglen - p.tiles * p.b2) * kD;
            __nv_bfloat16 *base =
                qbar + ((int64_t)bh * mpad + (int64_t)sg * seglen + (int64_t)p.tiles * p.b2) * kD;
            for (int64_t e = col; e < pad; e += (int64_t)nchunk * 128 * 8)
                *reinterpret_cast<uint4 *>(base + e) = make_uint4(0, 0, 0, 0);
        }
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
// producer of Z; warp 15: the producer of the query tiles.  setmaxnreg gives the
// softmax warpgroups 136 registers, the epilogue 128 and the producer warpgroup
// 112 (the MMA issuer keeps two cursors over the problems).  The keys are
// consumed in halves of 64: one 128-key chunk of Ktil and Z in shared memory
// serves two halves.
// Tensor memory: S_t,0 | S_t,1 (64 columns each, the two S buffers of tile t)
// at t*128, then O_0 | O_1 (128 columns each); P of a half overwrites the first
// 32 columns of its S buffer as packed bfloat16 pairs.
// =====================================================================
namespace ls {
constexpr int kThreads = 512;
constexpr int kSoftmaxRegs = 136, kEpilogueRegs = 128, kProducerRegs = 112;
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

// What one launch of the L-step kernel computes (mode):
//   kLsOut   the L-step with the output.  M side: the query rows (u, v), u in
//            T_g (a strided gather); N side: the Ktil rows [g][v][u'] with their
//            entropy panels; values: Z.  Writes the rows of Y.
//   kLsStat  (iterations before the last) the same logits without the products
//            with Z: writes each query row's log-sum-exp lam (raw logit units,
//            i.e. of S = q.Ktil + H') as a panel row [-lam_hi, -lam_lo, 0...].
//   kLsAgg   (query re-aggregation for the next R-step) the roles transposed:
//            M side: the Ktil rows u' of (g, v); N side and values: the query rows
//            (u, v), u in T_g, with the panels of -lam.  The row softmax over u of
//            q.Ktil[u'] - lam(u) (the entropy of block u' is constant along the row
//            and cancels) is L_v[u, u'] / sum_u L_v[u, u'], so the output row is the
//            aggregated query qbar[g][v][u'], written to the per-block buffer
//            [bh][u'][g*b2 + v][d] that the next R-step reads.
struct LsArgs {
    Problem p;
    int mode;
    int npairs;     // pairs of 128-row M tiles per (g, v)
    int nprob;      // problems of the unit range: units * b2 * npairs
    int prob0;      // first problem: unit_begin * b2 * npairs
    int mpad;       // kLsAgg: rows per block of the per-block aggregated queries
    float c_log2;   // (1/sqrt(d)) * log2(e)
    __nv_bfloat16 *out;   // kLsOut: Y; kLsAgg: aggregated queries [BH][b1][mpad][d]
    uint4 *lam;           // kLsStat: lam panels [BH][N] rows of 32 bytes
    int *status;
    long long limit;
    int stall;      // test hook: the MMA warp first waits on a barrier nothing completes
};

// One problem: (bh, g, v) and a pair of 128-row M tiles.  M rows m = m_first +
// t*128 + r are valid below m_end; the 3-D tensor maps take coordinates (x, y, z).
struct LsProblem {
    int bh, g, v;
    int m_y, m_z, m_first, m_end;   // M side: tile t starts at z = m_z + t*128
    int n_y, n_z, nkeys, nch;       // N side: chunk j starts at z = n_z + j*128
    int nh;                         // 64-key halves of the N side (the softmax's unit)
};

template <int MODE>
__device__ __forceinline__ LsProblem ls_problem(const LsArgs &a, int unit) {
    const Problem &p = a.p;
    LsProblem q;
    unit += a.prob0;
    const int pair = unit % a.npairs;
    unit /= a.npairs;
    if (MODE == kLsOut && p.key_tiles) {
        // key-column tiles: (bh, v) and a pair of tiles of all b1 query rows; the
        // keys are the t*slab rows of the q̄ rows v*t .. v*t + t - 1 of head bh
        const int slab = key_slab(p);
        q.v = unit % p.b2;
        q.bh = unit / p.b2;
        q.g = 0;
        q.m_y = q.v;
        q.m_first = 256 * pair;
        q.m_z = q.bh * p.b1 + q.m_first;
        q.m_end = p.b1;
        q.n_y = 0;
        q.n_z = ((q.bh * p.tiles * p.b2) + q.v * p.tiles) * slab;
        q.nkeys = p.tiles * slab;
        q.nch = (q.nkeys + 127) / 128;
        q.nh = (q.nkeys + 63) / 64;
        return q;
    }
    q.v = unit % p.b2;
    unit /= p.b2;
    q.g = unit % p.tiles;
    q.bh = unit / p.tiles;
    const int u_lo = tile_begin(q.g, p.b1, p.tiles), u_hi = tile_begin(q.g + 1, p.b1, p.tiles);
    const int slab = ((q.bh * p.tiles + q.g) * p.b2 + q.v) * p.b1k;   // Ktil row of block 0
    if (MODE != kLsAgg) {
        q.m_y = q.v;
        q.m_first = u_lo + 256 * pair;
        q.m_z = q.bh * p.b1 + q.m_first;
        q.m_end = u_hi;
        q.n_y = 0;
        q.n_z = slab;
        q.nkeys = p.b1k;
    } else {
        q.m_y = 0;
        q.m_first = 256 * pair;
        q.m_z = slab + q.m_first;
        q.m_end = p.b1k;
        q.n_y = q.v;
        q.n_z = q.bh * p.b1 + u_lo;
        q.nkeys = u_hi - u_lo;
    }
    q.nch = (q.nkeys + 127) / 128;
    q.nh = (q.nkeys + 63) / 64;
    return q;
}

// One TMA tile load of the L-step: a 3-D gather (x, y, z) or a 2-D row box (x, z).
__device__ __forceinline__ void ls_load(void *dst, const CUtensorMap *map, bool gather, int x,
                                        int y, int z, uint64_t *bar) {
    if (gather)
        tma_load_3d(dst, map, x, y, z, bar);
    else
        tma_load_2d(dst, map, x, z, bar);
}

template <int MODE>
__global__ void __launch_bounds__(ls::kThreads, 1)
tc_lstep_kernel(const __grid_constant__ CUtensorMap tmM, const __grid_constant__ CUtensorMap tmN,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmX,
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
    uint64_t *q_full = bars + 0;     // [2 tiles]: M tile loaded
    uint64_t *q_empty = bars + 2;    // [2 tiles]: the tile's last S MMA of a problem done
    uint64_t *k_full = bars + 4;     // [2 stages]: N chunk and its panel
    uint64_t *k_empty = bars + 6;    // [2 stages]: both S MMAs of the chunk done
    uint64_t *z_full = bars + 8;     // [2 stages]: value chunk
    uint64_t *z_empty = bars + 10;   // [2 stages]: both PV MMAs of the chunk done
    uint64_t *s_full = bars + 12;    // [2 tiles][2 S buffers]: S of a 64-key half
    uint64_t *p_full = bars + 16;    // [2 tiles][2 S buffers], one arrival per softmax warp
    uint64_t *o_full = bars + 20;    // [2 tiles]: the last PV MMA of a problem done
    uint64_t *o_free = bars + 22;    // [2 tiles], one arrival per epilogue warp: O_t read
    uint64_t *l_full = bars + 24;    // [2 tiles], one arrival per softmax warp: row sums written
    uint64_t *mma_done = bars + 26;
    uint64_t *stall_bar = bars + 27;   // never completed (fault-injection hook)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 28);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 29);
    uint64_t *pv_done = bars + 30;   // [2 tiles]: one phase per PV MMA of the tile
    float *lsum = reinterpret_cast<float *>(sm + ls::kL);   // [2][2][128]

    const Problem &p = a.p;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nmine = a.nprob > (int)blockIdx.x
                          ? (a.nprob - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    constexpr bool values = MODE != kLsStat;   // products with the values (Z or the queries)
    // the strided query gather (3-D map) is the M side, or in kLsAgg the N side;
    // the other side reads contiguous rows (2-D map)
    constexpr bool n_gather = MODE == kLsAgg;

    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; t++) {
            mbar_init(q_full + t, 1);
            mbar_init(q_empty + t, 1);
            mbar_init(k_full + t, 1);
            mbar_init(k_empty + t, 2);   // one commit per tile's MMA issuer
            mbar_init(z_full + t, 1);
            mbar_init(z_empty + t, 2);   // one commit per tile's MMA issuer
            for (int b = 0; b < 2; b++) {
                mbar_init(s_full + 2 * t + b, 1);
                mbar_init(p_full + 2 * t + b, 4);   // one arrival per softmax warp
            }
            mbar_init(pv_done + t, 1);
            mbar_init(o_full + t, 1);
            mbar_init(o_free + t, 4);   // one arrival per epilogue warp
            mbar_init(l_full + t, 4);   // one arrival per softmax warp
        }
        mbar_init(mma_done, 2);   // one commit per MMA issuer
        mbar_init(stall_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // the M side's extra K-step panel, all ones (so its swizzle is moot): times the
    // N side's panel [x_hi, x_lo, 0, ..., 0] it adds x = x_hi + x_lo to every logit
    // of the N row (the entropy H' of a key block, or -lam of a query row)
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
            // ---------------- producer of the N chunks and their panels: per chunk as
            // soon as the S MMAs of two chunks back are done (never behind an M-tile
            // load, which has its own warp)
            int issued[2] = {0, 0}, jc0 = 0;
            bool ok = true;
            for (int pi = 0; ok && pi < nmine; pi++) {
                const LsProblem pr = ls_problem<MODE>(a, blockIdx.x + pi * gridDim.x);
                for (int j = 0; j < pr.nch; j++) {
                    const int jc = jc0 + j, sk = jc & 1;
                    if (jc >= 2 && !wait_warp(k_empty + sk, ((jc >> 1) - 1) & 1, w)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        // rows past nkeys in the ragged last chunk belong to the next
                        // row block (or are zero-filled past the array): masked later
                        mbar_expect_tx(k_full + sk, kTile + ls::kPanelHx);
                        for (int pn = 0; pn < 2; pn++) {
                            if (n_gather)
                                ls_load_q(sm + ls::kK + sk * kTile + pn * kPanel, &tmN, pn * 64,
                                          pr.v, pr.n_z - pr.bh * p.b1 + j * 128, pr.bh, p,
                                          k_full + sk);
                            else
                                ls_load_kz(sm + ls::kK + sk * kTile + pn * kPanel, &tmN, pn,
                                           pr.n_z + j * 128, p, k_full + sk);
                        }
                        ls_load(sm + ls::kHx + sk * ls::kPanelHx, &tmX, n_gather, 0, pr.n_y,
                                pr.n_z + j * 128, k_full + sk);
                    }
                    issued[sk]++;
                }
                jc0 += pr.nch;
            }
            if (lane == 0)   // every issued copy lands before the CTA may exit
                for (int s = 0; s < 2; s++)
                    if (issued[s] > 0) wait_phase_cleanup(k_full + s, (issued[s] - 1) & 1, kCleanupPolls);
        } else if (warp == 14) {
            // ---------------- producer of the M tiles and the values.  Per problem:
            // first the two M tiles (each as soon as its own last S MMA of the
            // previous problem is done), with the next problem's rows prefetched
            // into L2, then the problem's value chunks (each as soon as the PV MMAs
            // of two chunks back are done).  Every wait points at an MMA that the
            // issuers reach without these loads: a tile's last S of the previous
            // problem follows that problem's value chunks in the issue order.
            int qloads = 0, issued_z[2] = {0, 0}, jc0 = 0;
            bool ok = true;
            for (int pi = 0; ok && pi < nmine; pi++) {
                const LsProblem pr = ls_problem<MODE>(a, blockIdx.x + pi * gridDim.x);
                for (int t = 0; t < 2; t++) {
                    if (pi > 0 && !wait_warp(q_empty + t, (pi - 1) & 1, w)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        mbar_expect_tx(q_full + t, kTile);
                        for (int pn = 0; pn < 2; pn++) {
                            if (!n_gather)
                                ls_load_q(sm + ls::kQ + t * kTile + pn * kPanel, &tmM, pn * 64,
                                          pr.v, pr.m_first + t * 128, pr.bh, p, q_full + t);
                            else   // kLsAgg: the Ktil rows are the M side
                                ls_load_kz(sm + ls::kQ + t * kTile + pn * kPanel, &tmM, pn,
                                           pr.m_z + t * 128, p, q_full + t);
                        }
                    }
                }
                if (!ok) break;
                qloads++;
                if (lane == 0 && pi + 1 < nmine) {
                    const LsProblem nx = ls_problem<MODE>(a, blockIdx.x + (pi + 1) * gridDim.x);
                    for (int t = 0; t < 2; t++)
                        for (int pn = 0; pn < 2; pn++) {
                            if (!n_gather && p.layout == kLayoutBNHD)
                                tma_prefetch_5d(&tmM, pn * 64, nx.bh % p.H, nx.v,
                                                nx.m_first + t * 128, nx.bh / p.H);
                            else if (!n_gather)
                                tma_prefetch_5d(&tmM, pn * 64, nx.v, nx.m_first + t * 128,
                                                nx.bh % p.H, nx.bh / p.H);
                            else {
                                int r, u, bh;
                                kz_coords(p, nx.m_z + t * 128, r, u, bh);
                                tma_prefetch_5d(&tmM, 0, r, pn, u, bh);
                            }
                        }
                }
                for (int j = 0; values && j < pr.nch; j++) {
                    const int jc = jc0 + j, st = jc & 1;
                    if (jc >= 2 && !wait_warp(z_empty + st, ((jc >> 1) - 1) & 1, w)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        mbar_expect_tx(z_full + st, kTile);
                        for (int pn = 0; pn < 2; pn++) {
                            if (n_gather)
                                ls_load_q(sm + ls::kZ + st * kTile + pn * kPanel, &tmV, pn * 64,
                                          pr.v, pr.n_z - pr.bh * p.b1 + j * 128, pr.bh, p,
                                          z_full + st);
                            else
                                ls_load_kz(sm + ls::kZ + st * kTile + pn * kPanel, &tmV, pn,
                                           pr.n_z + j * 128, p, z_full + st);
                        }
                    }
                    issued_z[st]++;
                }
                jc0 += pr.nch;
            }
            if (lane == 0) {   // every issued copy lands before the CTA may exit
                for (int t = 0; t < 2; t++)
                    if (qloads > 0) wait_phase_cleanup(q_full + t, (qloads - 1) & 1, kCleanupPolls);
                for (int st = 0; st < 2; st++)
                    if (issued_z[st] > 0)
                        wait_phase_cleanup(z_full + st, (issued_z[st] - 1) & 1, kCleanupPolls);
            }
        } else if (warp == 13 || warp == 15) {
            // ---------------- MMA issuers: warp 13 for tile 0, warp 15 for tile 1, so
            // that one tile's MMAs never queue behind a wait for the other tile's
            // softmax.  The unit is a 64-key half of a 128-key chunk; tile t has two
            // S buffers of 64 columns (tensor-memory columns t*128 + b*64), and half
            // hc (counted over the CTA's problems) uses buffer hc & 1.  Order: S of
            // the first two halves, then per half hc: PV(hc), S(hc + 2).  So the S
            // of the next half is already in its buffer while the softmax works on
            // this one.  S(hc + 2) overwrites the columns that PV(hc) reads as P:
            // tcgen05 MMAs issued by one thread execute in issue order, so it
            // follows PV(hc) without a wait.  Without values (kLsStat) there is no
            // PV: S(hc + 2) waits for the softmax to have read S(hc) (p_full).  The
            // stages of Ktil and Z are released by one commit from each issuer.
            const int t = warp == 13 ? 0 : 1;
            constexpr uint32_t idS = idesc_bf16(128, 64, 0, 0);
            constexpr uint32_t idO = idesc_bf16(128, 128, 0, 1);
            const uint64_t dQ = smem_desc_sw128(smem_u32(sm + ls::kQ + t * kTile), 16, 1024);
            const uint64_t dK = smem_desc_sw128(smem_u32(sm + ls::kK), 16, 1024);
            const uint64_t dZ = smem_desc_sw128(smem_u32(sm + ls::kZ), kPanel, 1024);
            const uint64_t dQx = smem_desc_sw32(smem_u32(sm + ls::kQx));
            const uint64_t dHx = smem_desc_sw32(smem_u32(sm + ls::kHx));
            constexpr uint32_t kTileDesc = kTile >> 4, kHxDesc = ls::kPanelHx >> 4;
            // rows 64..127 of a 128-row stage: 64 rows x 128 B (SW128), 64 rows x
            // 32 B (SW32), in descriptor units of 16 bytes
            constexpr uint32_t kHalfDesc = 64 * 128 >> 4, kHalfHxDesc = 64 * 32 >> 4;
            const uint32_t tS = tmem + t * 128, tO = tmem + 256 + t * 128;
            // fault injection: a wait that can only give up (bounded, then abort)
            bool ok = !a.stall || spin_warp(stall_bar, 0, w);
            // a position in the CTA's sequence of halves: half i of problem pi,
            // global half hc, chunk jc0 + i / 2
            struct Cursor {
                int pi, i, hc, jc0;
                LsProblem pr;
            };
            auto advance = [&](Cursor &c) {
                c.hc++;
                if (++c.i == c.pr.nh) {
                    c.i = 0;
                    c.jc0 += c.pr.nch;
                    if (++c.pi < nmine) c.pr = ls_problem<MODE>(a, blockIdx.x + c.pi * gridDim.x);
                }
            };
            auto issue_s = [&](const Cursor &c) -> bool {
                const int jc = c.jc0 + (c.i >> 1), sk = jc & 1, kh = c.i & 1, b = c.hc & 1;
                if (c.i == 0 && !spin_warp(q_full + t, c.pi & 1, w)) return false;
                if (kh == 0 && !spin_warp(k_full + sk, (jc >> 1) & 1, w)) return false;
                tc_fence_after();
                const uint32_t d = tS + b * 64;
                mma8_ss_k128(d, dQ, dK + sk * kTileDesc + kh * kHalfDesc, idS, 0u);
                mma1_ss_acc(d, dQx, dHx + sk * kHxDesc + kh * kHalfHxDesc, idS);   // + panel value
                mma_commit_warp(s_full + 2 * t + b);
                const bool last = c.i == c.pr.nh - 1;
                if (kh == 1 || last) mma_commit_warp(k_empty + sk);   // this tile read the stage
                if (last) mma_commit_warp(q_empty + t);   // tile t no longer read
                return true;
            };
            auto issue_pv = [&](const Cursor &c) -> bool {
                const int jc = c.jc0 + (c.i >> 1), st = jc & 1, kh = c.i & 1, b = c.hc & 1;
                if (values && kh == 0 && !spin_warp(z_full + st, (jc >> 1) & 1, w)) return false;
                if (!spin_warp(p_full + 2 * t + b, (c.hc >> 1) & 1, w)) return false;
                if (!values) return true;
                // the first PV of a problem overwrites O_t: the epilogue of the
                // previous problem must have read it
                if (c.i == 0 && c.pi > 0 && !spin_warp(o_free + t, (c.pi - 1) & 1, w)) return false;
                tc_fence_after();
                mma4_ts_mn64(tO, tS + b * 64, dZ + st * kTileDesc + kh * kHalfDesc, idO,
                             c.i > 0 ? 1u : 0u);
                mma_commit_warp(pv_done + t);
                const bool last = c.i == c.pr.nh - 1;
                if (kh == 1 || last) mma_commit_warp(z_empty + st);   // this tile read the stage
                if (last) mma_commit_warp(o_full + t);
                return true;
            };
            if (nmine > 0) {
                Cursor cs{0, 0, 0, 0, ls_problem<MODE>(a, blockIdx.x)};   // next S to issue
                Cursor cp = cs;                                          // next PV to issue
                for (int k = 0; ok && k < 2 && cs.pi < nmine; k++) {
                    ok = issue_s(cs);
                    advance(cs);
                }
                while (ok && cp.pi < nmine) {
                    const bool more = cs.pi < nmine;
                    ok = issue_pv(cp) && (!more || issue_s(cs));
                    if (more) advance(cs);
                    advance(cp);
                }
            }
            mma_commit_warp(mma_done);
            wait_phase_cleanup(mma_done, 0, kCleanupPolls);
        }
    } else if (warp >= 8) {
        // ---------------- epilogue warpgroup: per problem and tile, O_t / l to
        // bfloat16 rows of the output (Y, or the aggregated queries)
        regs_dec<ls::kEpilogueRegs>();
        const int wq = warp & 3;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        bool ok = values;
        for (int pi = 0; ok && pi < nmine; pi++) {
            const LsProblem pr = ls_problem<MODE>(a, blockIdx.x + pi * gridDim.x);
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
                const int m0w = pr.m_first + t * 128 + wq * 32;
                // kLsOut: Y row (u, v) = token m*b2 + v of head bh in the call's layout,
                // at obase + (m - m0w) * ostride
                const int64_t ostride = MODE == kLsOut ? (int64_t)p.b2 * tok_stride(p) : 0;
                __nv_bfloat16 *const obase =
                    MODE == kLsOut ? a.out + head_base(p, pr.bh, p.N) +
                                         ((int64_t)m0w * p.b2 + pr.v) * tok_stride(p)
                                   : a.out;
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
                        const int m = m0w + row;
                        if (m < pr.m_end) {
                            // kLsAgg: the aggregated query of block u' = m for row g*b2 + v
                            __nv_bfloat16 *dst =
                                MODE == kLsOut
                                    ? obase + row * ostride
                                    : a.out + (((int64_t)pr.bh * p.b1k + m) * a.mpad +
                                               pr.g * p.b2 + pr.v) * kD;
                            *reinterpret_cast<uint4 *>(dst + hf * 64 + c * 8) = val;
                        }
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
        const uint32_t tS0 = tmem + lane_off + t * 128;   // S buffer b at + b * 64
        const uint32_t tO = tmem + lane_off + 256 + t * 128;
        const uint64_t c2 = f2_pack(a.c_log2, a.c_log2);
        bool ok = true;
        int hc = 0;   // 64-key halves done by this tile over the CTA's problems
        for (int pi = 0; ok && pi < nmine; pi++) {
            const LsProblem pr = ls_problem<MODE>(a, blockIdx.x + pi * gridDim.x);
            float m_run = -INFINITY, l_run = 0.f;
            for (int i = 0; i < pr.nh; i++, hc++) {
                const int b = hc & 1;
                if (!wait_warp(s_full + 2 * t + b, (hc >> 1) & 1, w)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t tS = tS0 + b * 64;
                // S = q.Ktil + H' (kLsAgg: Ktil.q - lam): scaled by c_log2 it is the
                // logit in log2 units, so the maximum is taken on S itself
                float x[64];
                tmem_ld32f(tS, &x[0]);
                tmem_ld32f(tS + 32, &x[32]);
                tmem_wait_ld();
                const int nvalid = pr.nkeys - i * 64;   // N rows of this half inside the row
                if (nvalid < 64) {
                    // the ragged last half: rows past nkeys belong to the next row
                    // block (or are zero fill), so mask them by selection
#pragma unroll
                    for (int k = 0; k < 64; k++) x[k] = k < nvalid ? x[k] : -INFINITY;
                }
                float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int k = 0; k < 32; k++) mx4[k & 3] = fmax3(mx4[k & 3], x[2 * k], x[2 * k + 1]);
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
                uint32_t pk[32];
#pragma unroll
                for (int k = 0; k < 32; k++) {
                    const uint64_t d2 = f2_fma(f2_pack(x[2 * k], x[2 * k + 1]), c2, nmc2);
                    uint64_t e2;
                    constexpr int kEvery = ls::kPolyEvery > 0 ? ls::kPolyEvery : 1;
                    if (ls::kPolyEvery > 0 && (k % kEvery) == kEvery - 1 && nvalid >= 64) {
                        e2 = exp2_poly_x2(d2);
                    } else {
                        float lo, hi;
                        f2_unpack(d2, lo, hi);
                        e2 = f2_pack(fast_exp2(lo), fast_exp2(hi));
                    }
                    sum2[k & 3] = f2_add(sum2[k & 3], e2);
                    float p0, p1;
                    f2_unpack(e2, p0, p1);
                    pk[k] = pack_bf16(p0, p1);
                }
                // P (packed bfloat16 pairs) over the first 32 columns of the buffer
                if (values) tmem_st32(tS, pk);
                float s0, s1;
                f2_unpack(f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3])), s0, s1);
                l_run = l_run * alpha + (s0 + s1);
                if (values && i > 0 && __any_sync(0xffffffffu, rescale)) {
                    // O_t holds the products up to the previous half once PV_t of
                    // that half is done (it may still be running: S of this half
                    // was issued two halves back); then scale it in four slices
                    if (!wait_warp(pv_done + t, (hc - 1) & 1, w)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < 4; c++) {
                        float o[32];
                        tmem_ld32f(tO + c * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 32; k++) o[k] *= alpha;
                        tmem_st32f(tO + c * 32, o);
                    }
                }
                if (values) tmem_wait_st();
                tc_fence_before();
                mbar_arrive_warp(p_full + 2 * t + b);
            }
            if (!ok) break;
            if (values) {
                // the row sums for the epilogue.  Before publishing those of problem
                // pi the epilogue must have taken those of pi - 1 (its o_free
                // arrival follows its l_full wait): otherwise l_full could run two
                // phases ahead of the epilogue's parity wait when problems are short.
                // o_free cannot itself run ahead here, since the epilogue releases
                // problem pi only after these row sums.
                if (pi > 0 && !wait_warp(o_free + t, (pi - 1) & 1, w)) break;
                lsum[((pi & 1) * 2 + t) * 128 + wq * 32 + lane] = l_run;
                mbar_arrive_warp(l_full + t);
            } else {
                // the row's log-sum-exp in raw logit units, stored negated as a
                // bfloat16 pair (hi + lo within 2^-16 relative) in its panel row
                const int m = pr.m_first + t * 128 + wq * 32 + lane;
                if (m < pr.m_end) {
                    const float lam = m_run + fast_log2(l_run) / a.c_log2;
                    const __nv_bfloat16 hi = __float2bfloat16_rn(-lam);
                    const __nv_bfloat16 lo = __float2bfloat16_rn(-lam - __bfloat162float(hi));
                    const uint32_t pair = (uint32_t)__bfloat16_as_ushort(hi) |
                                          ((uint32_t)__bfloat16_as_ushort(lo) << 16);
                    uint4 *dst = a.lam + ((int64_t)pr.bh * p.N + (int64_t)m * p.b2 + pr.v) * 2;
                    dst[0] = make_uint4(pair, 0u, 0u, 0u);
                    dst[1] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
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
    float inv_c_log2;
    // 0: one set of aggregated queries per head (the first iteration, uniform L),
    // loaded once per head; 1: per block u' (later iterations), tile mt of block
    // u' at rows (bh*b1 + u')*mpad + mt*128, loaded per item into slot mt
    int qblk;
    int hdirect;         // 1: entropy panel rows by plain stores (no staging room)
    uint4 *hx;           // entropy panels [BH][t*b2][b1k] rows of 32 bytes (hdirect)
    int *status;
    long long limit;
    int stall;           // test hook: the MMA warp first waits on a barrier nothing completes
    // blocks per item (1, 2 or 4): when the t*b2 aggregated rows fill at most a half
    // (a quarter) of the 128-row tile, the tile holds `pack` copies of them in
    // segments of 128/pack rows, and one item covers `pack` consecutive blocks u':
    // segment s meets the keys of block u' + s (a block-diagonal mask on the logits)
    int pack;
    int gph;             // items (groups of `pack` blocks) per head
    // 1: R enters [Z | Ktil] = R [V | K] as two bfloat16 parts, R_hi + R_lo with
    // R_lo = R - R_hi rounded again (R to about 2^-16), in two passes of the TS
    // MMAs (the backward's recompute of the forward uses it)
    int split;
};
constexpr int kMaxQbarTiles = 4;   // slots of the per-block aggregated-query ring

template <int B2P>
struct RsLayout {
    static constexpr uint32_t kStage = 4 * B2P * 128;   // K and V: 2 panels each of B2P x 128 B
    static constexpr uint32_t kVOff = 2 * B2P * 128;    // V inside a stage
    static constexpr uint32_t kPanelKV = B2P * 128;
    __host__ __device__ static uint32_t kv(int nmt) { return (uint32_t)nmt * kTile; }
    // two stages, each the K and V panels of `pack` blocks
    __host__ __device__ static uint32_t stg(int nmt, int pack) {
        return kv(nmt) + 2 * kStage * (uint32_t)pack;
    }
    // entropy-panel staging of the softmax warps: 4 warps x 32 rows x 32 B, when
    // it fits (hdirect = 0); otherwise each softmax thread stores its panel row
    // with plain stores (hdirect = 1, no staging)
    __host__ __device__ static uint32_t hstg(int nmt, int pack) { return stg(nmt, pack) + 4 * 8192; }
    __host__ __device__ static uint32_t bar(int nmt, int hdirect, int pack) {
        return hstg(nmt, pack) + (hdirect ? 0 : 4 * 1024);
    }
    __host__ __device__ static uint32_t smem(int nmt, int hdirect, int pack) {
        return bar(nmt, hdirect, pack) + 256 + 1024;
    }
};

// SPLIT (the backward's recompute): R enters the TS products as R_hi + R_lo.  A
// template parameter, so that the forward's kernel carries none of it.
template <int B2P, int SPLIT>
__global__ void __launch_bounds__(384, 1)
tc_rstep_kernel(const __grid_constant__ CUtensorMap tmQb, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmZs,
                const __grid_constant__ CUtensorMap tmKs, const __grid_constant__ CUtensorMap tmHs,
                RsArgs a) {
    using L = RsLayout<B2P>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    const int nmt = a.nmt;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::bar(nmt, a.hdirect, a.pack));
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
    uint64_t *qs_full = bars + 20;     // [kMaxQbarTiles] per-block mode: slot mt loaded
    uint64_t *qs_empty = bars + 24;    // [kMaxQbarTiles] per-block mode: slot mt's S MMA done

    const Problem &p = a.p;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // (head, group of `pack` blocks) items of the heads that the unit range touches
    const int pack = a.pack, pseg = 128 / pack;
    const uint32_t kstage = L::kStage * pack, kpanel = L::kPanelKV * pack, kvoff = L::kVOff * pack;
    const int total = p.head_end() * a.gph;
    const int first = p.head_begin() * a.gph + blockIdx.x * a.bpc;
    const int nblk = min(a.bpc, total - first);
    const int nitems = nblk * nmt;

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
        for (int s = 0; s < kMaxQbarTiles; s++) {
            mbar_init(qs_full + s, 1);
            mbar_init(qs_empty + s, 1);
        }
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
        // ---------------- producer: qbar tiles per head (or per block), K and V per block
        if (lane == 0) {
            int heads = 0, cur = -1, issued[2] = {0, 0}, qissued[kMaxQbarTiles] = {0, 0, 0, 0};
            bool ok = true;
            for (int ib = 0; ib < nblk && ok; ib++) {
                const int fb = first + ib, bh = fb / a.gph, up = (fb % a.gph) * pack;
                if (a.qblk) {
                    // slot mt takes tile mt of this block once the S MMA of the
                    // previous block's tile mt is done
                    for (int mt = 0; mt < nmt && ok; mt++) {
                        if (ib >= 1 && !wait_phase(qs_empty + mt, (ib - 1) & 1, w)) {
                            ok = false;
                            break;
                        }
                        mbar_expect_tx(qs_full + mt, kTile);
                        for (int pn = 0; pn < 2; pn++)
                            tma_load_2d(sm + mt * kTile + pn * kPanel, &tmQb, pn * 64,
                                        fb * a.mpad + mt * 128, qs_full + mt);
                        qissued[mt]++;
                    }
                    if (!ok) break;
                } else if (bh != cur) {
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
                uint8_t *stage = sm + L::kv(nmt) + st * kstage;
                mbar_expect_tx(kv_full + st, kstage);
                // the b2 tokens of each block of the group, head bh: (x, token, head,
                // batch), or (x, head, token, batch) for [B][N][H][d] (increasing
                // strides); block s at row s*B2P of each panel.  A block past b1k
                // (the head's last group) reads zeros: every row stays finite.
                const bool bnhd = p.layout == kLayoutBNHD;
                const int hh = bh % p.H, bb = bh / p.H;
                for (int sg = 0; sg < pack; sg++) {
                    const int tok0 = (up + sg) * p.b2;
                    const int c1 = bnhd ? hh : tok0, c2 = bnhd ? tok0 : hh;
                    for (int pn = 0; pn < 2; pn++) {
                        tma_load_4d(stage + pn * kpanel + sg * L::kPanelKV, &tmK, pn * 64, c1, c2,
                                    bb, kv_full + st);
                        tma_load_4d(stage + kvoff + pn * kpanel + sg * L::kPanelKV, &tmV, pn * 64,
                                    c1, c2, bb, kv_full + st);
                    }
                }
                issued[st]++;
            }
            if (heads > 0) wait_phase_cleanup(q_full, (heads - 1) & 1, kCleanupPolls);
            for (int s = 0; s < 2; s++)
                if (issued[s] > 0)
                    wait_phase_cleanup(kv_full + s, (issued[s] - 1) & 1, kCleanupPolls);
            for (int mt = 0; mt < kMaxQbarTiles; mt++)   // the last load into each slot
                if (qissued[mt] > 0)
                    wait_phase_cleanup(qs_full + mt, (qissued[mt] - 1) & 1, kCleanupPolls);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer: the whole warp runs the loop, one elected
        // lane issues each MMA (see mma_ss_warp)
        {
            const uint32_t id1 = idesc_bf16(128, B2P * pack, 0, 0);
            constexpr uint32_t id2 = idesc_bf16(128, 128, 0, 1);
            const uint64_t dQ = smem_desc_sw128(smem_u32(sm), 16, 1024);
            const uint64_t dK = smem_desc_sw128(smem_u32(sm + L::kv(nmt)), 16, 1024);
            const uint64_t dV = smem_desc_sw128(smem_u32(sm + L::kv(nmt)), kpanel, 1024);
            int heads = 0;
            // fault injection: a wait that can only give up (bounded, then abort)
            bool ok = !a.stall || spin_warp(stall_bar, 0, w);
            // S = qbar_mt K_u'^T for item i into S buffer i & 1
            auto gemm1 = [&](int i) -> bool {
                const int ib = i / nmt, mt = i % nmt;
                const int fb = first + ib, bh = fb / a.gph;
                if (a.qblk) {
                    if (!wait_warp(qs_full + mt, ib & 1, w)) return false;
                } else if (mt == 0 && (ib == 0 || (fb - 1) / a.gph != bh)) {
                    if (!wait_warp(q_full, heads & 1, w)) return false;
                    heads++;
                }
                if (mt == 0 && !wait_warp(kv_full + (ib & 1), (ib >> 1) & 1, w)) return false;
                if (i >= 2 && !wait_warp(s_free + (i & 1), ((i >> 1) - 1) & 1, w)) return false;
                tc_fence_after();
                const uint64_t a0 = desc_plus(dQ, mt * kTile);
                const uint64_t b0 = desc_plus(dK, (ib & 1) * kstage);
#pragma unroll
                for (int kk = 0; kk < 8; kk++)
                    mma_ss_warp(tmem + (i & 1) * 128,
                           desc_plus(a0, (kk >> 2) * kPanel + (kk & 3) * 32),
                           desc_plus(b0, (kk >> 2) * kpanel + (kk & 3) * 32), id1, kk > 0);
                mma_commit_warp(s_full + (i & 1));
                if (a.qblk) {
                    mma_commit_warp(qs_empty + mt);   // slot mt may take the next block's tile
                } else {
                    const bool head_ends = (ib == nblk - 1) || ((fb + 1) / a.gph != bh);
                    if (mt == nmt - 1 && head_ends) mma_commit_warp(q_empty);
                }
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
                const uint64_t bz = desc_plus(dV, (ib & 1) * kstage + kvoff);
                const uint64_t bk = desc_plus(dV, (ib & 1) * kstage);
                if (i > 0 && !wait_warp(o_empty + 0, (i - 1) & 1, w)) break;
                tc_fence_after();
                // K = pack * B2P: the packed blocks' P columns (zero outside a row's
                // own segment) against their V (then K) rows
                for (int kk = 0; kk < (B2P / 16) * pack; kk++)
                    mma_ts_warp(tmem + 256, pa + kk * 8, desc_plus(bz, kk * 2048), id2, kk > 0 ? 1u : 0u);
                if constexpr (SPLIT != 0) {   // the low parts, (B2P / 16) * pack * 8 columns on
                    const int nks = (B2P / 16) * pack;
                    for (int kk = 0; kk < nks; kk++)
                        mma_ts_warp(tmem + 256, pa + (nks + kk) * 8, desc_plus(bz, kk * 2048), id2, 1u);
                }
                mma_commit_warp(o_full + 0);
                if (i > 0 && !wait_warp(o_empty + 1, (i - 1) & 1, w)) break;
                tc_fence_after();
                for (int kk = 0; kk < (B2P / 16) * pack; kk++)
                    mma_ts_warp(tmem + 384, pa + kk * 8, desc_plus(bk, kk * 2048), id2, kk > 0 ? 1u : 0u);
                if constexpr (SPLIT != 0) {
                    const int nks = (B2P / 16) * pack;
                    for (int kk = 0; kk < nks; kk++)
                        mma_ts_warp(tmem + 384, pa + (nks + kk) * 8, desc_plus(bk, kk * 2048), id2, 1u);
                }
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
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        // this thread's row: segment sg of the tile (block up + sg of the group) and
        // its aggregated-query row qrow (packed tiles: every segment repeats rows
        // 0 .. pseg - 1; otherwise mt * 128 + the tile row)
        const int trow = wq * 32 + lane, sg = trow / pseg;
        for (int i = 0; i < nitems; i++) {
            const int ib = i / nmt, mt = i % nmt;
            const int fb = first + ib, bh = fb / a.gph, up = (fb % a.gph) * pack;
            const int qrow = mt * 128 + trow % pseg;
            if (!wait_warp(s_full + (i & 1), (i >> 1) & 1, w)) break;
            tc_fence_after();
            const uint32_t tS = tmem + lane_off + (i & 1) * 128 + sg * B2P;
            // the row's B2P logits (its segment's columns): all TMEM loads in flight
            // together, one wait
            float x[B2P];
#pragma unroll
            for (int c = 0; c < B2P / 16; c++) tmem_ld16f(tS + c * 16, &x[c * 16]);
            tmem_wait_ld();
            if (p.key_tiles || p.b2 < B2P) {   // uniform branch
                // columns outside [lo, hi): the padding past b2, and with key-column
                // tiles the other tiles' columns (row r = v*t + g' of the tile stack
                // takes key tile g').  A large finite logit, not -inf: its
                // probability is exactly 0 and 0 * x stays finite in the entropy sum.
                int lo = 0, hi = p.b2;
                if (p.key_tiles) {   // t <= b2 <= 128: the products fit in 32 bits
                    const int gk = qrow % p.tiles;
                    lo = gk * p.b2 / p.tiles;
                    hi = (gk + 1) * p.b2 / p.tiles;
                }
#pragma unroll
                for (int col = 0; col < B2P; col++) x[col] = col >= lo && col < hi ? x[col] : -1e30f;
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
            // entropy of the row in log2 units, log2(sum 2^x) - E_R[x] = H / ln 2,
            // stored divided by c_log2 = s log2(e) (the L-step's logits are
            // S * c_log2) as a bfloat16 pair hi + lo in the row's entropy panel
            {
                // (l >= 1: the row maximum contributes 2^0, so the approximate
                // log2 is accurate to a few ulp of its result)
                const float hp = (mxr * a.c_log2 + fast_log2(l) - (ea + eb) * inv) * a.inv_c_log2;
                const __nv_bfloat16 hi = __float2bfloat16_rn(hp);
                const __nv_bfloat16 lo = __float2bfloat16_rn(hp - __bfloat162float(hi));
                const uint32_t pair = (uint32_t)__bfloat16_as_ushort(hi) |
                                      ((uint32_t)__bfloat16_as_ushort(lo) << 16);
                if (a.hdirect) {
                    const int row = qrow;
                    if (row < p.tiles * p.b2 && up + sg < p.b1k) {
                        uint4 *dst = a.hx + (((int64_t)bh * p.tiles * p.b2 + row) * key_slab(p) + up + sg) * 2;
                        dst[0] = make_uint4(pair, 0u, 0u, 0u);
                        dst[1] = make_uint4(0u, 0u, 0u, 0u);
                    }
                } else {
                    // the warp's 32 panel rows (32 B each) leave in one TMA store,
                    // which clips the rows past t*b2; the previous item's store must
                    // have finished reading the staging first
                    uint8_t *hs = sm + L::hstg(nmt, pack) + wq * 1024;
                    if (lane == 0) tma_store_wait_read_all();
                    __syncwarp();
                    *reinterpret_cast<uint4 *>(hs + lane * 32) = make_uint4(pair, 0u, 0u, 0u);
                    *reinterpret_cast<uint4 *>(hs + lane * 32 + 16) = make_uint4(0u, 0u, 0u, 0u);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {   // the warp's 32 rows lie in one segment
                        tma_store_4d(&tmHs, hs, 0, up + sg, mt * 128 + (wq * 32) % pseg, bh);
                        tma_store_commit();
                    }
                }
            }
            const uint64_t inv2 = f2_pack(inv, inv);
            // P of the PV MMA: K = pack * B2P bfloat16 values, packed in pairs from
            // the buffer's first column; this row's segment holds R, the others zero
            const uint32_t tP = tmem + lane_off + (i & 1) * 128;
#pragma unroll
            for (int c = 0; c < B2P / 16; c++) {
                uint32_t pk[8];
                if constexpr (SPLIT == 0) {
#pragma unroll
                    for (int k = 0; k < 8; k++) {
                        float p0, p1;
                        f2_unpack(f2_mul(pp[c * 8 + k], inv2), p0, p1);
                        pk[k] = pack_bf16(p0, p1);
                    }
                } else {   // R_lo = R - R_hi, rounded again, pack * B2P / 2 columns on
                    uint32_t pl[8];
#pragma unroll
                    for (int k = 0; k < 8; k++) {
                        float p0, p1;
                        f2_unpack(f2_mul(pp[c * 8 + k], inv2), p0, p1);
                        pk[k] = pack_bf16(p0, p1);
                        pl[k] = pack_bf16(p0 - __uint_as_float(pk[k] << 16),
                                          p1 - __uint_as_float(pk[k] & 0xFFFF0000u));
                    }
                    tmem_st8(tP + pack * (B2P / 2) + sg * (B2P / 2) + c * 8, pl);
                }
                tmem_st8(tP + sg * (B2P / 2) + c * 8, pk);
            }
            if (pack > 1) {
                uint32_t zk[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                for (int s2 = 0; s2 < pack; s2++)
                    if (s2 != sg)
#pragma unroll
                        for (int c = 0; c < B2P / 16; c++) {
                            tmem_st8(tP + s2 * (B2P / 2) + c * 8, zk);
                            if constexpr (SPLIT != 0)
                                tmem_st8(tP + pack * (B2P / 2) + s2 * (B2P / 2) + c * 8, zk);
                        }
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
        uint8_t *stg = sm + L::stg(nmt, pack) + wq * 8192;   // 2 panels x 32 rows x 128 B
        // the warp's 32 rows: segment sgw (block up + sgw), aggregated-query rows
        // from mt * 128 + r0w
        const int sgw = (wq * 32) / pseg, r0w = (wq * 32) % pseg;
        bool ok = true;
        for (int i = 0; ok && i < nitems; i++) {
            const int ib = i / nmt, mt = i % nmt;
            const int fb = first + ib, bh = fb / a.gph, up = (fb % a.gph) * pack;
            for (int part = 0; part < 2; part++) {
                if (!wait_warp(o_full + part, i & 1, w)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t pk[64];
#pragma unroll
                for (int c = 0; c < 4; c += 2) {   // two 32-column loads per wait
                    uint32_t o0[32], o1[32];
                    tmem_ld32(tmem + lane_off + 256 + part * 128 + c * 32, o0);
                    tmem_ld32(tmem + lane_off + 256 + part * 128 + c * 32 + 32, o1);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 16; k++) {
                        pk[c * 16 + k] =
                            pack_bf16(__uint_as_float(o0[2 * k]), __uint_as_float(o0[2 * k + 1]));
                        pk[c * 16 + 16 + k] =
                            pack_bf16(__uint_as_float(o1[2 * k]), __uint_as_float(o1[2 * k + 1]));
                    }
                }
                tc_fence_before();
                mbar_arrive_warp(o_empty + part);
                // each 64-column panel leaves in its own store group from staging
                // slot pn; the group that last read slot pn is two groups back, so
                // one younger group may still be reading while this panel is written
#pragma unroll
                for (int pn = 0; pn < 2; pn++) {
                    if (lane == 0) tma_store_wait_read_le1();
                    __syncwarp();
#pragma unroll
                    for (int c = 0; c < 8; c++) {   // 16-byte chunk c of the panel's 128-byte row
                        const int pos = c ^ (lane & 7);
                        *reinterpret_cast<uint4 *>(stg + pn * 4096 + lane * 128 + pos * 16) =
                            make_uint4(pk[pn * 32 + 4 * c], pk[pn * 32 + 4 * c + 1],
                                       pk[pn * 32 + 4 * c + 2], pk[pn * 32 + 4 * c + 3]);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_5d(part == 0 ? &tmZs : &tmKs, stg + pn * 4096, 0,
                                     mt * 128 + r0w, pn, up + sgw, bh);
                        tma_store_commit();
                    }
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

// Key-column tiles: the key rows u' in [b1k, slab) of every (head, q̄ row) hold
// Ktil = Z = 0 and the entropy panel [-1e30, 0, ...], so that the L-step's logit
// of such a row is -1e30 (its probability exactly 0) and its products stay
// finite.  One thread per 16 bytes: 16 of Ktil, 16 of Z (8 per 64-column panel
// of the [bh][u'][panel][r][64] layout) and 2 of the panel row [bh][r][slab].
__global__ void tc_keypad_kernel(__nv_bfloat16 *__restrict__ ktil, __nv_bfloat16 *__restrict__ z,
                                 uint4 *__restrict__ hx, Problem p) {
    const int slab = key_slab(p), npad = slab - p.b1k;
    const int64_t rows = (int64_t)p.BH * p.tiles * p.b2 * npad;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    const uint32_t neg = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(-1e30f));
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < rows * 34;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t pr = i / 34;
        const int part = (int)(i % 34);
        const int64_t rid = pr / npad;                        // bh * t * b2 + r
        const int up = p.b1k + (int)(pr % npad);              // a padding block row
        const int64_t rows = (int64_t)p.tiles * p.b2;
        const int64_t bh = rid / rows, r = rid % rows;
        if (part < 32) {
            const int pn = (part & 15) >> 3, c = part & 7;  // panel, 16-byte chunk
            const int64_t off = (((bh * slab + up) * 2 + pn) * rows + r) * 64;
            reinterpret_cast<uint4 *>((part < 16 ? ktil : z) + off)[c] = zero;
        } else {
            hx[(rid * slab + up) * 2 + (part - 32)] = part == 32 ? make_uint4(neg, 0u, 0u, 0u) : zero;
        }
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
              const uint64_t *strides, const uint32_t *box, CUtensorMapSwizzle swizzle) {
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

uint32_t rstep_smem(int b2p, int nmt, int hdirect, int pack) {
    switch (b2p) {
#define MONARCH_RS_CASE(V) \
    case V: return RsLayout<V>::smem(nmt, hdirect, pack);
        MONARCH_RS_CASE(16) MONARCH_RS_CASE(32) MONARCH_RS_CASE(48) MONARCH_RS_CASE(64)
        MONARCH_RS_CASE(80) MONARCH_RS_CASE(96) MONARCH_RS_CASE(112) MONARCH_RS_CASE(128)
#undef MONARCH_RS_CASE
    }
    return 0xFFFFFFFFu;
}

// Blocks per R-step item with the shared aggregated queries of the first
// iteration: 4 (2) when the t*b2 rows fit in a quarter (half) of the 128-row tile
// and the stages of that many blocks fit in shared memory, else 1.  (t*b2 <= 64
// implies b2 <= 64, so pack * B2P <= 128: the logits of a group fit one S buffer.)
int rstep_pack(const Problem &p) {
    const int rows = p.tiles * p.b2, b2p = b2_padded(p.b2);
    int pack = rows <= 32 ? 4 : rows <= 64 ? 2 : 1;
    while (pack > 1 && rstep_smem(b2p, 1, 1, pack) > (uint32_t)kMaxSmem) pack /= 2;
    return pack;
}

TcWorkspace carve(const Problem &p, void *base) {
    const size_t mpad = (size_t)qbar_tiles(p) * 128;
    const size_t kz = key_rows(p) * kD * 2;
    char *c = (char *)base;
    TcWorkspace ws;
    ws.qbar = (__nv_bfloat16 *)c;
    c += al256((size_t)p.BH * mpad * kD * 2);
    ws.ktil = (__nv_bfloat16 *)c;
    c += al256(kz);
    ws.z = (__nv_bfloat16 *)c;
    c += al256(kz);
    ws.hx = (uint4 *)c;
    c += al256(key_rows(p) * 32);
    ws.qblk = nullptr;
    ws.lam = nullptr;
    if (p.iters > 1) {
        ws.qblk = (__nv_bfloat16 *)c;
        c += al256((size_t)p.BH * p.b1k * mpad * kD * 2);
        ws.lam = (uint4 *)c;
    }
    return ws;
}

template <int B2P>
cudaError_t launch_rstep(const CUtensorMap *maps, const RsArgs &a, int grid, cudaStream_t s) {
    const uint32_t smem = RsLayout<B2P>::smem(a.nmt, a.hdirect, a.pack);
    if (a.split) {
        cudaError_t e = set_smem(tc_rstep_kernel<B2P, 1>, smem);
        if (e != cudaSuccess) return e;
        tc_rstep_kernel<B2P, 1><<<grid, 384, smem, s>>>(maps[0], maps[1], maps[2], maps[3],
                                                          maps[4], maps[5], a);
    } else {
        cudaError_t e = set_smem(tc_rstep_kernel<B2P, 0>, smem);
        if (e != cudaSuccess) return e;
        tc_rstep_kernel<B2P, 0><<<grid, 384, smem, s>>>(maps[0], maps[1], maps[2], maps[3],
                                                          maps[4], maps[5], a);
    }
    return cudaGetLastError();
}

int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

}  // namespace tcs

using namespace tcs;

bool sm100_supports(const Problem &p, monarch_dtype dtype) {
    if (dtype != MONARCH_BF16 || p.d != kD || p.b2 > 128) return false;
    // key-column tiles: the first iteration's kernels only (later iterations
    // run on the generic kernels)
    if (p.key_tiles && p.iters > 1) return false;
    // later iterations keep one slot per aggregated-query tile
    if (p.iters > 1 && qbar_tiles(p) > kMaxQbarTiles) return false;
    if (p.iters > 1 && (int64_t)p.BH * p.b1k * qbar_tiles(p) * 128 + 256 >= (1LL << 31)) return false;
    if (rstep_smem(b2_padded(p.b2), qbar_tiles(p), 1) > (uint32_t)kMaxSmem) return false;
    // TMA coordinates are 32-bit: every row index must fit
    if ((int64_t)key_rows(p) + 256 >= (1LL << 31)) return false;
    if ((int64_t)p.BH * p.Nk + 256 >= (1LL << 31) || (int64_t)p.BH * p.N + 256 >= (1LL << 31))
        return false;
    if ((int64_t)p.BH * qbar_tiles(p) * 128 >= (1LL << 31)) return false;

    if (encode_fn() == nullptr) return false;
    return true;
}

size_t sm100_workspace_bytes(const Problem &p, bool &overflow) {
    overflow = false;
    const size_t mpad = (size_t)qbar_tiles(p) * 128;
    const size_t kz = key_rows(p) * kD * 2;
    const size_t hx = key_rows(p) * 32;
    size_t bytes = al256((size_t)p.BH * mpad * kD * 2) + 2 * al256(kz) + al256(hx);
    if (p.iters > 1)
        bytes += al256((size_t)p.BH * p.b1k * mpad * kD * 2) + al256((size_t)p.BH * p.N * 32);
    return bytes;
}

namespace tcs {

// bfloat16 tensor maps of the L-step (128-row boxes): rows of a [rows][d] array
// (2-D), the strided query gather (3-D: y = column v, z = bh*b1 + u), and the
// same two forms for 32-byte panel rows.
bool map_rows(CUtensorMap *m, const void *base, uint64_t rows, uint32_t width,
              CUtensorMapSwizzle sw) {
    const uint64_t dims[2] = {width, rows};
    const uint64_t str[1] = {(uint64_t)width * 2};
    const uint32_t box[2] = {width == 16 ? 16u : 64u, 128};
    return make_map(m, base, 2, dims, str, box, sw);
}
bool map_gather(CUtensorMap *m, const void *base, const Problem &p, uint32_t width,
                CUtensorMapSwizzle sw) {
    const uint64_t dims[3] = {width, (uint64_t)p.b2, (uint64_t)p.BH * p.b1};
    const uint64_t str[2] = {(uint64_t)width * 2, (uint64_t)p.b2 * width * 2};
    const uint32_t box[3] = {width == 16 ? 16u : 64u, 1, 128};
    return make_map(m, base, 3, dims, str, box, sw);
}

// Keys or values in the call's layout as a 4-D map (x, token, head, batch), box
// (64, rows): a block's rows of one head; rows past Nk read zeros.
bool map_keys(CUtensorMap *m, const void *base, const Problem &p, uint32_t rows) {
    const uint64_t batch = (uint64_t)p.Nk * p.H * kD * 2;
    if (p.layout == kLayoutBNHD) {   // (x, head, token, batch)
        const uint64_t dims[4] = {(uint64_t)kD, (uint64_t)p.H, (uint64_t)p.Nk, (uint64_t)p.B};
        const uint64_t str[3] = {(uint64_t)kD * 2, (uint64_t)p.H * kD * 2, batch};
        const uint32_t box[4] = {64, 1, rows, 1};
        return make_map(m, base, 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
    }
    const uint64_t dims[4] = {(uint64_t)kD, (uint64_t)p.Nk, (uint64_t)p.H, (uint64_t)p.B};
    const uint64_t str[3] = {(uint64_t)kD * 2, (uint64_t)p.Nk * kD * 2, batch};
    const uint32_t box[4] = {64, rows, 1, 1};
    return make_map(m, base, 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}
// Queries in the call's layout as a 5-D map (x, v, u, head, batch), box (64, 1,
// 128): 128 block rows u at one column v (the inverse shuffle); rows past b1
// read zeros.
bool map_queries(CUtensorMap *m, const void *base, const Problem &p) {
    const uint64_t batch = (uint64_t)p.N * p.H * kD * 2;
    if (p.layout == kLayoutBNHD) {   // (x, head, v, u, batch)
        const uint64_t tok = (uint64_t)p.H * kD * 2;
        const uint64_t dims[5] = {(uint64_t)kD, (uint64_t)p.H, (uint64_t)p.b2, (uint64_t)p.b1,
                                  (uint64_t)p.B};
        const uint64_t str[4] = {(uint64_t)kD * 2, tok, (uint64_t)p.b2 * tok, batch};
        const uint32_t box[5] = {64, 1, 1, 128, 1};
        return make_map(m, base, 5, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
    }
    const uint64_t dims[5] = {(uint64_t)kD, (uint64_t)p.b2, (uint64_t)p.b1, (uint64_t)p.H,
                              (uint64_t)p.B};
    const uint64_t str[4] = {(uint64_t)kD * 2, (uint64_t)p.b2 * kD * 2, (uint64_t)p.N * kD * 2,
                             batch};
    const uint32_t box[5] = {64, 1, 128, 1, 1};
    return make_map(m, base, 5, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

cudaError_t run_rstep(const Problem &p, const TcWorkspace &ws, const void *k, const void *v,
                      int qblk, float c_log2, int *status, long long wait_limit, int stall,
                      cudaStream_t stream, int split) {
    const int nmt = qbar_tiles(p), mpad = nmt * 128, b2p = b2_padded(p.b2);
    CUtensorMap maps[6];
    const uint64_t dq[2] = {(uint64_t)kD, qblk ? (uint64_t)p.BH * p.b1k * mpad : (uint64_t)p.BH * mpad};
    const uint64_t s2[1] = {kD * 2};
    const uint32_t bq[2] = {64, 128};
    const uint64_t slab = (uint64_t)key_slab(p), rr = (uint64_t)p.tiles * p.b2;
    // Ktil and Z, [bh][u'][panel][r][64]: (x, r, panel, u', bh), one warp's 32 rows
    const uint64_t dst[5] = {64, rr, 2, slab, (uint64_t)p.BH};
    const uint64_t sst[4] = {128, rr * 128, 2 * rr * 128, slab * 2 * rr * 128};
    const uint32_t bst[5] = {64, 32, 1, 1, 1};
    // entropy panels, [bh][t*b2 rows][slab][16], stored 32 rows x 32 B per warp
    const uint64_t dhx[4] = {16, slab, (uint64_t)p.tiles * p.b2, (uint64_t)p.BH};
    const uint64_t shx[3] = {32, slab * 32, (uint64_t)p.tiles * p.b2 * slab * 32};
    const uint32_t bhx[4] = {16, 1, 32, 1};
    if (!make_map(&maps[0], qblk ? ws.qblk : ws.qbar, 2, dq, s2, bq) ||
        !map_keys(&maps[1], k, p, (uint32_t)b2p) || !map_keys(&maps[2], v, p, (uint32_t)b2p) ||
        !make_map(&maps[3], ws.z, 5, dst, sst, bst) || !make_map(&maps[4], ws.ktil, 5, dst, sst, bst) ||
        !make_map(&maps[5], ws.hx, 4, dhx, shx, bhx, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    const int pack = qblk ? 1 : rstep_pack(p);
    const int gph = (p.b1k + pack - 1) / pack;
    const int total = (p.head_end() - p.head_begin()) * gph;
    const int sms = sm_count();
    const int bpc = (total + sms - 1) / sms;
    const int grid = (total + bpc - 1) / bpc;
    const int hdirect = rstep_smem(b2p, nmt, 0, pack) > (uint32_t)kMaxSmem ? 1 : 0;
    RsArgs a{p, nmt, mpad, bpc, c_log2, 1.f / c_log2, qblk, hdirect, ws.hx, status, wait_limit,
             stall, pack, gph, split};
    ProfileScope scope(K_TC_RSTEP, stream);
    switch (b2p) {
        case 16: return launch_rstep<16>(maps, a, grid, stream);
        case 32: return launch_rstep<32>(maps, a, grid, stream);
        case 48: return launch_rstep<48>(maps, a, grid, stream);
        case 64: return launch_rstep<64>(maps, a, grid, stream);
        case 80: return launch_rstep<80>(maps, a, grid, stream);
        case 96: return launch_rstep<96>(maps, a, grid, stream);
        case 112: return launch_rstep<112>(maps, a, grid, stream);
        case 128: return launch_rstep<128>(maps, a, grid, stream);
    }
    return cudaErrorInvalidValue;
}

cudaError_t run_lstep(const Problem &p, const TcWorkspace &ws, const void *q, void *out, int mode,
                      float c_log2, int *status, long long wait_limit, int stall,
                      cudaStream_t stream) {
    const int mpad = qbar_tiles(p) * 128;
    CUtensorMap qg, kt, zt, xp;
    const uint64_t rows = key_rows(p);
    // Ktil and Z gathered from [bh][u'][panel][r][64]: 128 blocks u' of one row r
    const uint64_t rr = (uint64_t)p.tiles * p.b2, slab = (uint64_t)key_slab(p);
    const uint64_t dkz[5] = {64, rr, 2, slab, (uint64_t)p.BH};
    const uint64_t skz[4] = {128, rr * 128, 2 * rr * 128, slab * 2 * rr * 128};
    const uint32_t bkz[5] = {64, 1, 1, p.key_tiles ? 64u : 128u, 1};
    if (!map_queries(&qg, q, p) || !make_map(&kt, ws.ktil, 5, dkz, skz, bkz) ||
        !make_map(&zt, ws.z, 5, dkz, skz, bkz))
        return cudaErrorInvalidValue;
    const bool agg = mode == kLsAgg;
    if (agg ? !map_gather(&xp, ws.lam, p, 16, CU_TENSOR_MAP_SWIZZLE_32B)
            : !map_rows(&xp, ws.hx, rows, 16, CU_TENSOR_MAP_SWIZZLE_32B))
        return cudaErrorInvalidValue;
    // M-side rows per (g, v): the tile's queries, or (kLsAgg) the b1 Ktil rows
    // (with key-column tiles: all b1 query rows of each (head, column) problem)
    const int mrows = agg ? p.b1k : p.key_tiles ? p.b1 : tile_max_rows(p.b1, p.tiles);
    const int npairs = ((mrows + 127) / 128 + 1) / 2;
    const int units = p.key_tiles ? p.head_end() - p.head_begin() : p.unit_end - p.unit_begin;
    const int first = p.key_tiles ? p.head_begin() : p.unit_begin;
    const int nprob = units * p.b2 * npairs;
    LsArgs a{p, mode, npairs, nprob, first * p.b2 * npairs, mpad, c_log2,
             agg ? ws.qblk : (__nv_bfloat16 *)out, ws.lam, status, wait_limit, stall};
    const int grid = nprob < sm_count() ? nprob : sm_count();
    ProfileScope scope(mode == kLsOut ? K_TC_LSTEP : mode == kLsStat ? K_TC_LSTAT : K_TC_QAGG,
                       stream);
    cudaError_t e;
    switch (mode) {
        case kLsOut:
            e = set_smem(tc_lstep_kernel<kLsOut>, ls::kSmem);
            if (e != cudaSuccess) return e;
            tc_lstep_kernel<kLsOut><<<grid, ls::kThreads, ls::kSmem, stream>>>(qg, kt, zt, xp, a);
            break;
        case kLsStat:
            e = set_smem(tc_lstep_kernel<kLsStat>, ls::kSmem);
            if (e != cudaSuccess) return e;
            tc_lstep_kernel<kLsStat><<<grid, ls::kThreads, ls::kSmem, stream>>>(qg, kt, zt, xp, a);
            break;
        default:
            e = set_smem(tc_lstep_kernel<kLsAgg>, ls::kSmem);
            if (e != cudaSuccess) return e;
            tc_lstep_kernel<kLsAgg><<<grid, ls::kThreads, ls::kSmem, stream>>>(kt, qg, qg, xp, a);
            break;
    }
    return cudaGetLastError();
}

}  // namespace tcs

namespace tcs {

// S1: the first R-step's aggregated queries (uniform L: plain means).
cudaError_t run_qbar(const Problem &p, const void *q, const TcWorkspace &ws, cudaStream_t stream) {
    const int nchunk = (p.b2 * kD / 8 + 127) / 128;
    ProfileScope scope(K_TC_QBAR, stream);
    const int upb = p.key_tiles ? 1 : p.tiles;
    tc_qbar_kernel<<<(p.head_end() - p.head_begin()) * upb * nchunk, 128 * kQbarGroups, 0,
                     stream>>>((const __nv_bfloat16 *)q, ws.qbar, p, qbar_tiles(p) * 128,
                               rstep_pack(p));
    return cudaGetLastError();
}

}  // namespace tcs

cudaError_t sm100_forward(const Problem &p, const void *q, const void *k, const void *v,
                          void *out, void *workspace, int *status, long long wait_limit,
                          int stall, cudaStream_t stream) {
    const TcWorkspace ws = carve(p, workspace);
    const float c_log2 = p.scale * kLog2e;
    {
        cudaError_t e = run_qbar(p, q, ws, stream);
        if (e != cudaSuccess) return e;
    }
    if (key_slab(p) > p.b1k) {   // key-column tiles: the padding rows of every slab
        const int64_t work = (int64_t)p.BH * p.tiles * p.b2 * (key_slab(p) - p.b1k) * 34;
        const int blocks = (int)((work + 255) / 256 < 4 * 148 ? (work + 255) / 256 : 4 * 148);
        tc_keypad_kernel<<<blocks, 256, 0, stream>>>(ws.ktil, ws.z, ws.hx, p);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    // S2, then for every further iteration: the L-step's row statistics, the
    // re-aggregated queries (S4) and the R-step on them; then S3 with the output
    cudaError_t e = run_rstep(p, ws, k, v, 0, c_log2, status, wait_limit, stall, stream);
    for (int it = 1; e == cudaSuccess && it < p.iters; it++) {
        e = run_lstep(p, ws, q, out, kLsStat, c_log2, status, wait_limit, stall, stream);
        if (e == cudaSuccess)
            e = run_lstep(p, ws, q, out, kLsAgg, c_log2, status, wait_limit, stall, stream);
        if (e == cudaSuccess)
            e = run_rstep(p, ws, k, v, 1, c_log2, status, wait_limit, stall, stream);
    }
    if (e == cudaSuccess)
        e = run_lstep(p, ws, q, out, kLsOut, c_log2, status, wait_limit, stall, stream);
    return e;
}

}  // namespace monarch
