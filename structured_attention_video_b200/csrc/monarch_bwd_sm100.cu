// monarch_bwd_sm100.cu -- the backward pass of one iteration on the sm_100a
// tensor cores (bfloat16, d = 128, [B][H][N][d], self-attention, query-row
// tiles): the chain rule through the output, the L-step, the R-step and the
// query aggregation, as for the generic kernels of monarch_bwd.cu (the pages
// print no backward; they finetune through the attention: summary page,
// "Approach"; explainer page, "创新三：微调与高效内核").
#include "monarch_common.cuh"
#include "monarch_sm100.cuh"
#include "monarch_tc_shared.cuh"

#include <math.h>

namespace monarch {
namespace {

using namespace tcs;

// =====================================================================
// Backward of the L-step and the output on the tensor cores (bfloat16, d = 128,
// query-row tiles, one iteration).  Per (head, tile g, column v) problem, with
// the forward's row statistic lam (S units, S = q.Ktil raw) and delta = dy.y:
//   L = 2^((S + H' - lam) c_log2) (the L-step's probabilities), dP = dy.Z,
//   dS = L (dP - delta)  (the gradient of the natural logits s q.Ktil + H),
//   dZ = L^T dy,  dKtil = s dS^T q,  dH = sum over the tile's queries of dS,
//   dq (the L-step's part) = s dS Ktil.
// Three kernels of 256 threads, two per TMEM lane group: the logit products go to
// tensor memory, the threads overwrite them in place with the bfloat16 pairs of L
// and dS, and the accumulating products read those as their tensor-memory A
// operand.
//   tc_bwd_dkz_kernel: unit (bh, g, v, 128-key block); the key block's Ktil and Z
//     (M side) against each 128-query tile of the tile (N side): S^T, dP^T, then
//     dZ += L^T dy and dKtil += dS^T q over the query tiles; dH per key row.  The
//     two warps of a lane group split the query columns.
//   tc_bwd_dq_kernel<0>: unit (bh, g, v, pair of 128-query tiles); the queries and
//     dy of both tiles (M side) against each 64-key half: S, dP, and delta =
//     sum L dP per query row (= dy.y, from the same products that form dS, so that
//     every dS row sums to zero up to rounding).  Warps 0-3 take tile 0, warps 4-7
//     tile 1.
//   tc_bwd_dq_kernel<1>: the same units, then dq += dS Ktil over the halves.
// Every wait is bounded; on a time-out the CTA records MONARCH_ERR_TIMEOUT,
// drains its own copies and MMAs, frees its tensor memory and returns.
// =====================================================================
namespace lb {
// six 128 x 128 bfloat16 tiles: the operands loaded once (T0, T1) and two buffers of
// the ones loaded per step (T2, T3 and T4, T5), so that step i + 1's copies overlap
// step i's products and elementwise work
__host__ __device__ constexpr uint32_t tile(int i) { return (uint32_t)i * kTile; }
constexpr uint32_t kVec = 6 * kTile;             // 8 x 128 floats
constexpr uint32_t kBar = kVec + 8 * 512;
constexpr uint32_t kSmem = kBar + 128 + 1024;    // + slack to align the base to 1024
}  // namespace lb

struct LbArgs {
    Problem p;
    const uint4 *hx;        // entropy panels, one 32-byte row [H'_hi, H'_lo, 0...] per key row
    const uint4 *lam;       // row statistics, one 32-byte row [-lam_hi, -lam_lo, 0...] per query
    float *delta;           // [BH][N]: dy.y (written by tc_bwd_dq_kernel<0>)
    // dKtil and dZ in bfloat16, in the R-step's order [bh][u'][panel][r][64] (r = q̄
    // row g*b2 + v), and dH as float32 [bh][u'][r]: what the R-step side reads
    __nv_bfloat16 *dktb, *dzb;
    float *dhr;
    float *dql;             // [BH][N][d]: the L-step's part of dq
    float c_log2;
    int nkb;                // 128-key blocks per problem
    int nqt;                // 128-query tiles per problem (of the largest tile)
    int *status;
    long long limit;
};

__device__ __forceinline__ float pair_sum(uint32_t pr) {   // hi + lo of a bfloat16 pair
    return __uint_as_float(pr << 16) + __uint_as_float(pr & 0xFFFF0000u);
}

// Block-wide bounded wait: every thread polls, the CTA takes one decision.
__device__ __forceinline__ bool wait_block(uint64_t *bar, uint32_t parity, const WaitCtx &w) {
    const bool ok = wait_phase(bar, parity, w);
    return __syncthreads_and(ok) != 0;
}

__global__ void __launch_bounds__(256, 1)
tc_bwd_dkz_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDy,
                  const __grid_constant__ CUtensorMap tmKt, const __grid_constant__ CUtensorMap tmZ,
                  LbArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    const Problem &p = a.p;
    uint64_t *kz_bar = reinterpret_cast<uint64_t *>(sm + lb::kBar);
    uint64_t *qb_bar = kz_bar + 1;    // [2]: query tile buffers
    uint64_t *mma_bar = kz_bar + 3;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(kz_bar + 4);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(kz_bar + 5);
    float *vec = reinterpret_cast<float *>(sm + lb::kVec);   // [buffer][lam | delta][128]
    float *dh_part = vec + 512;                               // [128]: the second half's dH
    // two warps per group of 32 TMEM lanes: thread (j, half) takes key row j and the
    // half's 64 query columns (chunks 2*half, 2*half + 1)
    const int warp = threadIdx.x >> 5, j = (warp & 3) * 32 + (threadIdx.x & 31), half = warp >> 2;

    int unit = blockIdx.x;
    const int kb = unit % a.nkb;
    unit /= a.nkb;
    const int v = unit % p.b2;
    unit /= p.b2;
    const int g = unit % p.tiles, bh = unit / p.tiles;
    const int u_lo = tile_begin(g, p.b1, p.tiles), u_hi = tile_begin(g + 1, p.b1, p.tiles);
    const int64_t krow0 = (((int64_t)bh * p.tiles + g) * p.b2 + v) * p.b1k + (int64_t)kb * 128;
    const int nkv = min(128, p.b1k - kb * 128);
    const int nqt = (u_hi - u_lo + 127) / 128;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 4; i++) mbar_init(kz_bar + i, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);   // this warp's lanes
    const WaitCtx w{a.limit, a.status, abort_flag};
    uint32_t kz_issued = 0, kz_done = 0, mma_issued = 0, mma_done = 0;
    uint32_t qb_issued[2] = {0, 0}, qb_done[2] = {0, 0};

    // query tile cc into buffer b: its q and dy rows (thread 0), its lam and delta
    auto stage_q = [&](int cc, int b) {
        const int u0 = u_lo + 128 * cc, nqc = min(128, u_hi - u0);
        if (threadIdx.x == 0) {
            mbar_expect_tx(qb_bar + b, 2 * kTile);
            for (int pn = 0; pn < 2; pn++) {
                ls_load_q(sm + lb::tile(2 + 2 * b) + pn * kPanel, &tmQ, pn * 64, v, u0, bh, p,
                          qb_bar + b);
                ls_load_q(sm + lb::tile(3 + 2 * b) + pn * kPanel, &tmDy, pn * 64, v, u0, bh, p,
                          qb_bar + b);
            }
        }
        qb_issued[b]++;
        const int i = threadIdx.x;
        if (i < 128) {
            float lm = 0.f, dl = 0.f;
            if (i < nqc) {
                const int64_t tok = (int64_t)bh * p.N + (int64_t)(u0 + i) * p.b2 + v;
                lm = -pair_sum(a.lam[tok * 2].x);
                dl = a.delta[tok];
            }
            vec[b * 256 + i] = lm;
            vec[b * 256 + 128 + i] = dl;
        }
    };

    // the key block: Ktil and Z rows (128 blocks u' of row (g, v); past b1k: zeros),
    // then the first two query tiles
    if (threadIdx.x == 0) {
        mbar_expect_tx(kz_bar, 2 * kTile);
        for (int pn = 0; pn < 2; pn++) {
            ls_load_kz(sm + lb::tile(0) + pn * kPanel, &tmKt, pn, (int)krow0, p, kz_bar);
            ls_load_kz(sm + lb::tile(1) + pn * kPanel, &tmZ, pn, (int)krow0, p, kz_bar);
        }
    }
    kz_issued++;
    stage_q(0, 0);
    if (nqt > 1) stage_q(1, 1);
    const bool key_ok = j < nkv;
    const float hj = key_ok ? pair_sum(a.hx[(krow0 + j) * 2].x) : 0.f;
    bool ok = wait_block(kz_bar, 0, w);
    if (ok) kz_done++;

    const uint64_t dKt = smem_desc_sw128(smem_u32(sm + lb::tile(0)), 16, 1024);
    const uint64_t dZk = smem_desc_sw128(smem_u32(sm + lb::tile(1)), 16, 1024);
    constexpr uint32_t idS = idesc_bf16(128, 128, 0, 0), idO = idesc_bf16(128, 128, 0, 1);
    float dh_acc = 0.f;
    for (int c = 0; ok && c < nqt; c++) {
        const int b = c & 1, nqc = min(128, u_hi - (u_lo + 128 * c));
        const float *lq = vec + b * 256, *dq_s = vec + b * 256 + 128;
        const uint32_t tq = smem_u32(sm + lb::tile(2 + 2 * b)), ty = smem_u32(sm + lb::tile(3 + 2 * b));
        if (!(ok = wait_block(qb_bar + b, (c >> 1) & 1, w))) break;
        qb_done[b]++;
        if (warp == 0) {
            tc_fence_after();
            mma8_ss_k128(tmem, dKt, smem_desc_sw128(tq, 16, 1024), idS, 0u);          // S^T = Ktil q^T
            mma8_ss_k128(tmem + 128, dZk, smem_desc_sw128(ty, 16, 1024), idS, 0u);    // dP^T = Z dy^T
            mma_commit_warp(mma_bar);
        }
        mma_issued++;
        if (!(ok = wait_block(mma_bar, mma_done & 1, w))) break;
        mma_done++;
        tc_fence_after();
        // L^T and dS^T of this key row over the half's queries, packed in place: both
        // halves read all of their S^T and dP^T columns before either writes (the
        // packed pairs of the upper half land on columns the lower half reads)
        float sv[64], dv64[64];
        tmem_ld32f(tl + 64 * half, sv);
        tmem_ld32f(tl + 64 * half + 32, sv + 32);
        tmem_ld32f(tl + 128 + 64 * half, dv64);
        tmem_ld32f(tl + 128 + 64 * half + 32, dv64 + 32);
        tmem_wait_ld();
        __syncthreads();
#pragma unroll
        for (int cc = 0; cc < 2; cc++) {
            const int ch = 2 * half + cc;
            const float *s = sv + 32 * cc, *d = dv64 + 32 * cc;
            uint32_t pk[16], dk[16];
#pragma unroll
            for (int k = 0; k < 32; k += 2) {
                float pv[2], dv[2];
#pragma unroll
                for (int e = 0; e < 2; e++) {
                    const int i = ch * 32 + k + e;
                    const float pr = (key_ok && i < nqc)
                                         ? fast_exp2((s[k + e] + hj - lq[i]) * a.c_log2) : 0.f;
                    const float ds = pr * (d[k + e] - dq_s[i]);
                    dh_acc += ds;
                    pv[e] = pr;
                    dv[e] = ds;
                }
                pk[k / 2] = pack_bf16(pv[0], pv[1]);
                dk[k / 2] = pack_bf16(dv[0], dv[1]);
            }
            const uint32_t(&pk0)[8] = *reinterpret_cast<const uint32_t(*)[8]>(&pk[0]);
            const uint32_t(&pk1)[8] = *reinterpret_cast<const uint32_t(*)[8]>(&pk[8]);
            const uint32_t(&dk0)[8] = *reinterpret_cast<const uint32_t(*)[8]>(&dk[0]);
            const uint32_t(&dk1)[8] = *reinterpret_cast<const uint32_t(*)[8]>(&dk[8]);
            tmem_st8(tl + ch * 16, pk0);
            tmem_st8(tl + ch * 16 + 8, pk1);
            tmem_st8(tl + 128 + ch * 16, dk0);
            tmem_st8(tl + 128 + ch * 16 + 8, dk1);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        if (warp == 0) {
            tc_fence_after();
            mma8_ts_mn128(tmem + 256, tmem, smem_desc_sw128(ty, kPanel, 1024), idO,
                          c > 0 ? 1u : 0u);                                        // dZ += L^T dy
            mma8_ts_mn128(tmem + 384, tmem + 128, smem_desc_sw128(tq, kPanel, 1024), idO,
                          c > 0 ? 1u : 0u);                                        // += dS^T q
            mma_commit_warp(mma_bar);
        }
        mma_issued++;
        if (!(ok = wait_block(mma_bar, mma_done & 1, w))) break;
        mma_done++;
        tc_fence_after();
        if (c + 2 < nqt) stage_q(c + 2, b);   // buffer b is free again
    }
    if (half == 1) dh_part[j] = dh_acc;
    __syncthreads();
    if (ok && nqt > 0) {
        // key row u' of q̄ row r = g*b2 + v: 32 columns per chunk, two chunks per panel
        // (the half's panel)
        const int up = kb * 128 + j, r = g * p.b2 + v, rr = p.tiles * p.b2;
        const int64_t rowbase = ((int64_t)bh * p.b1k + up) * 2;   // panel 0 of (bh, u')
#pragma unroll 1
        for (int ch = 2 * half; ch < 2 * half + 2; ch++) {
            float z[32], kt[32];
            tmem_ld32f(tl + 256 + ch * 32, z);
            tmem_ld32f(tl + 384 + ch * 32, kt);
            tmem_wait_ld();
            if (key_ok) {
                const int64_t off = ((rowbase + ch / 2) * rr + r) * 64 + (ch & 1) * 32;
                uint4 *oz = reinterpret_cast<uint4 *>(a.dzb + off);
                uint4 *ok4 = reinterpret_cast<uint4 *>(a.dktb + off);
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    oz[e] = make_uint4(pack_bf16(z[8 * e], z[8 * e + 1]),
                                       pack_bf16(z[8 * e + 2], z[8 * e + 3]),
                                       pack_bf16(z[8 * e + 4], z[8 * e + 5]),
                                       pack_bf16(z[8 * e + 6], z[8 * e + 7]));
                    ok4[e] = make_uint4(pack_bf16(kt[8 * e] * p.scale, kt[8 * e + 1] * p.scale),
                                        pack_bf16(kt[8 * e + 2] * p.scale, kt[8 * e + 3] * p.scale),
                                        pack_bf16(kt[8 * e + 4] * p.scale, kt[8 * e + 5] * p.scale),
                                        pack_bf16(kt[8 * e + 6] * p.scale, kt[8 * e + 7] * p.scale));
                }
            }
        }
        if (key_ok && half == 0) a.dhr[((int64_t)bh * p.b1k + up) * rr + r] = dh_acc + dh_part[j];
    }
    // drain this CTA's own copies and MMAs before its tensor memory is freed
    if (threadIdx.x == 0) {
        if (kz_issued > kz_done) wait_phase_cleanup(kz_bar, 0, kCleanupPolls);
        for (int b = 0; b < 2; b++)
            if (qb_issued[b] > qb_done[b])
                wait_phase_cleanup(qb_bar + b, (qb_issued[b] - 1) & 1, kCleanupPolls);
    }
    if (warp == 0 && mma_issued > mma_done)
        wait_phase_cleanup(mma_bar, (mma_issued - 1) & 1, kCleanupPolls);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// The query side, two 128-query tiles of one problem per CTA: the keys stream in
// 64-key halves of Ktil and Z through a ring of three stages, so that each pass
// reads Ktil and Z once per pair of query tiles.  Tensor memory: per tile t, S at
// columns t*128 + [0, 64) and dP at t*128 + [64, 128) (dS packed over S), and the
// dq accumulators at 256 + t*128.
namespace lq {
constexpr uint32_t kHalf = 64 * 128 * 2;          // 64 key rows of 128 bfloat16: two 8 KB panels
constexpr uint32_t kSlot = 2 * kHalf;             // a half of Ktil, then of Z
constexpr int kNS = 3;
constexpr uint32_t kRing = 4 * kTile;             // after q and dy of the two tiles
constexpr uint32_t kHk = kRing + kNS * kSlot;     // [kNS][64] floats: H' of the half's keys
constexpr uint32_t kBar = kHk + kNS * 64 * 4;
constexpr uint32_t kSmem = kBar + 128 + 1024;     // + slack to align the base to 1024
}  // namespace lq

// Eight K-steps (K = 128) of D = A B^T, A a 128-row K-major SW128 tile (64-column
// panels 16 KB apart), B a 64-row one (panels 8 KB apart): N = 64.  The offset
// descriptors are formed inside the asm block; elect.sync picks the issuing lane.
__device__ __forceinline__ void mma8_ss_k128_b64(uint32_t d_tmem, uint64_t a, uint64_t b,
                                                 uint32_t idesc) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        ".reg .b64 a1, a2, a3, a4, a5, a6, a7, b1, b2, b3, b4, b5, b6, b7;\n\t"
        "add.s64 a1, %1, 2;\n\tadd.s64 a2, %1, 4;\n\tadd.s64 a3, %1, 6;\n\t"
        "add.s64 a4, %1, 1024;\n\tadd.s64 a5, %1, 1026;\n\tadd.s64 a6, %1, 1028;\n\t"
        "add.s64 a7, %1, 1030;\n\t"
        "add.s64 b1, %2, 2;\n\tadd.s64 b2, %2, 4;\n\tadd.s64 b3, %2, 6;\n\t"
        "add.s64 b4, %2, 512;\n\tadd.s64 b5, %2, 514;\n\tadd.s64 b6, %2, 516;\n\t"
        "add.s64 b7, %2, 518;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %3, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a2, b2, %3, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a3, b3, %3, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a4, b4, %3, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a5, b5, %3, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a6, b6, %3, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a7, b7, %3, 1;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc)
        : "memory");
}

template <int MODE>
__global__ void __launch_bounds__(256, 1)
tc_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDy,
                 const __grid_constant__ CUtensorMap tmKt, const __grid_constant__ CUtensorMap tmZ,
                 LbArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    const Problem &p = a.p;
    constexpr int NS = lq::kNS;
    uint64_t *q_bar = reinterpret_cast<uint64_t *>(sm + lq::kBar);
    uint64_t *kz_bar = q_bar + 1;     // [NS]: a half of Ktil and Z in its stage
    uint64_t *mma_bar = q_bar + 1 + NS;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(mma_bar + 2);
    float *hk = reinterpret_cast<float *>(sm + lq::kHk);
    // warps 0-3 take tile 0 of the pair, warps 4-7 tile 1: thread j of a tile, query row j
    const int warp = threadIdx.x >> 5, j = (warp & 3) * 32 + (threadIdx.x & 31), t = warp >> 2;

    int unit = blockIdx.x;
    const int npair = (a.nqt + 1) / 2;
    const int pair = unit % npair;
    unit /= npair;
    const int v = unit % p.b2;
    unit /= p.b2;
    const int g = unit % p.tiles, bh = unit / p.tiles;
    const int u_lo = tile_begin(g, p.b1, p.tiles), u_hi = tile_begin(g + 1, p.b1, p.tiles);
    const int u00 = u_lo + 256 * pair;                  // the pair's first query row
    const int nq0 = min(128, u_hi - u00), nq1 = min(128, u_hi - u00 - 128);
    if (nq0 <= 0) return;   // a tile shorter than the longest one: no such pair (uniform)
    const int ntl = nq1 > 0 ? 2 : 1;                    // query tiles of the pair
    const bool tile_ok = t < ntl;
    const int u0 = u00 + 128 * t;
    const int64_t slab0 = (((int64_t)bh * p.tiles + g) * p.b2 + v) * p.b1k;
    const int64_t tok = (int64_t)bh * p.N + (int64_t)(u0 + j) * p.b2 + v;
    const bool row_ok = tile_ok && j < (t ? nq1 : nq0);
    const float lam = row_ok ? -pair_sum(a.lam[tok * 2].x) : 0.f;
    const float dlt = (MODE == 1 && row_ok) ? a.delta[tok] : 0.f;
    const int nh = (p.b1k + 63) / 64;
    float dsum = 0.f;   // MODE 0: sum over the keys of L dP

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2 + NS; i++) mbar_init(q_bar + i, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const WaitCtx w{a.limit, a.status, abort_flag};
    uint32_t q_issued = 0, q_done = 0, mma_issued = 0, mma_done = 0;
    uint32_t kz_issued[NS], kz_done[NS];
#pragma unroll
    for (int st = 0; st < NS; st++) kz_issued[st] = kz_done[st] = 0;
    bool uncommitted = false;   // warp 0 issued products after its last commit

    // half h of the keys into stage h % NS: its Ktil and Z rows (thread 0; rows past b1k
    // read zeros) and its entropies
    auto stage = [&](int h) {
        const int st = h % NS;
        if (threadIdx.x == 0) {
            uint8_t *base = sm + lq::kRing + st * lq::kSlot;
            int r, u, b;
            kz_coords(p, (int)(slab0 + 64 * h), r, u, b);
            mbar_expect_tx(kz_bar + st, lq::kSlot);
            for (int pn = 0; pn < 2; pn++) {
                tma_load_5d(base + pn * (lq::kHalf / 2), &tmKt, 0, r, pn, u, b, kz_bar + st);
                tma_load_5d(base + lq::kHalf + pn * (lq::kHalf / 2), &tmZ, 0, r, pn, u, b, kz_bar + st);
            }
        }
        kz_issued[st]++;
        const int i = threadIdx.x;
        if (i < 64)
            hk[st * 64 + i] = 64 * h + i < p.b1k ? pair_sum(a.hx[(slab0 + 64 * h + i) * 2].x) : 0.f;
    };

    if (threadIdx.x == 0) {   // q and dy of the pair's tiles
        mbar_expect_tx(q_bar, 2 * ntl * kTile);
        for (int tt = 0; tt < ntl; tt++)
            for (int pn = 0; pn < 2; pn++) {
                ls_load_q(sm + lb::tile(2 * tt) + pn * kPanel, &tmQ, pn * 64, v, u00 + 128 * tt, bh, p, q_bar);
                ls_load_q(sm + lb::tile(2 * tt + 1) + pn * kPanel, &tmDy, pn * 64, v, u00 + 128 * tt, bh, p,
                          q_bar);
            }
    }
    q_issued++;
    for (int h = 0; h < NS && h < nh; h++) stage(h);
    bool ok = wait_block(q_bar, 0, w);
    if (ok) q_done++;

    constexpr uint32_t idS = idesc_bf16(128, 64, 0, 0), idO = idesc_bf16(128, 128, 0, 1);
    if constexpr (MODE == 0) {
        // delta needs no accumulator: the products of half h + 1 go to the other 256
        // columns of tensor memory (buffer (h + 1) & 1) while the threads work on half h
        auto issue = [&](int h) {   // warp 0
            const uint32_t kt = smem_u32(sm + lq::kRing + (h % NS) * lq::kSlot), zt = kt + lq::kHalf;
            const uint32_t tb = tmem + 256 * (h & 1);
            tc_fence_after();
            for (int tt = 0; tt < ntl; tt++) {
                mma8_ss_k128_b64(tb + tt * 128, smem_desc_sw128(smem_u32(sm + lb::tile(2 * tt)), 16, 1024),
                                 smem_desc_sw128(kt, 16, 1024), idS);                          // S = q Ktil^T
                mma8_ss_k128_b64(tb + tt * 128 + 64,
                                 smem_desc_sw128(smem_u32(sm + lb::tile(2 * tt + 1)), 16, 1024),
                                 smem_desc_sw128(zt, 16, 1024), idS);                          // dP = dy Z^T
            }
            mma_commit_warp(mma_bar);
        };
        if (ok && nh > 0 && (ok = wait_block(kz_bar, 0, w))) {
            kz_done[0]++;
            if (warp == 0) issue(0);
            mma_issued++;
        }
        for (int h = 0; ok && h < nh; h++) {
            const int st = h % NS;
            if (!(ok = wait_block(mma_bar, mma_done & 1, w))) break;
            mma_done++;
            if (h + 1 < nh) {   // half h + 1, loaded during an earlier step
                const int s1 = (h + 1) % NS;
                if (!(ok = wait_block(kz_bar + s1, ((h + 1) / NS) & 1, w))) break;
                kz_done[s1]++;
                if (warp == 0) issue(h + 1);
                mma_issued++;
            }
            // the products of half h - 1 are done: its stage takes half h + 2 (its
            // entropies were last read before the previous barrier)
            if (h >= 1 && h + 2 < nh) stage(h + 2);
            tc_fence_after();
            if (tile_ok) {
                const float *hkh = hk + st * 64;
                const uint32_t ts = tl + 256 * (h & 1) + t * 128;
                float sv[64], dv[64];
                tmem_ld32f(ts, sv);
                tmem_ld32f(ts + 32, sv + 32);
                tmem_ld32f(ts + 64, dv);
                tmem_ld32f(ts + 96, dv + 32);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 64; k++) {
                    const float pr = (row_ok && 64 * h + k < p.b1k)
                                         ? fast_exp2((sv[k] + hkh[k] - lam) * a.c_log2) : 0.f;
                    dsum = fmaf(pr, dv[k], dsum);
                }
            }
            // every thread is done with buffer h & 1: the products of half h + 2 may
            // overwrite it
            tc_fence_before();
            __syncthreads();
        }
    } else {
        for (int h = 0; ok && h < nh; h++) {
            const int st = h % NS;
            if (!(ok = wait_block(kz_bar + st, (h / NS) & 1, w))) break;
            kz_done[st]++;
            const uint32_t kt = smem_u32(sm + lq::kRing + st * lq::kSlot), zt = kt + lq::kHalf;
            if (warp == 0) {
                tc_fence_after();
                for (int tt = 0; tt < ntl; tt++) {
                    mma8_ss_k128_b64(tmem + tt * 128, smem_desc_sw128(smem_u32(sm + lb::tile(2 * tt)), 16, 1024),
                                     smem_desc_sw128(kt, 16, 1024), idS);                          // S = q Ktil^T
                    mma8_ss_k128_b64(tmem + tt * 128 + 64,
                                     smem_desc_sw128(smem_u32(sm + lb::tile(2 * tt + 1)), 16, 1024),
                                     smem_desc_sw128(zt, 16, 1024), idS);                          // dP = dy Z^T
                }
                mma_commit_warp(mma_bar);
                uncommitted = false;
            }
            mma_issued++;
            if (!(ok = wait_block(mma_bar, mma_done & 1, w))) break;
            mma_done++;
            // every product of half h - 1 is done too (the commit covers them): its stage
            // takes half h + 2 (its entropies were last read before the previous barrier)
            if (h >= 1 && h + 2 < nh) stage(h + 2);
            tc_fence_after();
            if (tile_ok) {
                const float *hkh = hk + st * 64;
                const uint32_t ts = tl + t * 128;
                float sv[64], dv[64];
                tmem_ld32f(ts, sv);
                tmem_ld32f(ts + 32, sv + 32);
                tmem_ld32f(ts + 64, dv);
                tmem_ld32f(ts + 96, dv + 32);
                tmem_wait_ld();
                {
                    uint32_t dk[32];
#pragma unroll
                    for (int k = 0; k < 64; k += 2) {
                        float dd[2];
#pragma unroll
                        for (int e = 0; e < 2; e++) {
                            const float pr = (row_ok && 64 * h + k + e < p.b1k)
                                                 ? fast_exp2((sv[k + e] + hkh[k + e] - lam) * a.c_log2) : 0.f;
                            dd[e] = pr * (dv[k + e] - dlt);
                        }
                        dk[k / 2] = pack_bf16(dd[0], dd[1]);
                    }
#pragma unroll
                    for (int q8 = 0; q8 < 4; q8++)
                        tmem_st8(ts + q8 * 8, *reinterpret_cast<const uint32_t(*)[8]>(&dk[q8 * 8]));
                    tmem_wait_st();
                }
            }
            // every thread is done with this half's columns (and in MODE 1 has stored dS)
            tc_fence_before();
            __syncthreads();
            if (warp == 0) {
                tc_fence_after();
                for (int tt = 0; tt < ntl; tt++)
                    mma4_ts_mn64(tmem + 256 + tt * 128, tmem + tt * 128, smem_desc_sw128(kt, lq::kHalf / 2, 1024),
                                 idO, h > 0 ? 1u : 0u);                                            // dq' += dS Ktil
                uncommitted = true;
            }
        }
    }
    if (MODE == 0) {
        if (ok && row_ok) a.delta[tok] = dsum;
    } else if (ok) {   // the last half's dq products, then dq' to memory
        if (warp == 0) {
            mma_commit_warp(mma_bar);
            uncommitted = false;
        }
        mma_issued++;
        if ((ok = wait_block(mma_bar, mma_done & 1, w))) mma_done++;
        tc_fence_after();
        if (ok && tile_ok) {
#pragma unroll 1
            for (int ch = 0; ch < 4; ch++) {
                float o[32];
                tmem_ld32f(tl + 256 + t * 128 + ch * 32, o);
                tmem_wait_ld();
                if (row_ok) {
                    float4 *dst = reinterpret_cast<float4 *>(a.dql + tok * kD + ch * 32);
#pragma unroll
                    for (int e = 0; e < 8; e++)
                        dst[e] = make_float4(o[4 * e] * p.scale, o[4 * e + 1] * p.scale,
                                             o[4 * e + 2] * p.scale, o[4 * e + 3] * p.scale);
                }
            }
        }
    }
    // drain this CTA's own copies and products before its tensor memory is freed
    if (warp == 0 && uncommitted) {
        mma_commit_warp(mma_bar);
        mma_issued++;
    }
    if (threadIdx.x == 0) {
        if (q_issued > q_done) wait_phase_cleanup(q_bar, 0, kCleanupPolls);
#pragma unroll
        for (int st = 0; st < NS; st++)
            if (kz_issued[st] > kz_done[st])
                wait_phase_cleanup(kz_bar + st, (kz_issued[st] - 1) & 1, kCleanupPolls);
    }
    if (warp == 0 && mma_issued > mma_done)
        wait_phase_cleanup(mma_bar, (mma_issued - 1) & 1, kCleanupPolls);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// =====================================================================
// Backward of the R-step and the query aggregation on the tensor cores.  Per
// (head, block u'), over the t*b2 aggregated rows r = (g, v) in 128-row tiles:
//   a = s q̄ K^T, R = softmax(a), dR = dKtil K^T + dZ V^T,
//   da = R (dR - sum R dR) - dH R (a - sum R a)   (dH/da = -R (a - E_R[a])),
//   dk = s da^T q̄ + R^T dKtil,  dv = R^T dZ  (complete in the CTA: the block's keys),
//   dq̄ = s sum over u' of da K  (tc_bwd_dqbar_kernel, over the blocks in chunks).
// tc_bwd_r_kernel: the logits and dR as tcgen05 products into tensor memory; two
// threads per row (warps w and w + 4 share a group of 32 TMEM lanes, each with
// half of the key chunks, their row sums met in shared memory) form R and s*da,
// write them as bfloat16 [row][key] tiles (the MN-major A operands of dk and dv,
// keys along M) and s*da to global memory; dk and dv accumulate in tensor memory
// over the row tiles.
// =====================================================================
namespace rb {
constexpr uint32_t kQ = 0;              // q̄ row tile (K-major for the logits, MN-major for dk)
constexpr uint32_t kDK = kTile;         // dKtil row tile
constexpr uint32_t kDZ = 2 * kTile;     // dZ row tile
constexpr uint32_t kDA = 3 * kTile;     // s*da as [row][key] (two 64-key panels)
constexpr uint32_t kR = 4 * kTile;      // R as [row][key]
constexpr uint32_t kKV = 5 * kTile;     // K then V of the block: 2 panels of B2P rows each
constexpr uint32_t kBar = kKV + 4 * 128 * 128;
constexpr uint32_t kSmem = kBar + 64 + 1024;
// tc_bwd_dqbar_kernel: a ring of stages, each one block's s*da tile and its K rows
// (two 64-column panels of B2P rows)
template <int B2P> struct Dq {
    static constexpr uint32_t kStage = kTile + 2 * B2P * 128;
    static constexpr int kNS = B2P <= 80 ? 4 : 3;
    static constexpr uint32_t kBar = kNS * kStage;
    static constexpr uint32_t kSmem = kBar + 128 + 1024;
};
}  // namespace rb

struct RbArgs {
    Problem p;
    int mpad;                    // rows per head of the q̄ tile stack
    const float *dhr;            // dH [bh][u'][r]
    __nv_bfloat16 *da;           // s*da [bh][u'][2][r][64]
    __nv_bfloat16 *dk, *dv;      // outputs [B][H][N][d]
    float *part;                 // partial dq̄ [bh][mt][ch][128][128]
    int nmt, nch, upc;           // row tiles, block chunks, blocks per chunk
    int *status;
    long long limit;
};

// byte offset of the 16-byte chunk c of row r in a 128-byte-swizzled panel
__device__ __forceinline__ uint32_t sw128(int r, int c) {
    return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

template <int B2P>
__global__ void __launch_bounds__(256, 1)
tc_bwd_r_kernel(const __grid_constant__ CUtensorMap tmQb, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDK,
                const __grid_constant__ CUtensorMap tmDZ, RbArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    const Problem &p = a.p;
    uint64_t *ld_bar = reinterpret_cast<uint64_t *>(sm + rb::kBar);
    uint64_t *mma_bar = ld_bar + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(ld_bar + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(ld_bar + 3);
    const int warp = threadIdx.x >> 5, r = (warp & 3) * 32 + (threadIdx.x & 31), half = warp >> 2;
    const int bh = blockIdx.x / p.b1k, up = blockIdx.x % p.b1k;
    const int rr = p.tiles * p.b2;
    constexpr uint32_t kPanelKV = B2P * 128;
    // the row's 16-key chunks: the first kC0 to half 0, the rest to half 1
    constexpr int kC = B2P / 16, kC0 = (kC + 1) / 2;
    const int nck = half ? kC - kC0 : kC0, kbase = half ? kC0 * 16 : 0;
    // the two halves' row sums (max, sum, E, rho), in the s*da tile before it is written
    float *red = reinterpret_cast<float *>(sm + rb::kDA);

    if (threadIdx.x == 0) {
        mbar_init(ld_bar, 1);
        mbar_init(mma_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const WaitCtx w{a.limit, a.status, abort_flag};
    uint32_t ld_issued = 0, ld_done = 0, mma_issued = 0, mma_done = 0;

    if (threadIdx.x == 0) {   // the block's b2 keys and values ([B][H][N][d]: (x, token, head, batch))
        const int tok0 = up * p.b2, hh = bh % p.H, bb = bh / p.H;
        mbar_expect_tx(ld_bar, 4 * kPanelKV);
        for (int pn = 0; pn < 2; pn++) {
            tma_load_4d(sm + rb::kKV + pn * kPanelKV, &tmK, pn * 64, tok0, hh, bb, ld_bar);
            tma_load_4d(sm + rb::kKV + 2 * kPanelKV + pn * kPanelKV, &tmV, pn * 64, tok0, hh, bb,
                        ld_bar);
        }
    }
    ld_issued++;
    bool ok = wait_block(ld_bar, ld_done & 1, w);
    if (ok) ld_done++;

    const uint64_t dQk = smem_desc_sw128(smem_u32(sm + rb::kQ), 16, 1024);
    const uint64_t dDKk = smem_desc_sw128(smem_u32(sm + rb::kDK), 16, 1024);
    const uint64_t dDZk = smem_desc_sw128(smem_u32(sm + rb::kDZ), 16, 1024);
    const uint64_t dKk = smem_desc_sw128(smem_u32(sm + rb::kKV), 16, 1024);
    const uint64_t dVk = smem_desc_sw128(smem_u32(sm + rb::kKV + 2 * kPanelKV), 16, 1024);
    // MN-major operands: 64-element groups 16 KB apart, K steps of 16 rows = 2 KB
    const uint64_t dQm = smem_desc_sw128(smem_u32(sm + rb::kQ), kPanel, 1024);
    const uint64_t dDKm = smem_desc_sw128(smem_u32(sm + rb::kDK), kPanel, 1024);
    const uint64_t dDZm = smem_desc_sw128(smem_u32(sm + rb::kDZ), kPanel, 1024);
    const uint64_t dDAm = smem_desc_sw128(smem_u32(sm + rb::kDA), kPanel, 1024);
    const uint64_t dRm = smem_desc_sw128(smem_u32(sm + rb::kR), kPanel, 1024);
    constexpr uint32_t idL = idesc_bf16(128, B2P, 0, 0), idO = idesc_bf16(128, 128, 1, 1);
    for (int mt = 0; ok && mt < a.nmt; mt++) {
        if (threadIdx.x == 0) {
            mbar_expect_tx(ld_bar, 3 * kTile);
            for (int pn = 0; pn < 2; pn++) {
                tma_load_2d(sm + rb::kQ + pn * kPanel, &tmQb, pn * 64, bh * a.mpad + mt * 128, ld_bar);
                tma_load_5d(sm + rb::kDK + pn * kPanel, &tmDK, 0, mt * 128, pn, up, bh, ld_bar);
                tma_load_5d(sm + rb::kDZ + pn * kPanel, &tmDZ, 0, mt * 128, pn, up, bh, ld_bar);
            }
        }
        ld_issued++;
        const int rg = mt * 128 + r;
        const bool row_ok = rg < rr;
        const float dh = row_ok ? a.dhr[((int64_t)bh * p.b1k + up) * rr + rg] : 0.f;
        if (!(ok = wait_block(ld_bar, ld_done & 1, w))) break;
        ld_done++;
        if (warp == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; kk++) {
                const uint32_t ao = (kk >> 2) * kPanel + (kk & 3) * 32;
                const uint32_t bo = (kk >> 2) * kPanelKV + (kk & 3) * 32;
                mma_ss_warp(tmem, desc_plus(dQk, ao), desc_plus(dKk, bo), idL, kk > 0);          // q̄ K^T
                mma_ss_warp(tmem + 128, desc_plus(dDKk, ao), desc_plus(dKk, bo), idL, kk > 0);   // dKtil K^T
            }
#pragma unroll
            for (int kk = 0; kk < 8; kk++) {
                const uint32_t ao = (kk >> 2) * kPanel + (kk & 3) * 32;
                const uint32_t bo = (kk >> 2) * kPanelKV + (kk & 3) * 32;
                mma_ss_warp(tmem + 128, desc_plus(dDZk, ao), desc_plus(dVk, bo), idL, 1u);       // + dZ V^T
            }
            mma_commit_warp(mma_bar);
        }
        mma_issued++;
        if (!(ok = wait_block(mma_bar, mma_done & 1, w))) break;
        mma_done++;
        tc_fence_after();
        // this row: R and s*da over this half's keys (x: the natural logits s*a,
        // y: dR; R is recomputed from x where it is needed, to keep two arrays)
        float x[kC0 * 16], y[kC0 * 16];
#pragma unroll
        for (int cc = 0; cc < kC0; cc++)
            if (cc < nck) {
                tmem_ld16f(tl + kbase + cc * 16, &x[cc * 16]);
                tmem_ld16f(tl + 128 + kbase + cc * 16, &y[cc * 16]);
            }
        tmem_wait_ld();
        float mx = -INFINITY;
#pragma unroll
        for (int k = 0; k < kC0 * 16; k++) {
            const bool kv = k < nck * 16 && kbase + k < p.b2;
            x[k] = kv ? x[k] * p.scale : 0.f;
            y[k] = kv ? y[k] : 0.f;
            mx = kv ? fmaxf(mx, x[k]) : mx;
        }
        red[half * 128 + r] = mx;
        __syncthreads();
        mx = fmaxf(mx, red[(half ^ 1) * 128 + r]);
        float l = 0.f;
#pragma unroll
        for (int k = 0; k < kC0 * 16; k++)
            l += (k < nck * 16 && kbase + k < p.b2) ? fast_exp2((x[k] - mx) * kLog2e) : 0.f;
        red[256 + half * 128 + r] = l;
        __syncthreads();
        l += red[256 + (half ^ 1) * 128 + r];   // the same sum in both halves (a + b = b + a)
        const float inv = 1.f / l;
        float E = 0.f, rho = 0.f;
#pragma unroll
        for (int k = 0; k < kC0 * 16; k++) {
            const float rk = (k < nck * 16 && kbase + k < p.b2) ? fast_exp2((x[k] - mx) * kLog2e) * inv : 0.f;
            E = fmaf(rk, x[k], E);
            rho = fmaf(rk, y[k], rho);
        }
        red[512 + half * 128 + r] = E;
        red[768 + half * 128 + r] = rho;
        __syncthreads();
        E += red[512 + (half ^ 1) * 128 + r];
        rho += red[768 + (half ^ 1) * 128 + r];
        __syncthreads();   // the sums are read before the s*da tile is written over them
        // s*da and R as bfloat16 [row][key] tiles; s*da also to global memory
        __nv_bfloat16 *dag = a.da + (((int64_t)bh * p.b1k + up) * 2 * rr + rg) * 64;
#pragma unroll
        for (int lc = 0; lc < 2 * kC0; lc++) {   // this half's 8-key chunks
            if (lc < 2 * nck) {
                const int key0 = kbase + 8 * lc, pn = key0 >> 6, ch = (key0 & 63) >> 3;
                uint32_t dw[4], rw[4];
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const int k = 8 * lc + 2 * e;
                    float d0 = 0.f, d1 = 0.f, r0 = 0.f, r1 = 0.f;
                    if (row_ok && key0 + 2 * e < p.b2) {
                        r0 = fast_exp2((x[k] - mx) * kLog2e) * inv;
                        d0 = p.scale * (r0 * (y[k] - rho) - dh * r0 * (x[k] - E));
                    }
                    if (row_ok && key0 + 2 * e + 1 < p.b2) {
                        r1 = fast_exp2((x[k + 1] - mx) * kLog2e) * inv;
                        d1 = p.scale * (r1 * (y[k + 1] - rho) - dh * r1 * (x[k + 1] - E));
                    }
                    dw[e] = pack_bf16(d0, d1);
                    rw[e] = pack_bf16(r0, r1);
                }
                const uint4 dv4 = make_uint4(dw[0], dw[1], dw[2], dw[3]);
                const uint4 rv4 = make_uint4(rw[0], rw[1], rw[2], rw[3]);
                *reinterpret_cast<uint4 *>(sm + rb::kDA + pn * kPanel + sw128(r, ch)) = dv4;
                *reinterpret_cast<uint4 *>(sm + rb::kR + pn * kPanel + sw128(r, ch)) = rv4;
                if (row_ok) reinterpret_cast<uint4 *>(dag + (int64_t)pn * rr * 64)[ch] = dv4;
            }
        }
        if (half == 1) {   // keys B2P..127 of the tiles (and of s*da's last panel): zeros
            const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
            for (int key0 = B2P; key0 < 128; key0 += 8) {
                const int pn = key0 >> 6, ch = (key0 & 63) >> 3;
                *reinterpret_cast<uint4 *>(sm + rb::kDA + pn * kPanel + sw128(r, ch)) = z4;
                *reinterpret_cast<uint4 *>(sm + rb::kR + pn * kPanel + sw128(r, ch)) = z4;
                if (row_ok && pn * 64 < B2P) reinterpret_cast<uint4 *>(dag + (int64_t)pn * rr * 64)[ch] = z4;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (warp == 0) {
            tc_fence_after();
            // dk += (s da)^T q̄ + R^T dKtil,  dv += R^T dZ: K = the tile's 128 rows
#pragma unroll
            for (int kk = 0; kk < 8; kk++)
                mma_ss_warp(tmem + 256, desc_plus(dDAm, kk * 2048), desc_plus(dQm, kk * 2048), idO,
                            (mt > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
            for (int kk = 0; kk < 8; kk++)
                mma_ss_warp(tmem + 256, desc_plus(dRm, kk * 2048), desc_plus(dDKm, kk * 2048), idO, 1u);
#pragma unroll
            for (int kk = 0; kk < 8; kk++)
                mma_ss_warp(tmem + 384, desc_plus(dRm, kk * 2048), desc_plus(dDZm, kk * 2048), idO,
                            (mt > 0 || kk > 0) ? 1u : 0u);
            mma_commit_warp(mma_bar);
        }
        mma_issued++;
        if (!(ok = wait_block(mma_bar, mma_done & 1, w))) break;
        mma_done++;
        tc_fence_after();
    }
    if (ok) {   // thread (m, half): key m of the block, the half's 64 columns
        const bool key_ok = r < p.b2;
        const int64_t tok = (int64_t)bh * p.N + (int64_t)up * p.b2 + r;
#pragma unroll 1
        for (int ch = 2 * half; ch < 2 * half + 2; ch++) {
            float o[32], u[32];
            tmem_ld32f(tl + 256 + ch * 32, o);
            tmem_ld32f(tl + 384 + ch * 32, u);
            tmem_wait_ld();
            if (key_ok) {
                uint4 *pk = reinterpret_cast<uint4 *>(a.dk + tok * kD + ch * 32);
                uint4 *pv = reinterpret_cast<uint4 *>(a.dv + tok * kD + ch * 32);
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    pk[e] = make_uint4(pack_bf16(o[8 * e], o[8 * e + 1]), pack_bf16(o[8 * e + 2], o[8 * e + 3]),
                                       pack_bf16(o[8 * e + 4], o[8 * e + 5]), pack_bf16(o[8 * e + 6], o[8 * e + 7]));
                    pv[e] = make_uint4(pack_bf16(u[8 * e], u[8 * e + 1]), pack_bf16(u[8 * e + 2], u[8 * e + 3]),
                                       pack_bf16(u[8 * e + 4], u[8 * e + 5]), pack_bf16(u[8 * e + 6], u[8 * e + 7]));
                }
            }
        }
    }
    if (threadIdx.x == 0 && ld_issued > ld_done)
        wait_phase_cleanup(ld_bar, (ld_issued - 1) & 1, kCleanupPolls);
    if (warp == 0 && mma_issued > mma_done)
        wait_phase_cleanup(mma_bar, (mma_issued - 1) & 1, kCleanupPolls);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// dq̄ partial sums: unit (bh, row tile mt, chunk ch of upc blocks): sum over the
// chunk's blocks of (s da) K, one tcgen05 product per block (K = the block's keys).
// The blocks stream through a ring of three or four stages, so that the copies of
// the next blocks are in flight while the tensor cores work on this one.
template <int B2P>
__global__ void __launch_bounds__(128, 1)
tc_bwd_dqbar_kernel(const __grid_constant__ CUtensorMap tmDA, const __grid_constant__ CUtensorMap tmK,
                    RbArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    const Problem &p = a.p;
    using C = rb::Dq<B2P>;
    constexpr int NS = C::kNS;
    uint64_t *ld_bar = reinterpret_cast<uint64_t *>(sm + C::kBar);   // [NS]: stage loaded
    uint64_t *mma_bar = ld_bar + NS;                                  // [NS]: stage read
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(ld_bar + 2 * NS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(ld_bar + 2 * NS + 1);
    const int warp = threadIdx.x >> 5, r = threadIdx.x;
    int unit = blockIdx.x;
    const int ch = unit % a.nch;
    unit /= a.nch;
    const int mt = unit % a.nmt, bh = unit / a.nmt;
    const int u_lo = ch * a.upc, u_hi = min(p.b1k, u_lo + a.upc), nb = max(0, u_hi - u_lo);
    constexpr uint32_t kPanelKV = B2P * 128;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2 * NS; i++) mbar_init(ld_bar + i, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, 128);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    const WaitCtx w{a.limit, a.status, abort_flag};
    uint32_t ld_issued[NS], ld_done[NS], mma_issued[NS], mma_done[NS];
#pragma unroll
    for (int st = 0; st < NS; st++) ld_issued[st] = ld_done[st] = mma_issued[st] = mma_done[st] = 0;
    constexpr uint32_t idO = idesc_bf16(128, 128, 0, 1);
    // block i of the chunk into stage i % NS (thread 0 issues the copies)
    auto load = [&](int i) {
        const int st = i % NS, up = u_lo + i;
        if (threadIdx.x == 0) {
            uint8_t *base = sm + st * C::kStage;
            const int tok0 = up * p.b2, hh = bh % p.H, bb = bh / p.H;
            mbar_expect_tx(ld_bar + st, 2 * kPanel + 2 * kPanelKV);
            for (int pn = 0; pn < 2; pn++) {
                tma_load_5d(base + pn * kPanel, &tmDA, 0, mt * 128, pn, up, bh, ld_bar + st);
                tma_load_4d(base + kTile + pn * kPanelKV, &tmK, pn * 64, tok0, hh, bb, ld_bar + st);
            }
        }
        ld_issued[st]++;
    };
    for (int i = 0; i < NS && i < nb; i++) load(i);
    bool ok = true;
    for (int i = 0; ok && i < nb; i++) {
        const int st = i % NS;
        if (!(ok = wait_block(ld_bar + st, (i / NS) & 1, w))) break;
        ld_done[st]++;
        if (warp == 0) {
            tc_fence_after();
            const uint64_t dA = smem_desc_sw128(smem_u32(sm + st * C::kStage), 16, 1024);
            const uint64_t dK = smem_desc_sw128(smem_u32(sm + st * C::kStage + kTile), kPanelKV, 1024);   // MN-major
#pragma unroll
            for (int kk = 0; kk < B2P / 16; kk++)
                mma_ss_warp(tmem, desc_plus(dA, (kk >> 2) * kPanel + (kk & 3) * 32),
                            desc_plus(dK, kk * 2048), idO, (i > 0 || kk > 0) ? 1u : 0u);
            mma_commit_warp(mma_bar + st);
        }
        mma_issued[st]++;
        // the previous block's products are done with its stage: refill it NS blocks on
        // (block i's products keep the tensor cores busy meanwhile)
        if (i >= 1 && i - 1 + NS < nb) {
            const int sp = (i - 1) % NS;
            if (!(ok = wait_block(mma_bar + sp, ((i - 1) / NS) & 1, w))) break;
            mma_done[sp]++;
            load(i - 1 + NS);
        }
    }
    if (ok && nb > 0) {   // the last block's commit covers every product before it
        const int sl = (nb - 1) % NS;
        if ((ok = wait_block(mma_bar + sl, ((nb - 1) / NS) & 1, w))) mma_done[sl]++;
        tc_fence_after();
    }
    if (ok) {
        float *dst = a.part + ((((int64_t)bh * a.nmt + mt) * a.nch + ch) * 128 + r) * 128;
#pragma unroll 1
        for (int cc = 0; cc < 4; cc++) {
            float o[32];
            if (u_hi > u_lo) {
                tmem_ld32f(tl + cc * 32, o);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int e = 0; e < 32; e++) o[e] = 0.f;
            }
            float4 *d4 = reinterpret_cast<float4 *>(dst + cc * 32);
#pragma unroll
            for (int e = 0; e < 8; e++) d4[e] = make_float4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
        }
    }
    // drain this CTA's own copies and products before its tensor memory is freed (a
    // phase that completed unobserved satisfies its wait at once)
#pragma unroll
    for (int st = 0; st < NS; st++) {
        if (threadIdx.x == 0 && ld_issued[st] > ld_done[st])
            wait_phase_cleanup(ld_bar + st, (ld_issued[st] - 1) & 1, kCleanupPolls);
        if (warp == 0 && mma_issued[st] > mma_done[st])
            wait_phase_cleanup(mma_bar + st, (mma_issued[st] - 1) & 1, kCleanupPolls);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

// dq̄ = the sum of the chunks' partials, in a fixed order (chunk 0, 1, ...), written
// over chunk 0: one thread per four elements of a (bh, row tile) stack, so every
// row's sum is taken once rather than once per query of its tile.
__global__ void tc_bwd_reduce_kernel(float *__restrict__ part, int64_t stacks, int nch) {
    const int64_t per = 128 * 128 / 4, total = stacks * per;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        float4 *src = reinterpret_cast<float4 *>(part) + (idx / per) * nch * per + idx % per;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int c2 = 0; c2 < nch; c2++) {
            const float4 x = src[(int64_t)c2 * per];
            acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
        }
        src[0] = acc;
    }
}

// dq = dq_L + dq̄[g][v] / |T_g| (the aggregation's mean), bfloat16 output; dq̄ is
// chunk 0 of each stack after tc_bwd_reduce_kernel.
__global__ void tc_bwd_combine_kernel(const float *__restrict__ dql, const float *__restrict__ part,
                                      __nv_bfloat16 *__restrict__ dq, Problem p, int nmt, int nch) {
    const int64_t total = (int64_t)p.BH * p.N * (kD / 4);
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t tok = idx / (kD / 4);
        const int j = (int)(idx % (kD / 4)) * 4;
        const int bh = (int)(tok / p.N), n = (int)(tok % p.N);
        const int u = n / p.b2, v = n % p.b2;
        int g = (int)(((int64_t)u * p.tiles) / p.b1);
        while (g + 1 < p.tiles && tile_begin(g + 1, p.b1, p.tiles) <= u) g++;
        const float inv = 1.f / (float)(tile_begin(g + 1, p.b1, p.tiles) - tile_begin(g, p.b1, p.tiles));
        const int rgl = g * p.b2 + v, mt = rgl / 128, rl = rgl % 128;
        const float4 acc =
            *reinterpret_cast<const float4 *>(part + (((int64_t)bh * nmt + mt) * nch * 128 + rl) * 128 + j);
        const float4 l4 = *reinterpret_cast<const float4 *>(dql + tok * kD + j);
        uint2 o;
        o.x = pack_bf16(l4.x + acc.x * inv, l4.y + acc.y * inv);
        o.y = pack_bf16(l4.z + acc.z * inv, l4.w + acc.w * inv);
        *reinterpret_cast<uint2 *>(dq + tok * kD + j) = o;
    }
}

}  // namespace

bool sm100_backward_supports(const Problem &p, monarch_dtype dtype) {
    return p.iters == 1 && !p.key_tiles && p.layout == kLayoutBHND && p.b1k == p.b1 &&
           p.unit_begin == 0 && p.unit_end == p.BH * p.tiles && sm100_supports(p, dtype);
}

namespace {

// Layout of the backward's workspace (tensor-core path).
struct BwTc {
    TcWorkspace fw;              // the forward's q̄, Ktil, Z, entropy panels; lam
    float *delta, *dql, *dhr, *part;
    __nv_bfloat16 *dktb, *dzb, *da;
    int nmt, upc, nch;
};
constexpr int kBlocksPerChunk = 32;   // blocks u' per dq̄ partial sum

size_t bw_tc_layout(const Problem &p, void *base, BwTc *out) {
    bool overflow = false;
    const size_t nq = (size_t)p.BH * p.N, rr = (size_t)p.tiles * p.b2;
    const int nmt = (int)((rr + 127) / 128), nch = (p.b1k + kBlocksPerChunk - 1) / kBlocksPerChunk;
    const size_t sizes[9] = {
        al256(sm100_workspace_bytes(p, overflow)),            // forward intermediates
        al256(nq * 32),                                       // lam panels
        al256(nq * 4),                                        // delta
        al256(nq * kD * 4),                                   // dql
        al256((size_t)p.BH * p.b1k * rr * 4),                 // dH rows
        al256((size_t)p.BH * p.b1k * rr * kD * 2),            // dKtil (bf16)
        al256((size_t)p.BH * p.b1k * rr * kD * 2),            // dZ (bf16)
        al256((size_t)p.BH * p.b1k * rr * kD * 2),            // s*da (bf16, keys padded to 128)
        al256((size_t)p.BH * nmt * nch * 128 * 128 * 4)};     // dq̄ partial sums
    size_t off[9], total = 0;
    for (int i = 0; i < 9; i++) {
        off[i] = total;
        total += sizes[i];
    }
    if (out) {
        char *c = (char *)base;
        out->fw = carve(p, c);
        out->fw.lam = (uint4 *)(c + off[1]);
        out->delta = (float *)(c + off[2]);
        out->dql = (float *)(c + off[3]);
        out->dhr = (float *)(c + off[4]);
        out->dktb = (__nv_bfloat16 *)(c + off[5]);
        out->dzb = (__nv_bfloat16 *)(c + off[6]);
        out->da = (__nv_bfloat16 *)(c + off[7]);
        out->part = (float *)(c + off[8]);
        out->nmt = nmt;
        out->upc = kBlocksPerChunk;
        out->nch = nch;
    }
    return total;
}

// stage 0: tc_bwd_r_kernel (dk, dv, s*da); stage 1: tc_bwd_dqbar_kernel (dq̄ partial sums)
template <int B2P>
cudaError_t launch_bwd_r(const CUtensorMap *m, const RbArgs &a, int stage, cudaStream_t s) {
    if (stage == 0) {
        const cudaError_t e = set_smem(tc_bwd_r_kernel<B2P>, rb::kSmem);
        if (e != cudaSuccess) return e;
        tc_bwd_r_kernel<B2P><<<(unsigned)(a.p.BH * a.p.b1k), 256, rb::kSmem, s>>>(m[0], m[1], m[2],
                                                                               m[3], m[4], a);
    } else {
        const cudaError_t e = set_smem(tc_bwd_dqbar_kernel<B2P>, rb::Dq<B2P>::kSmem);
        if (e != cudaSuccess) return e;
        tc_bwd_dqbar_kernel<B2P><<<(unsigned)(a.p.BH * a.nmt * a.nch), 128, rb::Dq<B2P>::kSmem, s>>>(
            m[5], m[1], a);
    }
    return cudaGetLastError();
}

}  // namespace

size_t sm100_backward_workspace_bytes(const Problem &p, bool &overflow) {
    overflow = false;
    return bw_tc_layout(p, nullptr, nullptr);
}

cudaError_t sm100_backward(const Problem &p, const void *q, const void *k, const void *v,
                           const void *dy, void *dq, void *dk, void *dv, void *workspace,
                           int *status, long long wait_limit, cudaStream_t stream) {
    BwTc w;
    bw_tc_layout(p, workspace, &w);
    const TcWorkspace &ws = w.fw;
    const float c_log2 = p.scale * kLog2e;
    // the forward on the tensor cores: q̄, the R-step (R in two bfloat16 parts, so that
    // Ktil and Z are exact to about 2^-16 before their own rounding) and the L-step's
    // row statistics lam
    cudaError_t e = run_qbar(p, q, ws, stream);
    if (e == cudaSuccess) e = run_rstep(p, ws, k, v, 0, c_log2, status, wait_limit, 0, stream, 1);
    if (e == cudaSuccess) e = run_lstep(p, ws, q, nullptr, kLsStat, c_log2, status, wait_limit, 0, stream);
    if (e != cudaSuccess) return e;
    const uint64_t rr = (uint64_t)p.tiles * p.b2, slab = (uint64_t)key_slab(p);
    const uint64_t dkz[5] = {64, rr, 2, slab, (uint64_t)p.BH};
    const uint64_t skz[4] = {128, rr * 128, 2 * rr * 128, slab * 2 * rr * 128};
    const uint32_t bkz[5] = {64, 1, 1, 128, 1};    // 128 blocks u' of one row r
    const uint32_t bkz64[5] = {64, 1, 1, 64, 1};   // 64 blocks u' of one row r
    const uint32_t brow[5] = {64, 128, 1, 1, 1};   // 128 rows r of one block u'
    CUtensorMap mq, mdy, mkt, mz, mkt64, mz64;
    if (!map_queries(&mq, q, p) || !map_queries(&mdy, dy, p) ||
        !make_map(&mkt, ws.ktil, 5, dkz, skz, bkz) || !make_map(&mz, ws.z, 5, dkz, skz, bkz) ||
        !make_map(&mkt64, ws.ktil, 5, dkz, skz, bkz64) || !make_map(&mz64, ws.z, 5, dkz, skz, bkz64))
        return cudaErrorInvalidValue;
    CUtensorMap rm[6];
    const int mpad = qbar_tiles(p) * 128, b2p = b2_padded(p.b2);
    const uint64_t dq2[2] = {(uint64_t)kD, (uint64_t)p.BH * mpad};
    const uint64_t sq2[1] = {kD * 2};
    const uint32_t bq2[2] = {64, 128};
    if (!make_map(&rm[0], ws.qbar, 2, dq2, sq2, bq2) || !map_keys(&rm[1], k, p, (uint32_t)b2p) ||
        !map_keys(&rm[2], v, p, (uint32_t)b2p) || !make_map(&rm[3], w.dktb, 5, dkz, skz, brow) ||
        !make_map(&rm[4], w.dzb, 5, dkz, skz, brow) || !make_map(&rm[5], w.da, 5, dkz, skz, brow))
        return cudaErrorInvalidValue;
    if ((e = set_smem(tc_bwd_dkz_kernel, lb::kSmem)) != cudaSuccess ||
        (e = set_smem(tc_bwd_dq_kernel<0>, lq::kSmem)) != cudaSuccess ||
        (e = set_smem(tc_bwd_dq_kernel<1>, lq::kSmem)) != cudaSuccess)
        return e;
    LbArgs la{p, ws.hx, ws.lam, w.delta, w.dktb, w.dzb, w.dhr, w.dql, c_log2, (p.b1k + 127) / 128,
              (tile_max_rows(p.b1, p.tiles) + 127) / 128, status, wait_limit};
    const int64_t probs = (int64_t)p.BH * p.tiles * p.b2, npair = (la.nqt + 1) / 2;
    {
        ProfileScope scope(K_TC_BWD_DELTA, stream);
        tc_bwd_dq_kernel<0><<<(unsigned)(probs * npair), 256, lq::kSmem, stream>>>(mq, mdy, mkt64, mz64, la);
    }
    {
        ProfileScope scope(K_TC_BWD_DKZ, stream);
        tc_bwd_dkz_kernel<<<(unsigned)(probs * la.nkb), 256, lb::kSmem, stream>>>(mq, mdy, mkt, mz, la);
    }
    {
        ProfileScope scope(K_TC_BWD_DQ, stream);
        tc_bwd_dq_kernel<1><<<(unsigned)(probs * npair), 256, lq::kSmem, stream>>>(mq, mdy, mkt64, mz64, la);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    RbArgs ra{p, mpad, w.dhr, w.da, (__nv_bfloat16 *)dk, (__nv_bfloat16 *)dv, w.part, w.nmt, w.nch,
              w.upc, status, wait_limit};
    auto launch_r = [&](int stage) -> cudaError_t {
        switch (b2p) {
            case 16: return launch_bwd_r<16>(rm, ra, stage, stream);
            case 32: return launch_bwd_r<32>(rm, ra, stage, stream);
            case 48: return launch_bwd_r<48>(rm, ra, stage, stream);
            case 64: return launch_bwd_r<64>(rm, ra, stage, stream);
            case 80: return launch_bwd_r<80>(rm, ra, stage, stream);
            case 96: return launch_bwd_r<96>(rm, ra, stage, stream);
            case 112: return launch_bwd_r<112>(rm, ra, stage, stream);
            case 128: return launch_bwd_r<128>(rm, ra, stage, stream);
            default: return cudaErrorInvalidValue;
        }
    };
    {
        ProfileScope scope(K_TC_BWD_R, stream);
        if ((e = launch_r(0)) != cudaSuccess) return e;
    }
    ProfileScope scope(K_TC_BWD_DQBAR, stream);
    if ((e = launch_r(1)) != cudaSuccess) return e;
    const int64_t stacks = (int64_t)p.BH * w.nmt, rtotal = stacks * 128 * 128 / 4;
    const int rblocks = (int)((rtotal + 255) / 256 < 148 * 32 ? (rtotal + 255) / 256 : 148 * 32);
    tc_bwd_reduce_kernel<<<rblocks, 256, 0, stream>>>(w.part, stacks, w.nch);
    const int64_t total = (int64_t)p.BH * p.N * (kD / 4);
    const int blocks = (int)((total + 255) / 256 < 148 * 32 ? (total + 255) / 256 : 148 * 32);
    tc_bwd_combine_kernel<<<blocks, 256, 0, stream>>>(w.dql, w.part, (__nv_bfloat16 *)dq, p, w.nmt,
                                                      w.nch);
    return cudaGetLastError();
}

}  // namespace monarch
