// monarch_bwd.cu -- backward pass of the Monarch attention (one iteration):
// the gradients dq, dk, dv of a scalar loss given dy, by the chain rule through
// the output, the L-step, the R-step and the query aggregation.  The pages
// describe finetuning through the Monarch attention (summary page, "Approach";
// explainer page, "创新三：微调与高效内核") but print no backward; this is the
// derivative of the forward map of the generic kernels, step by step:
//
//   L-step and output, per query row (u, v) of tile g, keys u' (blocks):
//     b = s q.Ktil[u'] + H[u'],  L = softmax(b),  y = sum L Z
//     delta = dy.y,  dL = dy.Z[u'],  db = L (dL - delta)
//     dq_(u,v) += s sum_u' db Ktil[u'];  dKtil[u'] += s sum_u db q;
//     dZ[u'] += sum_u L dy;  dH[u'] += sum_u db
//   R-step, per row v of R_{u',g}, keys v' of block u':
//     a = s qbar.k_(u',v'),  R = softmax(a),  E = sum R a,
//     dR = dKtil.k_(u',v') + dZ.v_(u',v'),  rho = sum R dR,
//     da = R (dR - rho) - dH R (a - E)          (dH/da = -R (a - E))
//     dqbar += s sum_v' da k_(u',v');  dk_(u',v') += sum_(g,v) s da qbar + R dKtil;
//     dv_(u',v') += sum_(g,v) R dZ
//   Aggregation: dq_(u,v) += dqbar[g][v] / |T_g|.
//
// SIMT kernels with float32 arithmetic for every supported shape and dtype
// (bfloat16 with d = 128 takes the tensor-core backward of monarch_sm100.cu).
// Each gradient element is written by exactly one warp (no atomics): the
// kernels are deterministic.  One warp per row; a CTA of GW warps shares chunks
// of KC rows staged in shared memory (rows padded to d+1 floats).
#include "monarch_common.cuh"
#include "monarch_sm100.cuh"

#include <math.h>

namespace monarch {

namespace {

constexpr int GW = 8;    // warps (rows) per CTA
constexpr int KC = 32;   // rows per shared-memory chunk

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Query rows (u, v) of tile g: the CTA covers GW consecutive u of one (bh, g, v).
struct QueryRow {
    int bh, g, v, u, u0, u1;
    bool active;
    int64_t bhg, tok;
};
__device__ __forceinline__ QueryRow query_row(const Problem &p) {
    QueryRow r;
    const int nug = (tile_max_rows(p.b1, p.tiles) + GW - 1) / GW;
    int64_t bid = blockIdx.x;
    const int ug = (int)(bid % nug);
    bid /= nug;
    r.v = (int)(bid % p.b2);
    bid /= p.b2;
    r.g = (int)(bid % p.tiles);
    r.bh = (int)(bid / p.tiles);
    r.u0 = tile_begin(r.g, p.b1, p.tiles);
    r.u1 = tile_begin(r.g + 1, p.b1, p.tiles);
    r.u = r.u0 + ug * GW + (int)(threadIdx.x >> 5);
    r.active = r.u < r.u1;
    r.bhg = (int64_t)r.bh * p.tiles + r.g;
    r.tok = (int64_t)r.bh * p.N + (int64_t)r.u * p.b2 + r.v;
    return r;
}

// B1: per query row, the L-step's log-sum-exp and delta = dy.y (y recomputed).
template <typename T, int D>
__global__ void __launch_bounds__(GW * 32)
bwd_lstats_kernel(const T *__restrict__ q, const T *__restrict__ dy,
                  const float *__restrict__ ktil, const float *__restrict__ z,
                  const float *__restrict__ hent, float *__restrict__ lse,
                  float *__restrict__ delta, Problem p) {
    constexpr int DS = D + 1, NJ = D / 32;
    extern __shared__ float sm[];
    float *sq = sm;               // [GW][D]
    float *sk = sq + GW * D;      // [KC][DS]
    float *sz = sk + KC * DS;     // [KC][DS]
    float *sh = sz + KC * DS;     // [KC]
    const QueryRow r = query_row(p);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (r.active)
        for (int j = lane; j < D; j += 32) sq[warp * D + j] = to_f32(q[r.tok * D + j]);
    const int64_t kbase = (r.bhg * p.b2 + r.v) * p.b1k;
    float m = -INFINITY, l = 0.f, acc[NJ];
#pragma unroll
    for (int i = 0; i < NJ; i++) acc[i] = 0.f;
    for (int c0 = 0; c0 < p.b1k; c0 += KC) {
        const int nk = min(KC, p.b1k - c0);
        __syncthreads();
        for (int idx = threadIdx.x; idx < nk * D; idx += blockDim.x) {
            const int rr = idx / D, j = idx % D;
            sk[rr * DS + j] = ktil[(kbase + c0 + rr) * D + j];
            sz[rr * DS + j] = z[(kbase + c0 + rr) * D + j];
        }
        if (threadIdx.x < nk) sh[threadIdx.x] = hent[kbase + c0 + threadIdx.x];
        __syncthreads();
        if (!r.active) continue;
        float b = -INFINITY;
        if (lane < nk) {
            float a = 0.f;
#pragma unroll 8
            for (int j = 0; j < D; j++) a = fmaf(sq[warp * D + j], sk[lane * DS + j], a);
            b = a * p.scale + sh[lane];
        }
        const float mn = fmaxf(m, warp_max(b));
        const float alpha = (m == -INFINITY) ? 0.f : expf(m - mn);
        const float e = lane < nk ? expf(b - mn) : 0.f;
        l = l * alpha + warp_sum(e);
        m = mn;
#pragma unroll
        for (int i = 0; i < NJ; i++) acc[i] *= alpha;
        for (int rr = 0; rr < nk; rr++) {
            const float er = __shfl_sync(0xffffffffu, e, rr);
#pragma unroll
            for (int i = 0; i < NJ; i++) acc[i] = fmaf(er, sz[rr * DS + lane + 32 * i], acc[i]);
        }
    }
    if (r.active) {
        float dd = 0.f;
#pragma unroll
        for (int i = 0; i < NJ; i++) dd = fmaf(to_f32(dy[r.tok * D + lane + 32 * i]), acc[i], dd);
        dd = warp_sum(dd) / l;
        if (lane == 0) {
            lse[r.tok] = m + logf(l);
            delta[r.tok] = dd;
        }
    }
}

// B2: per query row, the L-step's part of dq: s sum_u' db Ktil[u'].
template <typename T, int D>
__global__ void __launch_bounds__(GW * 32)
bwd_ldq_kernel(const T *__restrict__ q, const T *__restrict__ dy,
               const float *__restrict__ ktil, const float *__restrict__ z,
               const float *__restrict__ hent, const float *__restrict__ lse,
               const float *__restrict__ delta, float *__restrict__ dql, Problem p) {
    constexpr int DS = D + 1, NJ = D / 32;
    extern __shared__ float sm[];
    float *sq = sm;               // [GW][D]
    float *sdy = sq + GW * D;     // [GW][D]
    float *sk = sdy + GW * D;     // [KC][DS]
    float *sz = sk + KC * DS;     // [KC][DS]
    float *sh = sz + KC * DS;     // [KC]
    const QueryRow r = query_row(p);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float lrow = 0.f, drow = 0.f;
    if (r.active) {
        for (int j = lane; j < D; j += 32) {
            sq[warp * D + j] = to_f32(q[r.tok * D + j]);
            sdy[warp * D + j] = to_f32(dy[r.tok * D + j]);
        }
        lrow = lse[r.tok];
        drow = delta[r.tok];
    }
    const int64_t kbase = (r.bhg * p.b2 + r.v) * p.b1k;
    float acc[NJ];
#pragma unroll
    for (int i = 0; i < NJ; i++) acc[i] = 0.f;
    for (int c0 = 0; c0 < p.b1k; c0 += KC) {
        const int nk = min(KC, p.b1k - c0);
        __syncthreads();
        for (int idx = threadIdx.x; idx < nk * D; idx += blockDim.x) {
            const int rr = idx / D, j = idx % D;
            sk[rr * DS + j] = ktil[(kbase + c0 + rr) * D + j];
            sz[rr * DS + j] = z[(kbase + c0 + rr) * D + j];
        }
        if (threadIdx.x < nk) sh[threadIdx.x] = hent[kbase + c0 + threadIdx.x];
        __syncthreads();
        if (!r.active) continue;
        float db = 0.f;
        if (lane < nk) {
            float a = 0.f, dl = 0.f;
#pragma unroll 8
            for (int j = 0; j < D; j++) {
                a = fmaf(sq[warp * D + j], sk[lane * DS + j], a);
                dl = fmaf(sdy[warp * D + j], sz[lane * DS + j], dl);
            }
            const float L = expf(a * p.scale + sh[lane] - lrow);
            db = L * (dl - drow);
        }
        for (int rr = 0; rr < nk; rr++) {
            const float dbr = __shfl_sync(0xffffffffu, db, rr);
#pragma unroll
            for (int i = 0; i < NJ; i++) acc[i] = fmaf(dbr, sk[rr * DS + lane + 32 * i], acc[i]);
        }
    }
    if (r.active)
#pragma unroll
        for (int i = 0; i < NJ; i++) dql[r.tok * D + lane + 32 * i] = acc[i] * p.scale;
}

// B3: per (bh, g, v, u'), the L-step's gradients of its keys, values and bias:
// dKtil, dZ, dH summed over the query rows u of tile g.  The CTA covers GW
// consecutive u' of one (bh, g, v) and stages the tile's query rows in chunks.
template <typename T, int D>
__global__ void __launch_bounds__(GW * 32)
bwd_ldkz_kernel(const T *__restrict__ q, const T *__restrict__ dy,
                const float *__restrict__ ktil, const float *__restrict__ z,
                const float *__restrict__ hent, const float *__restrict__ lse,
                const float *__restrict__ delta, float *__restrict__ dkt,
                float *__restrict__ dz, float *__restrict__ dh, Problem p) {
    constexpr int DS = D + 1, NJ = D / 32;
    extern __shared__ float sm[];
    float *skw = sm;              // [GW][D]  this warp's Ktil row
    float *szw = skw + GW * D;    // [GW][D]  this warp's Z row
    float *sq = szw + GW * D;     // [KC][DS] query rows of the chunk
    float *sdy = sq + KC * DS;    // [KC][DS] their dy rows
    float *sl = sdy + KC * DS;    // [KC]     their log-sum-exp
    float *sd = sl + KC;          // [KC]     their delta
    const int nkg = (p.b1k + GW - 1) / GW;
    int64_t bid = blockIdx.x;
    const int kg = (int)(bid % nkg);
    bid /= nkg;
    const int v = (int)(bid % p.b2);
    bid /= p.b2;
    const int g = (int)(bid % p.tiles);
    const int bh = (int)(bid / p.tiles);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int up = kg * GW + warp;
    const bool active = up < p.b1k;
    const int64_t bhg = (int64_t)bh * p.tiles + g;
    const int64_t krow = (bhg * p.b2 + v) * p.b1k + up;
    float hw = 0.f;
    if (active) {
        for (int j = lane; j < D; j += 32) {
            skw[warp * D + j] = ktil[krow * D + j];
            szw[warp * D + j] = z[krow * D + j];
        }
        hw = hent[krow];
    }
    const int u0 = tile_begin(g, p.b1, p.tiles), u1 = tile_begin(g + 1, p.b1, p.tiles);
    float ak[NJ], az[NJ], ah = 0.f;
#pragma unroll
    for (int i = 0; i < NJ; i++) ak[i] = az[i] = 0.f;
    for (int c0 = u0; c0 < u1; c0 += KC) {
        const int nr = min(KC, u1 - c0);
        __syncthreads();
        for (int idx = threadIdx.x; idx < nr * D; idx += blockDim.x) {
            const int rr = idx / D, j = idx % D;
            const int64_t tok = (int64_t)bh * p.N + (int64_t)(c0 + rr) * p.b2 + v;
            sq[rr * DS + j] = to_f32(q[tok * D + j]);
            sdy[rr * DS + j] = to_f32(dy[tok * D + j]);
        }
        if (threadIdx.x < nr) {
            const int64_t tok = (int64_t)bh * p.N + (int64_t)(c0 + threadIdx.x) * p.b2 + v;
            sl[threadIdx.x] = lse[tok];
            sd[threadIdx.x] = delta[tok];
        }
        __syncthreads();
        if (!active) continue;
        float L = 0.f, db = 0.f;
        if (lane < nr) {
            float a = 0.f, dl = 0.f;
#pragma unroll 8
            for (int j = 0; j < D; j++) {
                a = fmaf(sq[lane * DS + j], skw[warp * D + j], a);
                dl = fmaf(sdy[lane * DS + j], szw[warp * D + j], dl);
            }
            L = expf(a * p.scale + hw - sl[lane]);
            db = L * (dl - sd[lane]);
        }
        ah += db;
        for (int rr = 0; rr < nr; rr++) {
            const float dbr = __shfl_sync(0xffffffffu, db, rr);
            const float lr = __shfl_sync(0xffffffffu, L, rr);
#pragma unroll
            for (int i = 0; i < NJ; i++) {
                ak[i] = fmaf(dbr, sq[rr * DS + lane + 32 * i], ak[i]);
                az[i] = fmaf(lr, sdy[rr * DS + lane + 32 * i], az[i]);
            }
        }
    }
    if (active) {
#pragma unroll
        for (int i = 0; i < NJ; i++) {
            dkt[krow * D + lane + 32 * i] = ak[i] * p.scale;
            dz[krow * D + lane + 32 * i] = az[i];
        }
        ah = warp_sum(ah);
        if (lane == 0) dh[krow] = ah;
    }
}

// B4: per R row (bh, g, v, u'), the statistics of the R-step backward in one
// online pass over the b2 keys of block u': the log-sum-exp of a, E = sum R a
// and rho = sum R dR.  The CTA covers GW consecutive v of one (bh, g, u').
template <typename T, int D>
__global__ void __launch_bounds__(GW * 32)
bwd_rstats_kernel(const T *__restrict__ k, const T *__restrict__ v,
                  const float *__restrict__ qbar, const float *__restrict__ dkt,
                  const float *__restrict__ dz, float *__restrict__ lsea,
                  float *__restrict__ ea, float *__restrict__ rho, Problem p) {
    constexpr int DS = D + 1;
    extern __shared__ float sm[];
    float *sqb = sm;              // [GW][D] qbar row
    float *sdk = sqb + GW * D;    // [GW][D] dKtil row
    float *sdz = sdk + GW * D;    // [GW][D] dZ row
    float *sk = sdz + GW * D;     // [KC][DS]
    float *sv = sk + KC * DS;     // [KC][DS]
    const int nvg = (p.b2 + GW - 1) / GW;
    int64_t bid = blockIdx.x;
    const int vg = (int)(bid % nvg);
    bid /= nvg;
    const int up = (int)(bid % p.b1k);
    bid /= p.b1k;
    const int g = (int)(bid % p.tiles);
    const int bh = (int)(bid / p.tiles);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int vrow = vg * GW + warp;
    const bool active = vrow < p.b2;
    const int64_t bhg = (int64_t)bh * p.tiles + g;
    const int64_t rrow = (bhg * p.b2 + vrow) * p.b1k + up;
    if (active)
        for (int j = lane; j < D; j += 32) {
            sqb[warp * D + j] = qbar[(bhg * p.b2 + vrow) * D + j];
            sdk[warp * D + j] = dkt[rrow * D + j];
            sdz[warp * D + j] = dz[rrow * D + j];
        }
    const int64_t base = ((int64_t)bh * p.Nk + (int64_t)up * p.b2) * D;
    float m = -INFINITY, l = 0.f, sa = 0.f, sr = 0.f;
    for (int c0 = 0; c0 < p.b2; c0 += KC) {
        const int nk = min(KC, p.b2 - c0);
        __syncthreads();
        for (int idx = threadIdx.x; idx < nk * D; idx += blockDim.x) {
            const int rr = idx / D, j = idx % D;
            sk[rr * DS + j] = to_f32(k[base + (int64_t)(c0 + rr) * D + j]);
            sv[rr * DS + j] = to_f32(v[base + (int64_t)(c0 + rr) * D + j]);
        }
        __syncthreads();
        if (!active) continue;
        float a = -INFINITY, dr = 0.f;
        if (lane < nk) {
            float x = 0.f, y = 0.f;
#pragma unroll 8
            for (int j = 0; j < D; j++) {
                x = fmaf(sqb[warp * D + j], sk[lane * DS + j], x);
                y = fmaf(sdk[warp * D + j], sk[lane * DS + j], y);
                y = fmaf(sdz[warp * D + j], sv[lane * DS + j], y);
            }
            a = x * p.scale;
            dr = y;
        }
        const float mn = fmaxf(m, warp_max(a));
        const float alpha = (m == -INFINITY) ? 0.f : expf(m - mn);
        const float e = lane < nk ? expf(a - mn) : 0.f;
        l = l * alpha + warp_sum(e);
        sa = sa * alpha + warp_sum(lane < nk ? e * a : 0.f);
        sr = sr * alpha + warp_sum(e * dr);
        m = mn;
    }
    if (active && lane == 0) {
        lsea[rrow] = m + logf(l);
        ea[rrow] = sa / l;
        rho[rrow] = sr / l;
    }
}

// The R-step backward's logit gradient of one (row, key) pair.
__device__ __forceinline__ void r_grad(float a, float dr, float lse_a, float e_a, float rho_r,
                                       float dh, float &R, float &da) {
    R = expf(a - lse_a);
    da = R * (dr - rho_r) - dh * R * (a - e_a);
}

// B5: per (bh, g, v), dqbar = s sum_u' sum_v' da k_(u',v').  The CTA covers GW
// consecutive v of one (bh, g) and walks every key block u' in chunks.
template <typename T, int D>
__global__ void __launch_bounds__(GW * 32)
bwd_rdqbar_kernel(const T *__restrict__ k, const T *__restrict__ v,
                  const float *__restrict__ qbar, const float *__restrict__ dkt,
                  const float *__restrict__ dz, const float *__restrict__ dh,
                  const float *__restrict__ lsea, const float *__restrict__ ea,
                  const float *__restrict__ rho, float *__restrict__ dqbar, Problem p) {
    constexpr int DS = D + 1, NJ = D / 32;
    extern __shared__ float sm[];
    float *sqb = sm;              // [GW][D]
    float *sdk = sqb + GW * D;    // [GW][D] dKtil row of (g, v, u')
    float *sdz = sdk + GW * D;    // [GW][D] dZ row of (g, v, u')
    float *sk = sdz + GW * D;     // [KC][DS]
    float *sv = sk + KC * DS;     // [KC][DS]
    const int nvg = (p.b2 + GW - 1) / GW;
    int64_t bid = blockIdx.x;
    const int vg = (int)(bid % nvg);
    bid /= nvg;
    const int g = (int)(bid % p.tiles);
    const int bh = (int)(bid / p.tiles);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int vrow = vg * GW + warp;
    const bool active = vrow < p.b2;
    const int64_t bhg = (int64_t)bh * p.tiles + g;
    if (active)
        for (int j = lane; j < D; j += 32) sqb[warp * D + j] = qbar[(bhg * p.b2 + vrow) * D + j];
    float acc[NJ];
#pragma unroll
    for (int i = 0; i < NJ; i++) acc[i] = 0.f;
    for (int up = 0; up < p.b1k; up++) {
        const int64_t rrow = (bhg * p.b2 + vrow) * p.b1k + up;
        float sl = 0.f, se = 0.f, sr = 0.f, shh = 0.f;
        if (active) {
            for (int j = lane; j < D; j += 32) {
                sdk[warp * D + j] = dkt[rrow * D + j];
                sdz[warp * D + j] = dz[rrow * D + j];
            }
            sl = lsea[rrow];
            se = ea[rrow];
            sr = rho[rrow];
            shh = dh[rrow];
        }
        const int64_t base = ((int64_t)bh * p.Nk + (int64_t)up * p.b2) * D;
        for (int c0 = 0; c0 < p.b2; c0 += KC) {
            const int nk = min(KC, p.b2 - c0);
            __syncthreads();
            for (int idx = threadIdx.x; idx < nk * D; idx += blockDim.x) {
                const int rr = idx / D, j = idx % D;
                sk[rr * DS + j] = to_f32(k[base + (int64_t)(c0 + rr) * D + j]);
                sv[rr * DS + j] = to_f32(v[base + (int64_t)(c0 + rr) * D + j]);
            }
            __syncthreads();
            if (!active) continue;
            float da = 0.f;
            if (lane < nk) {
                float x = 0.f, y = 0.f;
#pragma unroll 8
                for (int j = 0; j < D; j++) {
                    x = fmaf(sqb[warp * D + j], sk[lane * DS + j], x);
                    y = fmaf(sdk[warp * D + j], sk[lane * DS + j], y);
                    y = fmaf(sdz[warp * D + j], sv[lane * DS + j], y);
                }
                float R;
                r_grad(x * p.scale, y, sl, se, sr, shh, R, da);
            }
            for (int rr = 0; rr < nk; rr++) {
                const float dar = __shfl_sync(0xffffffffu, da, rr);
#pragma unroll
                for (int i = 0; i < NJ; i++) acc[i] = fmaf(dar, sk[rr * DS + lane + 32 * i], acc[i]);
            }
        }
    }
    if (active)
#pragma unroll
        for (int i = 0; i < NJ; i++) dqbar[(bhg * p.b2 + vrow) * D + lane + 32 * i] = acc[i] * p.scale;
}

// B6: per key token (bh, u', v'): dk = sum_(g,v) s da qbar[g][v] + R dKtil[g,v,u'],
// dv = sum_(g,v) R dZ[g,v,u'].  The CTA covers GW consecutive v' of one
// (bh, u') and stages the (g, v) rows in chunks.
template <typename T, int D>
__global__ void __launch_bounds__(GW * 32)
bwd_rdkv_kernel(const T *__restrict__ k, const T *__restrict__ v,
                const float *__restrict__ qbar, const float *__restrict__ dkt,
                const float *__restrict__ dz, const float *__restrict__ dh,
                const float *__restrict__ lsea, const float *__restrict__ ea,
                const float *__restrict__ rho, T *__restrict__ dk, T *__restrict__ dv,
                Problem p) {
    constexpr int DS = D + 1, NJ = D / 32;
    extern __shared__ float sm[];
    float *skw = sm;              // [GW][D] this warp's key
    float *svw = skw + GW * D;    // [GW][D] this warp's value
    float *sqb = svw + GW * D;    // [KC][DS] qbar rows of the chunk
    float *sdk = sqb + KC * DS;   // [KC][DS] dKtil rows
    float *sdz = sdk + KC * DS;   // [KC][DS] dZ rows
    float *sst = sdz + KC * DS;   // [4][KC]  lse_a, E, rho, dH
    const int nvg = (p.b2 + GW - 1) / GW;
    int64_t bid = blockIdx.x;
    const int vg = (int)(bid % nvg);
    bid /= nvg;
    const int up = (int)(bid % p.b1k);
    const int bh = (int)(bid / p.b1k);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int vp = vg * GW + warp;
    const bool active = vp < p.b2;
    const int64_t tok = (int64_t)bh * p.Nk + (int64_t)up * p.b2 + vp;
    if (active)
        for (int j = lane; j < D; j += 32) {
            skw[warp * D + j] = to_f32(k[tok * D + j]);
            svw[warp * D + j] = to_f32(v[tok * D + j]);
        }
    float ak[NJ], av[NJ];
#pragma unroll
    for (int i = 0; i < NJ; i++) ak[i] = av[i] = 0.f;
    const int nrows = p.tiles * p.b2;   // the (g, v) rows of this head
    for (int c0 = 0; c0 < nrows; c0 += KC) {
        const int nr = min(KC, nrows - c0);
        __syncthreads();
        for (int idx = threadIdx.x; idx < nr * D; idx += blockDim.x) {
            const int rr = idx / D, j = idx % D;
            const int64_t gv = (int64_t)bh * nrows + c0 + rr;   // (bh*t + g)*b2 + v
            sqb[rr * DS + j] = qbar[gv * D + j];
            sdk[rr * DS + j] = dkt[(gv * p.b1k + up) * D + j];
            sdz[rr * DS + j] = dz[(gv * p.b1k + up) * D + j];
        }
        if (threadIdx.x < nr) {
            const int64_t rrow = ((int64_t)bh * nrows + c0 + threadIdx.x) * p.b1k + up;
            sst[threadIdx.x] = lsea[rrow];
            sst[KC + threadIdx.x] = ea[rrow];
            sst[2 * KC + threadIdx.x] = rho[rrow];
            sst[3 * KC + threadIdx.x] = dh[rrow];
        }
        __syncthreads();
        if (!active) continue;
        float R = 0.f, da = 0.f;
        if (lane < nr) {
            float x = 0.f, y = 0.f;
#pragma unroll 8
            for (int j = 0; j < D; j++) {
                x = fmaf(sqb[lane * DS + j], skw[warp * D + j], x);
                y = fmaf(sdk[lane * DS + j], skw[warp * D + j], y);
                y = fmaf(sdz[lane * DS + j], svw[warp * D + j], y);
            }
            r_grad(x * p.scale, y, sst[lane], sst[KC + lane], sst[2 * KC + lane],
                   sst[3 * KC + lane], R, da);
        }
        for (int rr = 0; rr < nr; rr++) {
            const float dar = __shfl_sync(0xffffffffu, da, rr) * p.scale;
            const float rr_ = __shfl_sync(0xffffffffu, R, rr);
#pragma unroll
            for (int i = 0; i < NJ; i++) {
                ak[i] = fmaf(dar, sqb[rr * DS + lane + 32 * i], ak[i]);
                ak[i] = fmaf(rr_, sdk[rr * DS + lane + 32 * i], ak[i]);
                av[i] = fmaf(rr_, sdz[rr * DS + lane + 32 * i], av[i]);
            }
        }
    }
    if (active)
#pragma unroll
        for (int i = 0; i < NJ; i++) {
            dk[tok * D + lane + 32 * i] = from_f32<T>(ak[i]);
            dv[tok * D + lane + 32 * i] = from_f32<T>(av[i]);
        }
}

// B7: dq_(u,v) = (L-step part) + dqbar[g(u)][v] / |T_g|.
template <typename T>
__global__ void bwd_combine_dq_kernel(const float *__restrict__ dql,
                                      const float *__restrict__ dqbar, T *__restrict__ dq,
                                      Problem p) {
    const int64_t total = (int64_t)p.BH * p.N * p.d;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t tok = idx / p.d;
        const int j = (int)(idx % p.d);
        const int bh = (int)(tok / p.N), n = (int)(tok % p.N);
        const int u = n / p.b2, v = n % p.b2;
        int g = (int)(((int64_t)u * p.tiles) / p.b1);   // never above u's tile
        while (g + 1 < p.tiles && tile_begin(g + 1, p.b1, p.tiles) <= u) g++;
        const int rows = tile_begin(g + 1, p.b1, p.tiles) - tile_begin(g, p.b1, p.tiles);
        const int64_t gv = ((int64_t)bh * p.tiles + g) * p.b2 + v;
        dq[idx] = from_f32<T>(dql[idx] + dqbar[gv * p.d + j] / (float)rows);
    }
}

size_t a256(size_t x) { return (x + 255) & ~(size_t)255; }

template <typename K>
cudaError_t smem_opt_in(K kernel, size_t bytes) {
    return bytes > 48 * 1024
               ? cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)bytes)
               : cudaSuccess;
}

template <typename T, int D>
cudaError_t run_backward(const Problem &p, const T *q, const T *k, const T *v, const T *dy,
                         T *dq, T *dk, T *dv, const GenericWorkspace &fw, const BwdWorkspace &bw,
                         cudaStream_t stream) {
    constexpr int DS = D + 1;
    const size_t sm_ls = (GW * D + 2 * KC * DS + KC) * sizeof(float);
    const size_t sm_ldq = (2 * GW * D + 2 * KC * DS + KC) * sizeof(float);
    const size_t sm_ldkz = (2 * GW * D + 2 * KC * DS + 2 * KC) * sizeof(float);
    const size_t sm_rs = (3 * GW * D + 2 * KC * DS) * sizeof(float);
    const size_t sm_rdq = (3 * GW * D + 2 * KC * DS) * sizeof(float);
    const size_t sm_rdkv = (2 * GW * D + 3 * KC * DS + 4 * KC) * sizeof(float);
    cudaError_t e;
    if ((e = smem_opt_in(bwd_lstats_kernel<T, D>, sm_ls)) != cudaSuccess ||
        (e = smem_opt_in(bwd_ldq_kernel<T, D>, sm_ldq)) != cudaSuccess ||
        (e = smem_opt_in(bwd_ldkz_kernel<T, D>, sm_ldkz)) != cudaSuccess ||
        (e = smem_opt_in(bwd_rstats_kernel<T, D>, sm_rs)) != cudaSuccess ||
        (e = smem_opt_in(bwd_rdqbar_kernel<T, D>, sm_rdq)) != cudaSuccess ||
        (e = smem_opt_in(bwd_rdkv_kernel<T, D>, sm_rdkv)) != cudaSuccess)
        return e;
    const int64_t units = (int64_t)p.BH * p.tiles;
    const unsigned q_blocks = (unsigned)(units * p.b2 * ((tile_max_rows(p.b1, p.tiles) + GW - 1) / GW));
    const unsigned kz_blocks = (unsigned)(units * p.b2 * ((p.b1k + GW - 1) / GW));
    const unsigned rs_blocks = (unsigned)(units * p.b1k * ((p.b2 + GW - 1) / GW));
    const unsigned rq_blocks = (unsigned)(units * ((p.b2 + GW - 1) / GW));
    const unsigned kv_blocks = (unsigned)((int64_t)p.BH * p.b1k * ((p.b2 + GW - 1) / GW));
    {
        ProfileScope scope(K_BWD_L, stream);
        bwd_lstats_kernel<T, D><<<q_blocks, GW * 32, sm_ls, stream>>>(
            q, dy, fw.ktil, fw.z, fw.hent, bw.lse, bw.delta, p);
        bwd_ldq_kernel<T, D><<<q_blocks, GW * 32, sm_ldq, stream>>>(
            q, dy, fw.ktil, fw.z, fw.hent, bw.lse, bw.delta, bw.dql, p);
        bwd_ldkz_kernel<T, D><<<kz_blocks, GW * 32, sm_ldkz, stream>>>(
            q, dy, fw.ktil, fw.z, fw.hent, bw.lse, bw.delta, bw.dkt, bw.dz, bw.dh, p);
    }
    {
        ProfileScope scope(K_BWD_R, stream);
        bwd_rstats_kernel<T, D><<<rs_blocks, GW * 32, sm_rs, stream>>>(
            k, v, fw.qbar, bw.dkt, bw.dz, bw.lsea, bw.ea, bw.rho, p);
        bwd_rdqbar_kernel<T, D><<<rq_blocks, GW * 32, sm_rdq, stream>>>(
            k, v, fw.qbar, bw.dkt, bw.dz, bw.dh, bw.lsea, bw.ea, bw.rho, bw.dqbar, p);
        bwd_rdkv_kernel<T, D><<<kv_blocks, GW * 32, sm_rdkv, stream>>>(
            k, v, fw.qbar, bw.dkt, bw.dz, bw.dh, bw.lsea, bw.ea, bw.rho, dk, dv, p);
        const int64_t total = (int64_t)p.BH * p.N * p.d;
        const int blocks = (int)((total + 255) / 256 < 148 * 64 ? (total + 255) / 256 : 148 * 64);
        bwd_combine_dq_kernel<T><<<blocks, 256, 0, stream>>>(bw.dql, bw.dqbar, dq, p);
    }
    return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch_bwd(const Problem &p, const void *q, const void *k, const void *v,
                         const void *dy, void *dq, void *dk, void *dv,
                         const GenericWorkspace &fw, const BwdWorkspace &bw, cudaStream_t s) {
    const T *qq = (const T *)q, *kk = (const T *)k, *vv = (const T *)v, *gg = (const T *)dy;
    T *a = (T *)dq, *b = (T *)dk, *c = (T *)dv;
    switch (p.d) {
        case 32: return run_backward<T, 32>(p, qq, kk, vv, gg, a, b, c, fw, bw, s);
        case 64: return run_backward<T, 64>(p, qq, kk, vv, gg, a, b, c, fw, bw, s);
        case 128: return run_backward<T, 128>(p, qq, kk, vv, gg, a, b, c, fw, bw, s);
        default: return cudaErrorInvalidValue;
    }
}

size_t bwd_arrays_bytes(const Problem &p) {
    const size_t td = (size_t)p.BH * p.tiles * p.Nk * p.d;   // [BH][t][b2][b1k][d]
    const size_t tr = (size_t)p.BH * p.tiles * p.Nk;         // [BH][t][b2][b1k]
    const size_t nq = (size_t)p.BH * p.N;
    return 2 * a256(nq * 4) + a256(nq * p.d * 4) + 2 * a256(td * 4) + 4 * a256(tr * 4) +
           a256((size_t)p.BH * p.tiles * p.b2 * p.d * 4);
}

}  // namespace

size_t backward_workspace_bytes(const Problem &p, monarch_dtype dtype, bool &overflow) {
    if (sm100_backward_supports(p, dtype)) return sm100_backward_workspace_bytes(p, overflow);
    const size_t fwd = generic_workspace_bytes(p, overflow);
    if (overflow) return 0;
    return fwd + bwd_arrays_bytes(p);
}

BwdWorkspace backward_workspace_carve(const Problem &p, void *base, GenericWorkspace &fw) {
    bool overflow = false;
    fw = generic_workspace_carve(p, base);
    char *c = (char *)base + generic_workspace_bytes(p, overflow);
    const size_t td = (size_t)p.BH * p.tiles * p.Nk * p.d;
    const size_t tr = (size_t)p.BH * p.tiles * p.Nk;
    const size_t nq = (size_t)p.BH * p.N;
    BwdWorkspace bw;
    bw.lse = (float *)c;    c += a256(nq * 4);
    bw.delta = (float *)c;  c += a256(nq * 4);
    bw.dql = (float *)c;    c += a256(nq * p.d * 4);
    bw.dkt = (float *)c;    c += a256(td * 4);
    bw.dz = (float *)c;     c += a256(td * 4);
    bw.dh = (float *)c;     c += a256(tr * 4);
    bw.lsea = (float *)c;   c += a256(tr * 4);
    bw.ea = (float *)c;     c += a256(tr * 4);
    bw.rho = (float *)c;    c += a256(tr * 4);
    bw.dqbar = (float *)c;
    return bw;
}

cudaError_t generic_backward(const Problem &p, monarch_dtype dtype, const void *q, const void *k,
                             const void *v, const void *dy, void *dq, void *dk, void *dv,
                             void *workspace, int *status, long long wait_limit,
                             cudaStream_t stream) {
    // the workspace was sized for the same choice (backward_workspace_bytes)
    if (sm100_backward_supports(p, dtype)) {
        if (status == nullptr) return cudaErrorInvalidValue;
        return sm100_backward(p, q, k, v, dy, dq, dk, dv, workspace, status, wait_limit, stream);
    }
    GenericWorkspace fw;
    BwdWorkspace bw = backward_workspace_carve(p, workspace, fw);
    // the forward quantities the backward reads: qbar, Ktil, Z and H of the R-step
    cudaError_t e = generic_rstep_only(p, dtype, q, k, v, fw, stream);
    if (e != cudaSuccess) return e;
    if (dtype == MONARCH_F32)
        return dispatch_bwd<float>(p, q, k, v, dy, dq, dk, dv, fw, bw, stream);
    return dispatch_bwd<__nv_bfloat16>(p, q, k, v, dy, dq, dk, dv, fw, bw, stream);
}

}  // namespace monarch
