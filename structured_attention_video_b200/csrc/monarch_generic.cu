// monarch_generic.cu -- SIMT kernels of the Monarch attention forward pass for
// every supported shape and dtype (float32 arithmetic throughout).
//
// The forward pass follows MonarchAttention's alternating maximisation as the
// MonarchRT pages describe it (explainer page, "Monarch矩阵" section, Fig. 3;
// tiles from "创新二：平铺Monarch参数化", Fig. 2; the entropy term of the L
// update from the VMonarch abstract's online entropy inside a FlashAttention
// loop):
//   S1  qbar[g][v]        = mean_{u in T_g} q_(u,v)                 (first R-step, uniform L)
//   S2  R-step per (g, v, u'): online softmax over the b2 keys of block u' with
//       logits s*qbar.k_(u',v'); emits Ktil = R K, Z = R V and the entropy H
//   S3  L-step per query (u, v): online softmax over the b1 blocks with logits
//       s*q_(u,v).Ktil[g][v][u'] + H[g][v][u']; emits y = sum L Z (last round)
//       and the row log-sum-exp (rounds before the last)
//   S4  (iters > 1) qbar[g][v][u'] = sum_u L_v[u,u'] q_(u,v) / sum_u L_v[u,u'],
//       L recomputed from the saved log-sum-exp
// With key tiles (the other reading of the tiles: the key columns v' of every
// block split into t tiles) S1 and S4 aggregate over all b1 query rows, the
// R-step of key tile g' takes its softmax over the tile's columns only, and
// the L-step of each query row runs over the t*b1k (block, key tile) rows of
// Ktil, Z and H of its column.
// Each warp owns one softmax row; a CTA of 8 warps shares chunks of 32 keys
// staged in shared memory (rows padded to d+1 floats: conflict-free).
#include "monarch_common.cuh"

#include <math.h>

namespace monarch {

namespace {

constexpr int GW = 8;    // warps (softmax rows) per CTA
constexpr int KC = 32;   // keys per shared-memory chunk

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

// S1: qbar[bh][g][v][:] = mean over u in T_g of q[bh][u*b2+v][:]
template <typename T>
__global__ void qbar_mean_kernel(const T *__restrict__ q, float *__restrict__ qbar, Problem p) {
    const int64_t row_elems = (int64_t)p.b2 * p.d;
    // the (head, tile) units of the call: unit = bh * tiles + g
    const int64_t total = (int64_t)p.unit_end * row_elems;
    for (int64_t idx = (int64_t)p.unit_begin * row_elems + (int64_t)blockIdx.x * blockDim.x +
                       threadIdx.x;
         idx < total; idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t bhg = idx / row_elems, col = idx % row_elems;
        const int g = (int)(bhg % p.tiles), bh = (int)(bhg / p.tiles);
        const int u0 = unit_row_begin(p, g), u1 = unit_row_end(p, g);
        const int64_t ts = tok_stride(p);
        const T *src = q + head_base(p, bh, p.N) + (col / p.d) * ts + col % p.d;
        float acc = 0.f;
        for (int u = u0; u < u1; u++) acc += to_f32(src[(int64_t)u * p.b2 * ts]);
        qbar[idx] = acc / (float)(u1 - u0);
    }
}

// S2: one warp per R row (bh, g, v, u'); the CTA covers GW consecutive v of one
// (bh, g, u') and stages the block's keys and values in chunks of KC.
template <typename T, int D>
__global__ void __launch_bounds__(GW * 32)
rstep_kernel(const T *__restrict__ k, const T *__restrict__ v, const float *__restrict__ qbar,
             int64_t qbar_v_stride, int64_t qbar_up_stride, float *__restrict__ ktil,
             float *__restrict__ z, float *__restrict__ hent, Problem p) {
    constexpr int DS = D + 1, NJ = D / 32;
    extern __shared__ float sm[];
    float *sq = sm;               // [GW][D]
    float *sk = sq + GW * D;      // [KC][DS]
    float *sv = sk + KC * DS;     // [KC][DS]

    const int nvg = (p.b2 + GW - 1) / GW;
    int64_t bid = blockIdx.x + (int64_t)p.unit_begin * p.b1k * nvg;   // from the first unit
    const int vg = (int)(bid % nvg);
    bid /= nvg;
    const int up = (int)(bid % p.b1k);   // key block
    bid /= p.b1k;
    const int g = (int)(bid % p.tiles);
    const int bh = (int)(bid / p.tiles);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int vrow = vg * GW + warp;
    const bool active = vrow < p.b2;
    const int64_t bhg = (int64_t)bh * p.tiles + g;

    if (active) {
        const float *qr = qbar + (bhg * p.b2 + vrow) * qbar_v_stride + (int64_t)up * qbar_up_stride;
        for (int j = lane; j < D; j += 32) sq[warp * D + j] = qr[j];
    }
    const int64_t ts = tok_stride(p);
    const int64_t base = head_base(p, bh, p.Nk) + (int64_t)up * p.b2 * ts;
    const int kc0 = unit_col_begin(p, g), kc1 = unit_col_end(p, g);
    float m = -INFINITY, l = 0.f, e = 0.f;
    float acck[NJ], accv[NJ];
#pragma unroll
    for (int i = 0; i < NJ; i++) acck[i] = accv[i] = 0.f;

    for (int c0 = kc0; c0 < kc1; c0 += KC) {
        const int nk = min(KC, kc1 - c0);
        __syncthreads();
        for (int idx = threadIdx.x; idx < nk * D; idx += blockDim.x) {
            const int r = idx / D, j = idx % D;
            sk[r * DS + j] = to_f32(k[base + (int64_t)(c0 + r) * ts + j]);
            sv[r * DS + j] = to_f32(v[base + (int64_t)(c0 + r) * ts + j]);
        }
        __syncthreads();
        if (!active) continue;
        float s = -INFINITY;
        if (lane < nk) {
            float acc = 0.f;
#pragma unroll 8
            for (int j = 0; j < D; j++) acc = fmaf(sq[warp * D + j], sk[lane * DS + j], acc);
            s = acc * p.scale;
        }
        const float mn = fmaxf(m, warp_max(s));
        const float alpha = (m == -INFINITY) ? 0.f : expf(m - mn);
        const float pr = (lane < nk) ? expf(s - mn) : 0.f;
        const float ps = warp_sum(pr), pe = warp_sum(lane < nk ? pr * s : 0.f);
        l = l * alpha + ps;
        e = e * alpha + pe;
        m = mn;
#pragma unroll
        for (int i = 0; i < NJ; i++) {
            acck[i] *= alpha;
            accv[i] *= alpha;
        }
        for (int r = 0; r < nk; r++) {
            const float pr_r = __shfl_sync(0xffffffffu, pr, r);
#pragma unroll
            for (int i = 0; i < NJ; i++) {
                acck[i] = fmaf(pr_r, sk[r * DS + lane + 32 * i], acck[i]);
                accv[i] = fmaf(pr_r, sv[r * DS + lane + 32 * i], accv[i]);
            }
        }
    }
    if (active) {
        const float inv = 1.f / l;
        const int64_t row = (bhg * p.b2 + vrow) * p.b1k + up;
#pragma unroll
        for (int i = 0; i < NJ; i++) {
            ktil[row * D + lane + 32 * i] = acck[i] * inv;
            z[row * D + lane + 32 * i] = accv[i] * inv;
        }
        // entropy of the row: lse - E_R[logit]
        if (lane == 0) hent[row] = (m + logf(l)) - e * inv;
    }
}

// S3: one warp per query (u, v) of tile g; the CTA covers GW consecutive u of
// one (bh, g, v) and stages Ktil, Z and H of that (g, v) in chunks of KC blocks.
template <typename T, int D>
__global__ void __launch_bounds__(GW * 32)
lstep_kernel(const T *__restrict__ q, const float *__restrict__ ktil, const float *__restrict__ z,
             const float *__restrict__ hent, T *__restrict__ out, float *__restrict__ lse_out,
             Problem p) {
    constexpr int DS = D + 1, NJ = D / 32;
    extern __shared__ float sm[];
    float *sq = sm;               // [GW][D]
    float *sk = sq + GW * D;      // [KC][DS]
    float *sz = sk + KC * DS;     // [KC][DS]
    float *sh = sz + KC * DS;     // [KC]

    // query tiles: a unit (bh, g) per grid slice; key tiles: a head per slice,
    // its rows u over all b1 and its keys over the t key tiles
    const int nug = (p.key_tiles ? p.b1 + GW - 1 : tile_max_rows(p.b1, p.tiles) + GW - 1) / GW;
    const int nseg = p.key_tiles ? p.tiles : 1;
    int64_t bid = blockIdx.x + (int64_t)(p.key_tiles ? p.head_begin() : p.unit_begin) * p.b2 * nug;
    const int ug = (int)(bid % nug);
    bid /= nug;
    const int vcol = (int)(bid % p.b2);
    bid /= p.b2;
    const int g = p.key_tiles ? 0 : (int)(bid % p.tiles);
    const int bh = (int)(p.key_tiles ? bid : bid / p.tiles);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u0 = unit_row_begin(p, g), u1 = unit_row_end(p, g);
    const int u = u0 + ug * GW + warp;
    const bool active = u < u1;
    const int64_t tok = (int64_t)bh * p.N + (int64_t)u * p.b2 + vcol;   // workspace index
    const int64_t qoff = head_base(p, bh, p.N) + ((int64_t)u * p.b2 + vcol) * tok_stride(p);

    if (active)
        for (int j = lane; j < D; j += 32) sq[warp * D + j] = to_f32(q[qoff + j]);
    float m = -INFINITY, l = 0.f;
    float acc[NJ];
#pragma unroll
    for (int i = 0; i < NJ; i++) acc[i] = 0.f;

    // chunk ch covers keys [c0, c0 + nk) of segment sg: the rows of block
    // u' = c0 .. of (g, v), g the unit's tile or, with key tiles, key tile sg
    const int nchunk = (p.b1k + KC - 1) / KC;
    for (int ch = 0; ch < nseg * nchunk; ch++) {
        const int sg = ch / nchunk, c0 = (ch % nchunk) * KC;
        const int64_t kbase =
            (((int64_t)bh * p.tiles + (p.key_tiles ? sg : g)) * p.b2 + vcol) * p.b1k;
        const int nk = min(KC, p.b1k - c0);
        __syncthreads();
        for (int idx = threadIdx.x; idx < nk * D; idx += blockDim.x) {
            const int r = idx / D, j = idx % D;
            sk[r * DS + j] = ktil[(kbase + c0 + r) * D + j];
            sz[r * DS + j] = z[(kbase + c0 + r) * D + j];
        }
        if (threadIdx.x < nk) sh[threadIdx.x] = hent[kbase + c0 + threadIdx.x];
        __syncthreads();
        if (!active) continue;
        float s = -INFINITY;
        if (lane < nk) {
            float a = 0.f;
#pragma unroll 8
            for (int j = 0; j < D; j++) a = fmaf(sq[warp * D + j], sk[lane * DS + j], a);
            s = a * p.scale + sh[lane];
        }
        const float mn = fmaxf(m, warp_max(s));
        const float alpha = (m == -INFINITY) ? 0.f : expf(m - mn);
        const float pr = (lane < nk) ? expf(s - mn) : 0.f;
        l = l * alpha + warp_sum(pr);
        m = mn;
#pragma unroll
        for (int i = 0; i < NJ; i++) acc[i] *= alpha;
        for (int r = 0; r < nk; r++) {
            const float pr_r = __shfl_sync(0xffffffffu, pr, r);
#pragma unroll
            for (int i = 0; i < NJ; i++) acc[i] = fmaf(pr_r, sz[r * DS + lane + 32 * i], acc[i]);
        }
    }
    if (active) {
        if (out) {
            const float inv = 1.f / l;
#pragma unroll
            for (int i = 0; i < NJ; i++) out[qoff + lane + 32 * i] = from_f32<T>(acc[i] * inv);
        }
        if (lse_out && lane == 0) lse_out[tok] = m + logf(l);
    }
}

// S4: one warp per (bh, g, v, u'); weights L_v[u,u'] over u in T_g recomputed
// as exp(s*q_(u,v).Ktil[u'] + H[u'] - lse_(u,v)).  H[u'] is the same for every
// u and cancels in the normalised mean, so it is left out; the weights are
// taken relative to their maximum (the ratio is unchanged, nothing underflows).
template <typename T, int D>
__global__ void __launch_bounds__(GW * 32)
qbar_weighted_kernel(const T *__restrict__ q, const float *__restrict__ ktil,
                     const float *__restrict__ lse, float *__restrict__ qbar, Problem p) {
    constexpr int DS = D + 1, NJ = D / 32;
    extern __shared__ float sm[];
    float *skt = sm;              // [GW][D]   this warp's Ktil row
    float *sq = skt + GW * D;     // [KC][DS]  query rows of the chunk
    float *sl = sq + KC * DS;     // [KC]

    const int nupg = (p.b1k + GW - 1) / GW;
    int64_t bid = blockIdx.x + (int64_t)p.unit_begin * p.b2 * nupg;   // from the first unit
    const int upg = (int)(bid % nupg);
    bid /= nupg;
    const int vcol = (int)(bid % p.b2);
    bid /= p.b2;
    const int g = (int)(bid % p.tiles);
    const int bh = (int)(bid / p.tiles);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int up = upg * GW + warp;
    const bool active = up < p.b1k;
    const int u0 = unit_row_begin(p, g), u1 = unit_row_end(p, g);
    const int64_t bhg = (int64_t)bh * p.tiles + g;
    const int64_t row = (bhg * p.b2 + vcol) * p.b1k + up;

    if (active)
        for (int j = lane; j < D; j += 32) skt[warp * D + j] = ktil[row * D + j];
    float m = -INFINITY, l = 0.f;
    float acc[NJ];
#pragma unroll
    for (int i = 0; i < NJ; i++) acc[i] = 0.f;

    for (int c0 = u0; c0 < u1; c0 += KC) {
        const int nk = min(KC, u1 - c0);
        __syncthreads();
        for (int idx = threadIdx.x; idx < nk * D; idx += blockDim.x) {
            const int r = idx / D, j = idx % D;
            const int64_t tok = (int64_t)(c0 + r) * p.b2 + vcol;
            sq[r * DS + j] = to_f32(q[head_base(p, bh, p.N) + tok * tok_stride(p) + j]);
        }
        if (threadIdx.x < nk)
            sl[threadIdx.x] = lse[(int64_t)bh * p.N + (int64_t)(c0 + threadIdx.x) * p.b2 + vcol];
        __syncthreads();
        if (!active) continue;
        float s = -INFINITY;
        if (lane < nk) {
            float a = 0.f;
#pragma unroll 8
            for (int j = 0; j < D; j++) a = fmaf(skt[warp * D + j], sq[lane * DS + j], a);
            s = a * p.scale - sl[lane];
        }
        const float mn = fmaxf(m, warp_max(s));
        const float alpha = (m == -INFINITY) ? 0.f : expf(m - mn);
        const float pr = (lane < nk) ? expf(s - mn) : 0.f;
        l = l * alpha + warp_sum(pr);
        m = mn;
#pragma unroll
        for (int i = 0; i < NJ; i++) acc[i] *= alpha;
        for (int r = 0; r < nk; r++) {
            const float pr_r = __shfl_sync(0xffffffffu, pr, r);
#pragma unroll
            for (int i = 0; i < NJ; i++) acc[i] = fmaf(pr_r, sq[r * DS + lane + 32 * i], acc[i]);
        }
    }
    if (active) {
        const float inv = 1.f / l;
#pragma unroll
        for (int i = 0; i < NJ; i++) qbar[row * D + lane + 32 * i] = acc[i] * inv;
    }
}

__global__ void index_maps_kernel(int N, int b1, int b2, int tiles, int32_t *u_of_n,
                                  int32_t *v_of_n, int32_t *perm, int32_t *tile_lo) {
    const int64_t limit = N > tiles + 1 ? (int64_t)N : (int64_t)tiles + 1;
    for (int64_t n = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; n < limit;
         n += (int64_t)gridDim.x * blockDim.x) {
        if (n < N) {
            const int u = block_row(n, b2), v = block_col(n, b2);
            if (u_of_n) u_of_n[n] = u;
            if (v_of_n) v_of_n[n] = v;
            if (perm) perm[n] = (int32_t)shuffle(u, v, b1);
        }
        if (tile_lo && n <= tiles) tile_lo[n] = tile_begin((int)n, b1, tiles);
    }
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

template <typename T, int D>
cudaError_t run_generic(const Problem &p, const T *q, const T *k, const T *v, T *out,
                        const GenericWorkspace &ws, cudaStream_t stream) {
    const size_t smem_r = (GW * D + 2 * KC * (D + 1)) * sizeof(float);
    const size_t smem_l = (GW * D + 2 * KC * (D + 1) + KC) * sizeof(float);
    const size_t smem_w = (GW * D + KC * (D + 1) + KC) * sizeof(float);
    const int64_t units = p.unit_end - p.unit_begin;
    const int64_t nmean = units * p.b2 * p.d;
    const int mean_blocks = (int)((nmean + 255) / 256 < 148 * 64 ? (nmean + 255) / 256 : 148 * 64);
    {
        ProfileScope scope(K_QBAR_MEAN, stream);
        qbar_mean_kernel<T><<<mean_blocks, 256, 0, stream>>>(q, ws.qbar, p);
    }
    const unsigned r_blocks = (unsigned)(units * p.b1k * ((p.b2 + GW - 1) / GW));
    const unsigned l_blocks =
        p.key_tiles ? (unsigned)((int64_t)(p.head_end() - p.head_begin()) * p.b2 * ((p.b1 + GW - 1) / GW))
                    : (unsigned)(units * p.b2 * ((tile_max_rows(p.b1, p.tiles) + GW - 1) / GW));
    const unsigned w_blocks = (unsigned)(units * p.b2 * ((p.b1k + GW - 1) / GW));
    for (int it = 0; it < p.iters; it++) {
        const bool last = it == p.iters - 1;
        const int64_t vstride = it == 0 ? (int64_t)p.d : (int64_t)p.b1k * p.d;
        const int64_t upstride = it == 0 ? 0 : (int64_t)p.d;
        {
            ProfileScope scope(K_RSTEP, stream);
            rstep_kernel<T, D><<<r_blocks, GW * 32, smem_r, stream>>>(
                k, v, ws.qbar, vstride, upstride, ws.ktil, ws.z, ws.hent, p);
        }
        {
            ProfileScope scope(K_LSTEP, stream);
            lstep_kernel<T, D><<<l_blocks, GW * 32, smem_l, stream>>>(
                q, ws.ktil, ws.z, ws.hent, last ? out : nullptr, last ? nullptr : ws.lse, p);
        }
        if (!last) {
            ProfileScope scope(K_QBAR_WEIGHTED, stream);
            qbar_weighted_kernel<T, D><<<w_blocks, GW * 32, smem_w, stream>>>(q, ws.ktil, ws.lse,
                                                                              ws.qbar, p);
        }
    }
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t run_rstep_only(const Problem &p, const T *q, const T *k, const T *v,
                           const GenericWorkspace &ws, cudaStream_t stream) {
    const size_t smem_r = (GW * D + 2 * KC * (D + 1)) * sizeof(float);
    const int64_t units = p.unit_end - p.unit_begin;
    const int64_t nmean = units * p.b2 * p.d;
    const int mean_blocks = (int)((nmean + 255) / 256 < 148 * 64 ? (nmean + 255) / 256 : 148 * 64);
    {
        ProfileScope scope(K_QBAR_MEAN, stream);
        qbar_mean_kernel<T><<<mean_blocks, 256, 0, stream>>>(q, ws.qbar, p);
    }
    const unsigned r_blocks = (unsigned)(units * p.b1k * ((p.b2 + GW - 1) / GW));
    ProfileScope scope(K_RSTEP, stream);
    rstep_kernel<T, D><<<r_blocks, GW * 32, smem_r, stream>>>(k, v, ws.qbar, (int64_t)p.d, 0,
                                                            ws.ktil, ws.z, ws.hent, p);
    return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch_d(const Problem &p, const void *q, const void *k, const void *v, void *out,
                       const GenericWorkspace &ws, cudaStream_t stream) {
    const T *qq = (const T *)q, *kk = (const T *)k, *vv = (const T *)v;
    T *oo = (T *)out;
    switch (p.d) {
        case 32: return run_generic<T, 32>(p, qq, kk, vv, oo, ws, stream);
        case 64: return run_generic<T, 64>(p, qq, kk, vv, oo, ws, stream);
        case 128: return run_generic<T, 128>(p, qq, kk, vv, oo, ws, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

size_t generic_workspace_bytes(const Problem &p, bool &overflow) {
    const long double big = (long double)p.BH * p.tiles * p.Nk * p.d * 4.0L * 4.0L;
    overflow = big > (long double)(1ULL << 62);
    if (overflow) return 0;
    const size_t td = (size_t)p.BH * p.tiles * p.Nk * p.d;   // one [BH][t][b2][b1k][d] array
    const size_t qb = p.iters > 1 ? td : (size_t)p.BH * p.tiles * p.b2 * p.d;
    return align256(qb * 4) + 2 * align256(td * 4) + align256((size_t)p.BH * p.tiles * p.Nk * 4) +
           (p.iters > 1 ? align256((size_t)p.BH * p.N * 4) : 0);
}

GenericWorkspace generic_workspace_carve(const Problem &p, void *base) {
    const size_t td = (size_t)p.BH * p.tiles * p.Nk * p.d;
    const size_t qb = p.iters > 1 ? td : (size_t)p.BH * p.tiles * p.b2 * p.d;
    char *c = (char *)base;
    GenericWorkspace ws;
    ws.qbar = (float *)c;
    c += align256(qb * 4);
    ws.ktil = (float *)c;
    c += align256(td * 4);
    ws.z = (float *)c;
    c += align256(td * 4);
    ws.hent = (float *)c;
    c += align256((size_t)p.BH * p.tiles * p.Nk * 4);
    ws.lse = p.iters > 1 ? (float *)c : nullptr;
    return ws;
}

cudaError_t generic_forward(const Problem &p, monarch_dtype dtype, const void *q, const void *k,
                            const void *v, void *out, const GenericWorkspace &ws,
                            cudaStream_t stream) {
    if (dtype == MONARCH_F32) return dispatch_d<float>(p, q, k, v, out, ws, stream);
    return dispatch_d<__nv_bfloat16>(p, q, k, v, out, ws, stream);
}

cudaError_t generic_rstep_only(const Problem &p, monarch_dtype dtype, const void *q,
                               const void *k, const void *v, const GenericWorkspace &ws,
                               cudaStream_t stream) {
    switch (p.d) {
#define MONARCH_RO_CASE(D)                                                                    \
    case D:                                                                                   \
        return dtype == MONARCH_F32                                                           \
                   ? run_rstep_only<float, D>(p, (const float *)q, (const float *)k,          \
                                              (const float *)v, ws, stream)                   \
                   : run_rstep_only<__nv_bfloat16, D>(p, (const __nv_bfloat16 *)q,            \
                                                      (const __nv_bfloat16 *)k,               \
                                                      (const __nv_bfloat16 *)v, ws, stream);
        MONARCH_RO_CASE(32) MONARCH_RO_CASE(64) MONARCH_RO_CASE(128)
#undef MONARCH_RO_CASE
    }
    return cudaErrorInvalidValue;
}

cudaError_t index_maps_device(int N, int b1, int b2, int tiles, int32_t *u_of_n, int32_t *v_of_n,
                              int32_t *perm, int32_t *tile_lo, cudaStream_t stream) {
    const int blocks = (int)(((int64_t)N + 1 + 255) / 256 < 4096 ? ((int64_t)N + 1 + 255) / 256 : 4096);
    index_maps_kernel<<<blocks, 256, 0, stream>>>(N, b1, b2, tiles, u_of_n, v_of_n, perm, tile_lo);
    return cudaGetLastError();
}

}  // namespace monarch
