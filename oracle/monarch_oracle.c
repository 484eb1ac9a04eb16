/*
 * monarch_oracle.c -- plain float64 CPU oracle of the tiled MonarchRT attention
 * forward pass.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this code.  It shares nothing with the CUDA path:
 * no header, no helper, no table.  It is deliberately slow and literal: one
 * loop nest per step of the method, no blocking, no fusion.
 *
 * What it computes (sources: "MonarchRT: Efficient Attention for Real-Time
 * Video Generation", the arXiv abstract; the Chinese explainer page
 * "卡内基梅隆大学提出MonarchRT…", sections "Monarch矩阵：一种统一而强大的结构化近似工具"
 * (Monarch matrices; Fig. 3, MonarchAttention's alternating optimisation of L
 * and R from Q and K), "创新一：块对齐策略" (block alignment, N = f*h*w,
 * (b1, b2) = (f*h, w)) and "创新二：平铺Monarch参数化" (tiled Monarch, Fig. 2);
 * the VMonarch abstract for the entropy term of the L update).  The pages
 * print no formula; the update rules below are the plainest reading of them:
 *
 *   Tokens n = u*b2 + v, u in [b1] (block row), v in [b2] (column).
 *   M[(u,v),(u',v')] = L_v[u,u'] * R_{u',g(u)}[v,v'],   s = 1/sqrt(d),
 *   where the tile g(u) is the g with floor(g*b1/t) <= u < floor((g+1)*b1/t).
 *   M is the maximiser, over row-stochastic L and R, of
 *       F(L,R) = sum_rows [ sum_cols M_ij * s*q_i.k_j + entropy(M_i,:) ],
 *   the variational form of softmax, approached by alternating exact
 *   maximisation over R and over L:
 *     init      L_v[u,:] = 1/b1 (uniform)
 *     R-step    for every u', tile g, column v, with weights w_u = L_v[u,u'],
 *               u in T_g:  qbar = sum_u w_u q_(u,v) / sum_u w_u,
 *               R_{u',g}[v,:] = softmax_v'( s*qbar.k_(u',v') ),
 *               H = entropy of that row = lse - sum_v' R*logit,
 *               Ktil = sum_v' R k_(u',v'),  Z = sum_v' R v_(u',v')
 *     L-step    for every (u,v), g = g(u):
 *               L_v[u,:] = softmax_u'( s*q_(u,v).Ktil[g,v,u'] + H[g,v,u'] )
 *     output    y_(u,v) = sum_u' L_v[u,u'] Z[g(u),v,u']      (= M V)
 *   One iteration is an R-step followed by an L-step.
 *
 * Every step for token column v and tile g reads only the query rows
 * (u in T_g, v), all keys and all values, and writes only the outputs of
 * those rows; the oracle therefore loops over independent (head, g, v)
 * problems, which changes no arithmetic of any output.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL 1
#define ORACLE_ENOMEM 2

/* first block row of tile g: floor(g*b1/t) */
static int tile_first_row(int g, int b1, int tiles)
{
    return (int)(((int64_t)g * b1) / tiles);
}

/* Index maps of the method: u(n), v(n), the perfect shuffle P(n) = v*b1 + u,
 * the tile boundaries and the tile of every block row. */
int oracle_index_maps(int f, int h, int w, int b1, int b2, int tiles,
                      int32_t *u_of_n, int32_t *v_of_n, int32_t *perm,
                      int32_t *tile_lo, int32_t *tile_of_u)
{
    int64_t N = (int64_t)f * h * w;
    if (f < 1 || h < 1 || w < 1 || b1 < 1 || b2 < 1 || (int64_t)b1 * b2 != N ||
        tiles < 1 || tiles > b1)
        return ORACLE_EINVAL;
    for (int64_t n = 0; n < N; n++) {
        int u = (int)(n / b2), v = (int)(n % b2);
        u_of_n[n] = u;
        v_of_n[n] = v;
        perm[n] = v * b1 + u;
    }
    for (int g = 0; g <= tiles; g++)
        tile_lo[g] = tile_first_row(g, b1, tiles);
    for (int g = 0; g < tiles; g++)
        for (int u = tile_lo[g]; u < tile_lo[g + 1]; u++)
            tile_of_u[u] = g;
    return ORACLE_OK;
}

static size_t workspace_doubles(int d, int b1, int b1k, int b2, int tiles)
{
    int nq_max = (b1 + tiles - 1) / tiles + 1;
    int mx = b1k > b2 ? b1k : b2;
    return (size_t)nq_max * b1k + (size_t)b1k * b2 + 2 * (size_t)b1k * d + b1k + d + mx;
}

/*
 * One (tile g, column c) problem of one head: runs `half_steps` alternating
 * half-steps (R, L, R, L, ...) and writes y for the rows (u, c), u in T_g.
 * q, y: one head, [b1*b2][d] row-major (the queries; b1 block rows split
 * into the tiles); k, v: one head, [b1k*b2][d] (the keys and values in b1k
 * blocks of b2 tokens).  b1k = b1 is self-attention over one clip; b1k > b1
 * is the chunked setting in which the queries of the current chunk of frames
 * attend to a cache of earlier frames as well as to their own.
 * L_out (optional) [b2][b1][b1k]: L_c[u][u'] for u in T_g.
 * R_out (optional) [b1k][tiles][b2][b2]: R_{u',g}[c][:].
 */
static void solve_problem(const double *q, const double *k, const double *v, double *y,
                          int d, int b1, int b1k, int b2, int tiles, int g, int c,
                          int half_steps, double *L_out, double *R_out, double *ws)
{
    const double s = 1.0 / sqrt((double)d);
    const int u0 = tile_first_row(g, b1, tiles), u1 = tile_first_row(g + 1, b1, tiles);
    const int nq = u1 - u0;
    double *L = ws;                          /* [nq][b1k]  L_c[u][u'], u in T_g */
    double *R = L + (size_t)nq * b1k;        /* [b1k][b2]  R_{u',g}[c][:]       */
    double *Kt = R + (size_t)b1k * b2;       /* [b1k][d]   Ktil[g][c][u']       */
    double *Z = Kt + (size_t)b1k * d;        /* [b1k][d]   Z[g][c][u']          */
    double *H = Z + (size_t)b1k * d;         /* [b1k]      entropy of R row     */
    double *qbar = H + b1k;                  /* [d]                             */
    double *logit = qbar + d;                /* [max(b1k, b2)]                  */

    for (size_t i = 0; i < (size_t)nq * b1k; i++)
        L[i] = 1.0 / b1k;

    for (int step = 0; step < half_steps; step++) {
        if ((step & 1) == 0) {
            /* R-step: every block u' of tile g, row c of R_{u',g} */
            for (int up = 0; up < b1k; up++) {
                double wsum = 0.0;
                for (int j = 0; j < d; j++)
                    qbar[j] = 0.0;
                for (int u = u0; u < u1; u++) {
                    double wgt = L[(size_t)(u - u0) * b1k + up];
                    const double *qr = q + ((int64_t)u * b2 + c) * d;
                    wsum += wgt;
                    for (int j = 0; j < d; j++)
                        qbar[j] += wgt * qr[j];
                }
                /* a block that no row of the tile weighs does not enter F;
                 * the oracle then takes qbar = 0 (a uniform R row) */
                for (int j = 0; j < d; j++)
                    qbar[j] = wsum > 0.0 ? qbar[j] / wsum : 0.0;

                double mx = -INFINITY;
                for (int vp = 0; vp < b2; vp++) {
                    const double *kr = k + ((int64_t)up * b2 + vp) * d;
                    double acc = 0.0;
                    for (int j = 0; j < d; j++)
                        acc += qbar[j] * kr[j];
                    logit[vp] = s * acc;
                    if (logit[vp] > mx)
                        mx = logit[vp];
                }
                double sum = 0.0;
                for (int vp = 0; vp < b2; vp++)
                    sum += exp(logit[vp] - mx);
                double lse = mx + log(sum);
                double ent = lse;
                for (int vp = 0; vp < b2; vp++) {
                    double r = exp(logit[vp] - lse);
                    R[(size_t)up * b2 + vp] = r;
                    ent -= r * logit[vp];
                }
                H[up] = ent;
                for (int j = 0; j < d; j++) {
                    double kt = 0.0, z = 0.0;
                    for (int vp = 0; vp < b2; vp++) {
                        double r = R[(size_t)up * b2 + vp];
                        kt += r * k[((int64_t)up * b2 + vp) * d + j];
                        z += r * v[((int64_t)up * b2 + vp) * d + j];
                    }
                    Kt[(size_t)up * d + j] = kt;
                    Z[(size_t)up * d + j] = z;
                }
            }
        } else {
            /* L-step: every query row u of tile g at column c */
            for (int u = u0; u < u1; u++) {
                const double *qr = q + ((int64_t)u * b2 + c) * d;
                double mx = -INFINITY;
                for (int up = 0; up < b1k; up++) {
                    double acc = 0.0;
                    for (int j = 0; j < d; j++)
                        acc += qr[j] * Kt[(size_t)up * d + j];
                    logit[up] = s * acc + H[up];
                    if (logit[up] > mx)
                        mx = logit[up];
                }
                double sum = 0.0;
                for (int up = 0; up < b1k; up++)
                    sum += exp(logit[up] - mx);
                double lse = mx + log(sum);
                for (int up = 0; up < b1k; up++)
                    L[(size_t)(u - u0) * b1k + up] = exp(logit[up] - lse);
            }
        }
    }

    /* output: y_(u,c) = sum_u' L_c[u,u'] Z[u'] */
    for (int u = u0; u < u1; u++) {
        double *yr = y + ((int64_t)u * b2 + c) * d;
        for (int j = 0; j < d; j++) {
            double acc = 0.0;
            for (int up = 0; up < b1k; up++)
                acc += L[(size_t)(u - u0) * b1k + up] * Z[(size_t)up * d + j];
            yr[j] = acc;
        }
    }

    if (L_out)
        for (int u = u0; u < u1; u++)
            for (int up = 0; up < b1k; up++)
                L_out[((int64_t)c * b1 + u) * b1k + up] = L[(size_t)(u - u0) * b1k + up];
    if (R_out)
        for (int up = 0; up < b1k; up++)
            for (int vp = 0; vp < b2; vp++)
                R_out[(((int64_t)up * tiles + g) * b2 + c) * b2 + vp] = R[(size_t)up * b2 + vp];
}

static int check_shape(int N, int d, int b1, int b2, int tiles, int half_steps)
{
    if (N < 1 || d < 1 || b1 < 1 || b2 < 1 || (int64_t)b1 * b2 != N || tiles < 1 ||
        tiles > b1 || half_steps < 1)
        return ORACLE_EINVAL;
    return ORACLE_OK;
}

/*
 * Full forward pass over BH heads.  q, k, v, y: [BH][N][d].  half_steps = 2*iters
 * for the method; other counts stop after the matching half-step (the output
 * then uses the latest L and the latest R).  L_out [BH][b2][b1][b1] and R_out
 * [BH][b1][tiles][b2][b2] are optional.  nthreads <= 0 uses the OpenMP default.
 */
int oracle_monarch_attn(const double *q, const double *k, const double *v, double *y,
                        int BH, int N, int d, int b1, int b2, int tiles, int half_steps,
                        double *L_out, double *R_out, int nthreads)
{
    if (BH < 1 || check_shape(N, d, b1, b2, tiles, half_steps))
        return ORACLE_EINVAL;
    const int64_t nprob = (int64_t)BH * tiles * b2;
    const size_t wsz = workspace_doubles(d, b1, b1, b2, tiles);
    int err = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double *ws = (double *)malloc(wsz * sizeof(double));
        if (!ws) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = ORACLE_ENOMEM;
        }
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int64_t p = 0; p < nprob; p++) {
            if (!ws)
                continue;
            int bh = (int)(p / ((int64_t)tiles * b2));
            int g = (int)((p / b2) % tiles);
            int c = (int)(p % b2);
            size_t off = (size_t)bh * N * d;
            solve_problem(q + off, k + off, v + off, y + off, d, b1, b1, b2, tiles, g, c,
                          half_steps,
                          L_out ? L_out + (size_t)bh * b2 * b1 * b1 : NULL,
                          R_out ? R_out + (size_t)bh * b1 * tiles * b2 * b2 : NULL, ws);
        }
        free(ws);
    }
    return err;
}

/*
 * Selected (head, tile, column) problems only: probs[3*i .. 3*i+2] = (bh, g, c).
 * Writes the rows (u, c), u in T_g, of head bh in y [BH][N][d]; other rows are
 * left untouched.  Used for sampled parity checks and for the timed CPU baseline.
 */
int oracle_monarch_problems(const double *q, const double *k, const double *v, double *y,
                            int BH, int N, int d, int b1, int b2, int tiles, int half_steps,
                            int nprob, const int32_t *probs, int nthreads)
{
    if (BH < 1 || nprob < 0 || check_shape(N, d, b1, b2, tiles, half_steps))
        return ORACLE_EINVAL;
    for (int i = 0; i < nprob; i++)
        if (probs[3 * i] < 0 || probs[3 * i] >= BH || probs[3 * i + 1] < 0 ||
            probs[3 * i + 1] >= tiles || probs[3 * i + 2] < 0 || probs[3 * i + 2] >= b2)
            return ORACLE_EINVAL;
    const size_t wsz = workspace_doubles(d, b1, b1, b2, tiles);
    int err = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double *ws = (double *)malloc(wsz * sizeof(double));
        if (!ws) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = ORACLE_ENOMEM;
        }
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int i = 0; i < nprob; i++) {
            if (!ws)
                continue;
            int bh = probs[3 * i], g = probs[3 * i + 1], c = probs[3 * i + 2];
            size_t off = (size_t)bh * N * d;
            solve_problem(q + off, k + off, v + off, y + off, d, b1, b1, b2, tiles, g, c,
                          half_steps, NULL, NULL, ws);
        }
        free(ws);
    }
    return err;
}

/*
 * Queries of one chunk of frames against keys and values that also hold
 * earlier frames (a cache): q, y [BH][b1*b2][d], k, v [BH][b1k*b2][d], with
 * the b2 tokens of a block row shared by both (the video width for the
 * aligned blocks) and b1k >= 1 key blocks.  Every step is the one above with
 * the key blocks u' running over [b1k]; the tiles split the b1 query block
 * rows.  L_out [BH][b2][b1][b1k] and R_out [BH][b1k][tiles][b2][b2] optional.
 */
int oracle_monarch_attn_kv(const double *q, const double *k, const double *v, double *y,
                           int BH, int d, int b1, int b1k, int b2, int tiles, int half_steps,
                           double *L_out, double *R_out, int nthreads)
{
    if (BH < 1 || b1k < 1 || check_shape(b1 * b2, d, b1, b2, tiles, half_steps))
        return ORACLE_EINVAL;
    const int64_t nprob = (int64_t)BH * tiles * b2;
    const size_t wsz = workspace_doubles(d, b1, b1k, b2, tiles);
    const size_t nq = (size_t)b1 * b2 * d, nk = (size_t)b1k * b2 * d;
    int err = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double *ws = (double *)malloc(wsz * sizeof(double));
        if (!ws) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = ORACLE_ENOMEM;
        }
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int64_t p = 0; p < nprob; p++) {
            if (!ws)
                continue;
            int bh = (int)(p / ((int64_t)tiles * b2));
            int g = (int)((p / b2) % tiles);
            int c = (int)(p % b2);
            solve_problem(q + bh * nq, k + bh * nk, v + bh * nk, y + bh * nq, d, b1, b1k, b2,
                          tiles, g, c, half_steps,
                          L_out ? L_out + (size_t)bh * b2 * b1 * b1k : NULL,
                          R_out ? R_out + (size_t)bh * b1k * tiles * b2 * b2 : NULL, ws);
        }
        free(ws);
    }
    return err;
}

/*
 * The other reading of the tiles ("创新二：平铺Monarch参数化": each block is split
 * into tiles that are factorised independently): the tiles split the KEY
 * columns v' of every block instead of the query rows u.
 *   Key tile g' holds the columns T'_g' = [floor(g'*b2/t), floor((g'+1)*b2/t)),
 *   t in [1, b2].  A super-key is a (block u', key tile g') pair; there are
 *   b1k*t of them.
 *   M[(u,v),(u',v')] = L_v[u, (u',g'(v'))] * R_{u',g'(v')}[v,v'], where L_v[u,:]
 *   is a distribution over the super-keys and R_{u',g'}[v,:] one over the
 *   columns of tile g'.
 * The same variational objective gives the same two half-steps:
 *   init      L_v[u,:] = 1/(b1k*t)
 *   R-step    per (u', g', v): qbar = sum_u L_v[u,(u',g')] q_(u,v) / sum_u L,
 *             over ALL query rows u in [b1];  R = softmax over v' in T'_g' of
 *             s*qbar.k_(u',v');  H = its entropy;  Ktil, Z = sum_v' R k, R v
 *   L-step    per (u, v): L_v[u,:] = softmax over (u',g') of
 *             s*q_(u,v).Ktil[v,(u',g')] + H[v,(u',g')]
 *   output    y_(u,v) = sum_(u',g') L_v[u,(u',g')] Z[v,(u',g')]
 * t = 1 is plain Monarch (the same map as one query tile); t = b2 makes every
 * tile a single key column, R = 1, H = 0, and the L-step a softmax over all
 * N keys: exact attention.  Every step for column v reads all query rows
 * (u, v), all keys and all values and writes only the rows (u, v), so the
 * oracle loops over independent (head, v) problems.
 * Super-key j = g'*b1k + u'.  L_out (optional) [b2][b1][t*b1k];
 * R_out (optional) [b1k][t][b2][b2] with zeros outside the tile's columns.
 */
static int key_tile_first_col(int g, int b2, int tiles)
{
    return (int)(((int64_t)g * b2) / tiles);
}

static size_t keytiles_workspace_doubles(int d, int b1, int b1k, int b2, int tiles)
{
    size_t nsk = (size_t)tiles * b1k;
    size_t mx = nsk > (size_t)b2 ? nsk : (size_t)b2;
    return (size_t)b1 * nsk + nsk * b2 + 2 * nsk * d + nsk + d + mx;
}

static void solve_problem_keytiles(const double *q, const double *k, const double *v,
                                   double *y, int d, int b1, int b1k, int b2, int tiles,
                                   int c, int half_steps, double *L_out, double *R_out,
                                   double *ws)
{
    const double s = 1.0 / sqrt((double)d);
    const int nsk = tiles * b1k;
    double *L = ws;                          /* [b1][nsk]   L_c[u][j]            */
    double *R = L + (size_t)b1 * nsk;        /* [nsk][b2]   R_{u',g'}[c][:]      */
    double *Kt = R + (size_t)nsk * b2;       /* [nsk][d]    Ktil[c][j]           */
    double *Z = Kt + (size_t)nsk * d;        /* [nsk][d]    Z[c][j]              */
    double *H = Z + (size_t)nsk * d;         /* [nsk]       entropy of R row     */
    double *qbar = H + nsk;                  /* [d]                              */
    double *logit = qbar + d;                /* [max(nsk, b2)]                   */

    for (size_t i = 0; i < (size_t)b1 * nsk; i++)
        L[i] = 1.0 / nsk;

    for (int step = 0; step < half_steps; step++) {
        if ((step & 1) == 0) {
            /* R-step: every super-key j = (u', g'), row c of R_{u',g'} */
            for (int g = 0; g < tiles; g++) {
                const int c0 = key_tile_first_col(g, b2, tiles);
                const int c1 = key_tile_first_col(g + 1, b2, tiles);
                for (int up = 0; up < b1k; up++) {
                    const int j = g * b1k + up;
                    double wsum = 0.0;
                    for (int jj = 0; jj < d; jj++)
                        qbar[jj] = 0.0;
                    for (int u = 0; u < b1; u++) {
                        double wgt = L[(size_t)u * nsk + j];
                        const double *qr = q + ((int64_t)u * b2 + c) * d;
                        wsum += wgt;
                        for (int jj = 0; jj < d; jj++)
                            qbar[jj] += wgt * qr[jj];
                    }
                    for (int jj = 0; jj < d; jj++)
                        qbar[jj] = wsum > 0.0 ? qbar[jj] / wsum : 0.0;

                    double mx = -INFINITY;
                    for (int vp = c0; vp < c1; vp++) {
                        const double *kr = k + ((int64_t)up * b2 + vp) * d;
                        double acc = 0.0;
                        for (int jj = 0; jj < d; jj++)
                            acc += qbar[jj] * kr[jj];
                        logit[vp] = s * acc;
                        if (logit[vp] > mx)
                            mx = logit[vp];
                    }
                    double sum = 0.0;
                    for (int vp = c0; vp < c1; vp++)
                        sum += exp(logit[vp] - mx);
                    double lse = mx + log(sum);
                    double ent = lse;
                    for (int vp = 0; vp < b2; vp++)
                        R[(size_t)j * b2 + vp] = 0.0;
                    for (int vp = c0; vp < c1; vp++) {
                        double r = exp(logit[vp] - lse);
                        R[(size_t)j * b2 + vp] = r;
                        ent -= r * logit[vp];
                    }
                    H[j] = ent;
                    for (int jj = 0; jj < d; jj++) {
                        double kt = 0.0, z = 0.0;
                        for (int vp = c0; vp < c1; vp++) {
                            double r = R[(size_t)j * b2 + vp];
                            kt += r * k[((int64_t)up * b2 + vp) * d + jj];
                            z += r * v[((int64_t)up * b2 + vp) * d + jj];
                        }
                        Kt[(size_t)j * d + jj] = kt;
                        Z[(size_t)j * d + jj] = z;
                    }
                }
            }
        } else {
            /* L-step: every query row u at column c, over all super-keys */
            for (int u = 0; u < b1; u++) {
                const double *qr = q + ((int64_t)u * b2 + c) * d;
                double mx = -INFINITY;
                for (int j = 0; j < nsk; j++) {
                    double acc = 0.0;
                    for (int jj = 0; jj < d; jj++)
                        acc += qr[jj] * Kt[(size_t)j * d + jj];
                    logit[j] = s * acc + H[j];
                    if (logit[j] > mx)
                        mx = logit[j];
                }
                double sum = 0.0;
                for (int j = 0; j < nsk; j++)
                    sum += exp(logit[j] - mx);
                double lse = mx + log(sum);
                for (int j = 0; j < nsk; j++)
                    L[(size_t)u * nsk + j] = exp(logit[j] - lse);
            }
        }
    }

    /* output: y_(u,c) = sum_j L_c[u,j] Z[j] */
    for (int u = 0; u < b1; u++) {
        double *yr = y + ((int64_t)u * b2 + c) * d;
        for (int jj = 0; jj < d; jj++) {
            double acc = 0.0;
            for (int j = 0; j < nsk; j++)
                acc += L[(size_t)u * nsk + j] * Z[(size_t)j * d + jj];
            yr[jj] = acc;
        }
    }

    if (L_out)
        for (int u = 0; u < b1; u++)
            for (int j = 0; j < nsk; j++)
                L_out[((int64_t)c * b1 + u) * nsk + j] = L[(size_t)u * nsk + j];
    if (R_out)
        for (int g = 0; g < tiles; g++)
            for (int up = 0; up < b1k; up++)
                for (int vp = 0; vp < b2; vp++)
                    R_out[(((int64_t)up * tiles + g) * b2 + c) * b2 + vp] =
                        R[(size_t)(g * b1k + up) * b2 + vp];
}

/*
 * Key-column tiles over BH heads of self-attention: q, k, v, y [BH][N][d],
 * t in [1, b2].  With nprob >= 0 only the listed (bh, c) problems
 * (probs[2*i], probs[2*i+1]) run, writing the rows (u, c) of head bh of y and
 * leaving the others untouched; with nprob < 0 every problem runs and the
 * optional L_out [BH][b2][b1][t*b1] and R_out [BH][b1][t][b2][b2] are filled.
 */
int oracle_monarch_attn_keytiles(const double *q, const double *k, const double *v,
                                 double *y, int BH, int N, int d, int b1, int b2, int tiles,
                                 int half_steps, double *L_out, double *R_out, int nprob,
                                 const int32_t *probs, int nthreads)
{
    if (BH < 1 || N < 1 || d < 1 || b1 < 1 || b2 < 1 || (int64_t)b1 * b2 != N ||
        tiles < 1 || tiles > b2 || half_steps < 1)
        return ORACLE_EINVAL;
    for (int i = 0; i < nprob; i++)
        if (probs[2 * i] < 0 || probs[2 * i] >= BH || probs[2 * i + 1] < 0 ||
            probs[2 * i + 1] >= b2)
            return ORACLE_EINVAL;
    const int64_t ntask = nprob >= 0 ? nprob : (int64_t)BH * b2;
    const size_t wsz = keytiles_workspace_doubles(d, b1, b1, b2, tiles);
    const size_t nsk = (size_t)tiles * b1;
    int err = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double *ws = (double *)malloc(wsz * sizeof(double));
        if (!ws) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = ORACLE_ENOMEM;
        }
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int64_t p = 0; p < ntask; p++) {
            if (!ws)
                continue;
            int bh = nprob >= 0 ? probs[2 * p] : (int)(p / b2);
            int c = nprob >= 0 ? probs[2 * p + 1] : (int)(p % b2);
            size_t off = (size_t)bh * N * d;
            int full = nprob < 0;
            solve_problem_keytiles(q + off, k + off, v + off, y + off, d, b1, b1, b2, tiles, c,
                                   half_steps,
                                   (full && L_out) ? L_out + (size_t)bh * b2 * b1 * nsk : NULL,
                                   (full && R_out) ? R_out + (size_t)bh * b1 * tiles * b2 * b2
                                                   : NULL,
                                   ws);
        }
        free(ws);
    }
    return err;
}

/* Number of threads the OpenMP runtime would use (1 without OpenMP). */
/*
 * Backward pass of one iteration (iters = 1) by the chain rule, step by step.
 * There is no backward in the pages; this is the derivative of the forward
 * map above (its plain definition, written out), which the finetuning of the
 * summary page ("Approach") and the explainer page ("创新三") trains through.
 * Given dy = dPhi/dy for some scalar Phi, it returns dPhi/dq, dPhi/dk and
 * dPhi/dv.  Per (tile g, column c) problem, with the forward quantities of
 * solve_problem (qbar, R, H, Ktil, Z, L):
 *   L-step and output (y_u = sum_u' L[u,u'] Z[u'], b = s q_u.Ktil + H):
 *     dL[u,u'] = dy_u.Z[u'],  db[u,u'] = L[u,u'] (dL[u,u'] - sum_u'' L dL),
 *     dq_u += s sum_u' db Ktil[u'],   dKtil[u'] += s sum_u db q_u,
 *     dZ[u'] += sum_u L[u,u'] dy_u,   dH[u'] += sum_u db[u,u'].
 *   R-step (a = s qbar.k_(u',v'), R = softmax(a), H = lse(a) - sum R a,
 *   Ktil = sum R k, Z = sum R v):
 *     dR[v'] = dKtil[u'].k_(u',v') + dZ[u'].v_(u',v'),
 *     da[v'] = R (dR - sum R dR) - dH[u'] R (a - sum R a)   (dH/da = -R (a - E_R a)),
 *     dqbar += s sum_v' da k_(u',v'),
 *     dk_(u',v') += s da qbar + R dKtil[u'],   dv_(u',v') += R dZ[u'].
 *   Aggregation (qbar = mean over u in T_g of q_(u,c)):  dq_(u,c) += dqbar / |T_g|.
 * q, k, v, dy, dq, dk, dv: [BH][N][d]; dq, dk, dv are overwritten.
 */
int oracle_monarch_attn_bwd(const double *q, const double *k, const double *v,
                            const double *dy, double *dq, double *dk, double *dv, int BH,
                            int N, int d, int b1, int b2, int tiles, int nthreads)
{
    if (BH < 1 || check_shape(N, d, b1, b2, tiles, 2))
        return ORACLE_EINVAL;
    const double s = 1.0 / sqrt((double)d);
    const size_t per_head = (size_t)N * d;
    memset(dq, 0, (size_t)BH * per_head * sizeof(double));
    memset(dk, 0, (size_t)BH * per_head * sizeof(double));
    memset(dv, 0, (size_t)BH * per_head * sizeof(double));
    const int nq_max = (b1 + tiles - 1) / tiles + 1;
    /* per thread: A, R [b1][b2]; Kt, Z, dKt, dZ [b1][d]; H, dH [b1];
     * L, dB [nq_max][b1]; qbar, dqbar [d]; row [max(b1, b2)] */
    const size_t wsz = 2 * (size_t)b1 * b2 + 4 * (size_t)b1 * d + 2 * (size_t)b1 +
                       2 * (size_t)nq_max * b1 + 2 * (size_t)d + (size_t)(b1 > b2 ? b1 : b2);
    int err = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double *ws = (double *)malloc(wsz * sizeof(double));
        if (!ws) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = ORACLE_ENOMEM;
        }
        /* heads in parallel: the problems of one head all add into its dk, dv */
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int bh = 0; bh < BH; bh++) {
            if (!ws)
                continue;
            const double *qh = q + (size_t)bh * per_head, *kh = k + (size_t)bh * per_head;
            const double *vh = v + (size_t)bh * per_head, *dyh = dy + (size_t)bh * per_head;
            double *dqh = dq + (size_t)bh * per_head, *dkh = dk + (size_t)bh * per_head;
            double *dvh = dv + (size_t)bh * per_head;
            double *A = ws, *R = A + (size_t)b1 * b2, *Kt = R + (size_t)b1 * b2;
            double *Z = Kt + (size_t)b1 * d, *dKt = Z + (size_t)b1 * d, *dZ = dKt + (size_t)b1 * d;
            double *H = dZ + (size_t)b1 * d, *dH = H + b1, *L = dH + b1;
            double *dB = L + (size_t)nq_max * b1, *qbar = dB + (size_t)nq_max * b1;
            double *dqbar = qbar + d, *row = dqbar + d;
            for (int g = 0; g < tiles; g++) {
                const int u0 = tile_first_row(g, b1, tiles), u1 = tile_first_row(g + 1, b1, tiles);
                const int nq = u1 - u0;
                for (int c = 0; c < b2; c++) {
                    /* ---- forward, as in solve_problem (one R-step from uniform L) */
                    for (int j = 0; j < d; j++) {
                        double acc = 0.0;
                        for (int u = u0; u < u1; u++)
                            acc += qh[((int64_t)u * b2 + c) * d + j];
                        qbar[j] = acc / nq;
                    }
                    for (int up = 0; up < b1; up++) {
                        double mx = -INFINITY;
                        for (int vp = 0; vp < b2; vp++) {
                            double acc = 0.0;
                            for (int j = 0; j < d; j++)
                                acc += qbar[j] * kh[((int64_t)up * b2 + vp) * d + j];
                            A[(size_t)up * b2 + vp] = s * acc;
                            if (s * acc > mx)
                                mx = s * acc;
                        }
                        double sum = 0.0;
                        for (int vp = 0; vp < b2; vp++)
                            sum += exp(A[(size_t)up * b2 + vp] - mx);
                        const double lse = mx + log(sum);
                        double ent = lse;
                        for (int vp = 0; vp < b2; vp++) {
                            R[(size_t)up * b2 + vp] = exp(A[(size_t)up * b2 + vp] - lse);
                            ent -= R[(size_t)up * b2 + vp] * A[(size_t)up * b2 + vp];
                        }
                        H[up] = ent;
                        for (int j = 0; j < d; j++) {
                            double kt = 0.0, z = 0.0;
                            for (int vp = 0; vp < b2; vp++) {
                                kt += R[(size_t)up * b2 + vp] * kh[((int64_t)up * b2 + vp) * d + j];
                                z += R[(size_t)up * b2 + vp] * vh[((int64_t)up * b2 + vp) * d + j];
                            }
                            Kt[(size_t)up * d + j] = kt;
                            Z[(size_t)up * d + j] = z;
                        }
                    }
                    for (int u = u0; u < u1; u++) {
                        const double *qr = qh + ((int64_t)u * b2 + c) * d;
                        double mx = -INFINITY;
                        for (int up = 0; up < b1; up++) {
                            double acc = 0.0;
                            for (int j = 0; j < d; j++)
                                acc += qr[j] * Kt[(size_t)up * d + j];
                            row[up] = s * acc + H[up];
                            if (row[up] > mx)
                                mx = row[up];
                        }
                        double sum = 0.0;
                        for (int up = 0; up < b1; up++)
                            sum += exp(row[up] - mx);
                        const double lse = mx + log(sum);
                        for (int up = 0; up < b1; up++)
                            L[(size_t)(u - u0) * b1 + up] = exp(row[up] - lse);
                    }
                    /* ---- L-step and output backward */
                    memset(dKt, 0, (size_t)b1 * d * sizeof(double));
                    memset(dZ, 0, (size_t)b1 * d * sizeof(double));
                    memset(dH, 0, (size_t)b1 * sizeof(double));
                    for (int u = u0; u < u1; u++) {
                        const double *qr = qh + ((int64_t)u * b2 + c) * d;
                        const double *dyr = dyh + ((int64_t)u * b2 + c) * d;
                        double *Lr = L + (size_t)(u - u0) * b1, *dBr = dB + (size_t)(u - u0) * b1;
                        double ldl = 0.0;
                        for (int up = 0; up < b1; up++) {
                            double acc = 0.0;
                            for (int j = 0; j < d; j++)
                                acc += dyr[j] * Z[(size_t)up * d + j];
                            row[up] = acc;   /* dL[u,u'] */
                            ldl += Lr[up] * acc;
                        }
                        for (int up = 0; up < b1; up++)
                            dBr[up] = Lr[up] * (row[up] - ldl);
                        double *dqr = dqh + ((int64_t)u * b2 + c) * d;
                        for (int j = 0; j < d; j++) {
                            double acc = 0.0;
                            for (int up = 0; up < b1; up++)
                                acc += dBr[up] * Kt[(size_t)up * d + j];
                            dqr[j] += s * acc;
                        }
                        for (int up = 0; up < b1; up++) {
                            for (int j = 0; j < d; j++) {
                                dKt[(size_t)up * d + j] += s * dBr[up] * qr[j];
                                dZ[(size_t)up * d + j] += Lr[up] * dyr[j];
                            }
                            dH[up] += dBr[up];
                        }
                    }
                    /* ---- R-step backward */
                    for (int j = 0; j < d; j++)
                        dqbar[j] = 0.0;
                    for (int up = 0; up < b1; up++) {
                        const double *Rr = R + (size_t)up * b2, *Ar = A + (size_t)up * b2;
                        double rdr = 0.0, ea = 0.0;
                        for (int vp = 0; vp < b2; vp++) {
                            const double *kr = kh + ((int64_t)up * b2 + vp) * d;
                            const double *vr = vh + ((int64_t)up * b2 + vp) * d;
                            double acc = 0.0;
                            for (int j = 0; j < d; j++)
                                acc += dKt[(size_t)up * d + j] * kr[j] + dZ[(size_t)up * d + j] * vr[j];
                            row[vp] = acc;   /* dR[v'] */
                            rdr += Rr[vp] * acc;
                            ea += Rr[vp] * Ar[vp];
                        }
                        for (int vp = 0; vp < b2; vp++) {
                            const double da = Rr[vp] * (row[vp] - rdr) - dH[up] * Rr[vp] * (Ar[vp] - ea);
                            const double *kr = kh + ((int64_t)up * b2 + vp) * d;
                            double *dkr = dkh + ((int64_t)up * b2 + vp) * d;
                            double *dvr = dvh + ((int64_t)up * b2 + vp) * d;
                            for (int j = 0; j < d; j++) {
                                dqbar[j] += s * da * kr[j];
                                dkr[j] += s * da * qbar[j] + Rr[vp] * dKt[(size_t)up * d + j];
                                dvr[j] += Rr[vp] * dZ[(size_t)up * d + j];
                            }
                        }
                    }
                    for (int u = u0; u < u1; u++)
                        for (int j = 0; j < d; j++)
                            dqh[((int64_t)u * b2 + c) * d + j] += dqbar[j] / nq;
                }
            }
        }
        free(ws);
    }
    return err;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
