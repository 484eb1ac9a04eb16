/*
 * monarch_attn.h -- C ABI of the tiled MonarchRT attention forward pass on
 * NVIDIA B200 (sm_100a).
 *
 * The operation (sources: "MonarchRT: Efficient Attention for Real-Time Video
 * Generation", abstract; the explainer page "卡内基梅隆大学提出MonarchRT…", sections
 * "Monarch矩阵" with Fig. 3, "创新一：块对齐策略" and "创新二：平铺Monarch参数化" with
 * Fig. 2; the VMonarch abstract for the entropy term).  The pages print no
 * formulas; this library computes the following reading of them.
 *
 *   Video tokens n = (fi*h + hi)*w + wi, N = f*h*w, split as n = u*b2 + v with
 *   block row u in [b1] and column v in [b2] (b1*b2 = N; the aligned choice is
 *   (b1, b2) = (f*h, w)).  Attention softmax(Q K^T / sqrt(d)) is replaced by a
 *   Monarch matrix M = P^T L P R: R has b1 diagonal blocks of b2 x b2, L has b2
 *   diagonal blocks of b1 x b1, P is the perfect shuffle u*b2+v -> v*b1+u.  With
 *   t tiles the block rows split into T_g = [floor(g*b1/t), floor((g+1)*b1/t))
 *   and each tile g owns its own R:  M[(u,v),(u',v')] = L_v[u,u'] R_{u',g(u)}[v,v'].
 *   L and R come from `iters` rounds of alternating maximisation of
 *   sum_rows [<M_i, s q_i K^T> + entropy(M_i)], s = 1/sqrt(d), from uniform L:
 *     R-step: R_{u',g}[v,:] = softmax_v'(s qbar.k_(u',v')), qbar the L-weighted
 *             mean of the queries (u in T_g, v); it also yields the row entropy
 *             H, Ktil = R K_u' and Z = R V_u';
 *     L-step: L_v[u,:] = softmax_u'(s q_(u,v).Ktil[g,v,u'] + H[g,v,u']);
 *   and the output is Y = M V, i.e. y_(u,v) = sum_u' L_v[u,u'] Z[g(u),v,u'].
 *
 * Tensor layout: Q, K, V and Y are contiguous [B][H][N][d] arrays (d
 * innermost, token order as above) in the dtype given; Y has the dtype of the
 * inputs.  All arithmetic after loading is float32 (bfloat16 operands of the
 * tensor-core products, float32 accumulation and softmax).
 *
 * Conventions for every entry point:
 *   - No call throws, aborts or traps; every call returns a monarch_status.
 *   - Arguments are validated on the host before anything is enqueued; a call
 *     that fails validation enqueues nothing and writes nothing.
 *   - Device work is asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream).  The caller keeps ownership of every buffer and
 *     must keep it alive until that work has finished.
 *   - The library keeps no global state other than a per-device cache of
 *     kernel attributes and a device-side status word (see
 *     monarch_last_device_status).
 */
#ifndef MONARCH_ATTN_H
#define MONARCH_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MONARCH_API __attribute__((visibility("default")))
#else
#define MONARCH_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream, declared without the CUDA headers. */
typedef struct CUstream_st *monarch_stream_t;

typedef enum {
    MONARCH_F32 = 0,  /* float32 inputs and output                                */
    MONARCH_BF16 = 1  /* bfloat16 inputs and output (raw 16-bit storage)           */
} monarch_dtype;

typedef enum {
    MONARCH_OK = 0,
    MONARCH_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, bad dtype        */
    MONARCH_ERR_SHAPE = 2,       /* b1*b2 != f*h*w, tiles outside [1, b1], iters < 1,
                                    or a size too large for the index arithmetic     */
    MONARCH_ERR_ALIGN = 3,       /* a pointer not 16-byte aligned                    */
    MONARCH_ERR_UNSUPPORTED = 4, /* d not in {32, 64, 128}                           */
    MONARCH_ERR_NO_MEMORY = 5,   /* workspace allocation failed, or ws_bytes too small */
    MONARCH_ERR_CUDA = 6,        /* a CUDA runtime call or kernel launch failed      */
    MONARCH_ERR_TIMEOUT = 7,     /* a device-side bounded wait gave up (see below)   */
    MONARCH_ERR_SCRATCH_LIMIT = 8 /* needs more scratch than monarch_attn_fwd_noalloc's
                                     static buffer (MONARCH_NOALLOC_SCRATCH_BYTES)    */
} monarch_status;

/*
 * Forward pass with a library-managed workspace.
 *   q, k, v   device pointers, [B][H][N][d] in `dtype`, N = f*h*w, read only.
 *   out       device pointer, [B][H][N][d] in `dtype`, fully overwritten.
 *   B, H      batch and heads (>= 1).     f, h, w  video latent grid (>= 1).
 *   d         head dimension: 32, 64 or 128.
 *   b1, b2    Monarch block sizes, b1*b2 = N (aligned choice: (f*h, w)).
 *   tiles     tiles per block, 1 <= tiles <= b1.   iters  alternating rounds, >= 1.
 * The workspace (monarch_attn_workspace_bytes) is taken with stream-ordered
 * cudaMallocAsync on `stream` and released with cudaFreeAsync on it.
 * Source: MonarchRT explainer page, "Monarch矩阵" (M = P L P^T R), "创新一"
 * (blocks aligned to the latent grid) and "创新二" (tiles); the entropy term
 * and the alternating rounds: VMonarch abstract (MonarchAttention's
 * variational form).
 */
MONARCH_API monarch_status monarch_attn_fwd(const void *q, const void *k, const void *v, void *out,
                                int B, int H, int f, int h, int w, int d, int b1, int b2,
                                int tiles, int iters, monarch_dtype dtype,
                                monarch_stream_t stream);

/*
 * Forward pass that allocates nothing.  (No counterpart in the MonarchRT
 * pages: this is a deployment convenience of this library.)
 *
 * For callers that may not allocate device memory: code whose host framework
 * owns every device allocation and forbids others, or loops where the implicit
 * device synchronisation of cudaMalloc/cudaFree is not acceptable.  The call
 * takes no workspace argument and calls no cudaMalloc, cudaFree, cudaMallocAsync
 * or other allocating routine: its scratch space is one file-scope static
 * device array of MONARCH_NOALLOC_SCRATCH_BYTES (64 MiB), which every GPU that
 * loads the library's no-allocation module holds until the process exits.
 *
 * Arguments and layout as monarch_attn_fwd (q, k, v, out: caller-owned device
 * buffers).  It runs the generic kernel family (any supported shape and dtype)
 * with its float32 intermediates placed in the static array; problems whose
 * scratch exceeds the array are rejected with MONARCH_ERR_SCRATCH_LIMIT before
 * anything is enqueued.  The 480p chunk shape (B=1, H=12, d=128, N=4680) fits.
 *
 * The first call in each CUDA context (normally the primary context of each
 * device) looks up the array's device address with cudaGetSymbolAddress, with
 * that context current, and caches it under the context's id, so a context that
 * was reset or replaced gets a fresh lookup; make that first call before any
 * stream capture.  Every call on a device shares the one array, which keeps
 * the contents of the last call; nothing in it needs to start at zero.  Calls
 * that overlap on the GPU (different streams without ordering, or several host
 * threads) race on the array and give wrong results: serialise them.
 * Source: the operation of monarch_attn_fwd; the allocation-free form has no
 * counterpart in the pages.
 */
#define MONARCH_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

MONARCH_API monarch_status monarch_attn_fwd_noalloc(const void *q, const void *k, const void *v,
                                                    void *out, int B, int H, int f, int h,
                                                    int w, int d, int b1, int b2, int tiles,
                                                    int iters, monarch_dtype dtype,
                                                    monarch_stream_t stream);

/*
 * Workspace bytes that monarch_attn_fwd_ws needs for these arguments, or 0 if
 * the arguments fail validation.  Pure host function; enqueues nothing.
 * The workspace holds the aggregated queries, Ktil = R K and Z = R V for
 * every (head, tile, column, block), the entropies H and, for iters > 1,
 * the per-block aggregated queries and the row log-sum-exp of the L-step.
 * Source: no counterpart in the pages (a property of this implementation).
 */
MONARCH_API size_t monarch_attn_workspace_bytes(int B, int H, int f, int h, int w, int d, int b1, int b2,
                                    int tiles, int iters, monarch_dtype dtype);

/*
 * Forward pass with a caller-owned workspace: device memory of at least
 * monarch_attn_workspace_bytes(...) bytes, 256-byte aligned.  Other arguments
 * as monarch_attn_fwd.  Returns MONARCH_ERR_NO_MEMORY if ws_bytes is too small.
 * The workspace contents need no initialisation and are garbage afterwards.
 * Two calls that share a workspace must not overlap on the GPU.
 * Source: as monarch_attn_fwd.
 */
MONARCH_API monarch_status monarch_attn_fwd_ws(const void *q, const void *k, const void *v, void *out,
                                   int B, int H, int f, int h, int w, int d, int b1, int b2,
                                   int tiles, int iters, monarch_dtype dtype, void *workspace,
                                   size_t ws_bytes, monarch_stream_t stream);

/*
 * Forward pass over a contiguous range of (batch, head, tile) units, for
 * splitting one call's work across GPUs or streams.  Unit index
 * ((b*H + h)*tiles + g), 0 <= unit_begin <= unit_end <= B*H*tiles.  A unit
 * is independent of every other one from the aggregated query to its output
 * (the method's tiles each own their R factor; explainer page, "创新二：平铺
 * Monarch参数化"), so the union of calls over a partition of the units gives
 * exactly the output of one full call, bit for bit.  Writes only the output
 * rows of those units, i.e. rows (u, v) with u in tile g, every v, of head
 * (b, h); every other row of out is left untouched.  q, k, v must hold the
 * whole clip.  Workspace and other arguments as monarch_attn_fwd_ws (the
 * workspace size does not depend on the range; the tensor-core path computes
 * the R-step of every tile of the heads that the range touches).
 * Returns MONARCH_ERR_SHAPE for a range outside [0, B*H*tiles].
 * Source: explainer page, "创新二：平铺Monarch参数化" (independent tiles).
 */
MONARCH_API monarch_status monarch_attn_fwd_units_ws(const void *q, const void *k, const void *v,
                                                     void *out, int B, int H, int f, int h, int w,
                                                     int d, int b1, int b2, int tiles, int iters,
                                                     monarch_dtype dtype, int unit_begin,
                                                     int unit_end, void *workspace,
                                                     size_t ws_bytes, monarch_stream_t stream);

/*
 * Forward pass on tensors in another layout.  layout = MONARCH_LAYOUT_BHND is
 * [B][H][N][d] (monarch_attn_fwd_ws); MONARCH_LAYOUT_BNHD is [B][N][H][d], the
 * heads of each token contiguous, as in the attention layers of video diffusion
 * transformers.  q, k, v and out all use `layout`; the workspace
 * (monarch_attn_workspace_bytes, the same for both layouts) and every other
 * argument are those of monarch_attn_fwd_ws.  Both kernel families read the
 * strided rows directly (no transposed copies).  Returns MONARCH_ERR_INVALID_ARG
 * for another layout value.
 * Source: the survey's strided-input variant of the explainer page's video token
 * layout ("创新一：块对齐策略": N = f*h*w tokens per head).
 */
typedef enum { MONARCH_LAYOUT_BHND = 0, MONARCH_LAYOUT_BNHD = 1 } monarch_layout;

MONARCH_API monarch_status monarch_attn_fwd_layout_ws(const void *q, const void *k, const void *v,
                                                      void *out, int B, int H, int f, int h,
                                                      int w, int d, int b1, int b2, int tiles,
                                                      int iters, monarch_dtype dtype,
                                                      monarch_layout layout, void *workspace,
                                                      size_t ws_bytes, monarch_stream_t stream);

/*
 * Forward pass with the tiles on either axis.  The tiled parameterisation splits
 * every block into t tiles that are factorised independently; which axis is
 * split is a reading:
 *   MONARCH_TILE_QUERY_ROWS   (every other entry point) the query rows u of each
 *       block: tile g = rows [floor(g*b1/t), floor((g+1)*b1/t)) owns its own
 *       R_{u',g}; 1 <= tiles <= b1; tiles = b1 is exact attention.
 *   MONARCH_TILE_KEY_COLUMNS  the key columns v' of each block: key tile g' =
 *       columns [floor(g'*b2/t), floor((g'+1)*b2/t)); R_{u',g'}[v,:] is a softmax
 *       over the tile's columns of s*qbar.k with qbar aggregated over all b1
 *       query rows of column v, and each query row's L is a softmax over the
 *       b1*t (block u', key tile g') super-keys of s*q.Ktil + H;
 *       1 <= tiles <= b2; tiles = b2 is exact attention.
 * tiles = 1 is plain Monarch on both axes.  `layout` as monarch_attn_fwd_layout_ws;
 * the workspace is monarch_attn_tiled_workspace_bytes (0 if the arguments fail
 * validation; MONARCH_ERR_NO_MEMORY if ws_bytes is smaller), 256-byte aligned;
 * monarch_attn_tiled_path reports the kernel family as monarch_attn_path does
 * (key-column tiles take the tensor-core kernels for one iteration, the generic
 * kernels for more).  Other arguments, errors and
 * ownership as monarch_attn_fwd_ws; MONARCH_ERR_INVALID_ARG for another axis value.
 * Source: explainer page, "创新二：平铺Monarch参数化" (each block split into tiles
 * factorised independently; the axis is not stated there).
 */
typedef enum { MONARCH_TILE_QUERY_ROWS = 0, MONARCH_TILE_KEY_COLUMNS = 1 } monarch_tile_axis;

MONARCH_API size_t monarch_attn_tiled_workspace_bytes(int B, int H, int f, int h, int w, int d,
                                                      int b1, int b2, int tiles, int iters,
                                                      monarch_dtype dtype,
                                                      monarch_tile_axis axis);
MONARCH_API int monarch_attn_tiled_path(int B, int H, int f, int h, int w, int d, int b1, int b2,
                                        int tiles, int iters, monarch_dtype dtype,
                                        monarch_tile_axis axis);
MONARCH_API monarch_status monarch_attn_fwd_tiled_ws(const void *q, const void *k, const void *v,
                                                     void *out, int B, int H, int f, int h,
                                                     int w, int d, int b1, int b2, int tiles,
                                                     int iters, monarch_dtype dtype,
                                                     monarch_tile_axis axis,
                                                     monarch_layout layout, void *workspace,
                                                     size_t ws_bytes, monarch_stream_t stream);

/*
 * Queries of a chunk of frames against keys and values that also hold earlier
 * frames (a key/value cache), as in chunk-by-chunk autoregressive video
 * generation (the Self-Forcing setting of the MonarchRT pages: summary page,
 * "Setup"; explainer page, the autoregressive models it evaluates).
 *   q, out   [B][H][fq*h*w][d]: the chunk's queries and output.
 *   k, v     [B][H][fk*h*w][d]: keys and values of fk >= 1 frames (the cached
 *            frames followed by the chunk's own, or any other order).
 *   b1*b2 = fq*h*w, b1k*b2 = fk*h*w: b2 tokens per block row on both sides
 *            (aligned: b2 = w, b1 = fq*h, b1k = fk*h); the tiles split the b1
 *            query block rows.
 * The Monarch factors become L_v of b1 x b1k and R_{u',g} of b2 x b2 for the b1k
 * key blocks; every step is that of monarch_attn_fwd with the key blocks
 * running over [b1k].  fq = fk with the same tensors is monarch_attn_fwd.
 * Workspace: monarch_attn_kv_workspace_bytes (0 if the arguments fail
 * validation).  Errors and ownership as monarch_attn_fwd_ws.
 * monarch_attn_kv_path reports the kernel family as monarch_attn_path does.
 * Source: summary page, "Setup" (chunked autoregressive generation with a
 * cache of earlier frames); the factor shapes b1 x b1k are this library's
 * reading of the method for unequal query and key lengths.
 */
MONARCH_API size_t monarch_attn_kv_workspace_bytes(int B, int H, int fq, int fk, int h, int w,
                                                   int d, int b1, int b1k, int b2, int tiles,
                                                   int iters, monarch_dtype dtype);
MONARCH_API int monarch_attn_kv_path(int B, int H, int fq, int fk, int h, int w, int d, int b1,
                                     int b1k, int b2, int tiles, int iters, monarch_dtype dtype);
MONARCH_API monarch_status monarch_attn_fwd_kv_ws(const void *q, const void *k, const void *v,
                                                  void *out, int B, int H, int fq, int fk, int h,
                                                  int w, int d, int b1, int b1k, int b2,
                                                  int tiles, int iters, monarch_dtype dtype,
                                                  void *workspace, size_t ws_bytes,
                                                  monarch_stream_t stream);

/*
 * Backward pass of one iteration (iters must be 1; else MONARCH_ERR_UNSUPPORTED).
 * Given dy = dPhi/dY for a scalar loss Phi of the output of monarch_attn_fwd with
 * the same arguments, writes dq = dPhi/dQ, dk = dPhi/dK, dv = dPhi/dV: the chain
 * rule through the output, the L-step (L = softmax(s q.Ktil + H)), the R-step
 * (R = softmax(s qbar.k), its entropy H, Ktil = R K, Z = R V) and the query
 * aggregation (qbar = mean of the tile's queries).
 *   q, k, v, dy   device pointers, [B][H][N][d] in `dtype`, read only.
 *   dq, dk, dv    device pointers, [B][H][N][d] in `dtype`, fully overwritten.
 * Other arguments as monarch_attn_fwd.  Where the forward takes the tensor-core
 * kernels (bfloat16, d = 128; monarch_attn_path = 1) the backward does too: it
 * recomputes the forward's intermediates on the tensor cores and forms every
 * gradient with tcgen05 products (bfloat16 operands, float32 accumulation).  Every
 * other shape and dtype runs on generic float32 kernels.  Both are deterministic
 * (no atomics; reductions in a fixed order).  The workspace
 * (monarch_attn_bwd_workspace_bytes, 0 if the arguments fail validation or
 * iters != 1) holds the forward intermediates and the backward's.
 * monarch_attn_bwd takes it with cudaMallocAsync on `stream`; monarch_attn_bwd_ws
 * uses the caller's (256-byte aligned; MONARCH_ERR_NO_MEMORY if too small).
 * Source: the pages print no backward; they finetune through the attention
 * (summary page, "Approach"; explainer page, "创新三：微调与高效内核").  This is
 * the derivative of the forward map above.
 */
MONARCH_API size_t monarch_attn_bwd_workspace_bytes(int B, int H, int f, int h, int w, int d,
                                                    int b1, int b2, int tiles, int iters,
                                                    monarch_dtype dtype);
MONARCH_API monarch_status monarch_attn_bwd_ws(const void *q, const void *k, const void *v,
                                               const void *dy, void *dq, void *dk, void *dv,
                                               int B, int H, int f, int h, int w, int d, int b1,
                                               int b2, int tiles, int iters, monarch_dtype dtype,
                                               void *workspace, size_t ws_bytes,
                                               monarch_stream_t stream);
MONARCH_API monarch_status monarch_attn_bwd(const void *q, const void *k, const void *v,
                                            const void *dy, void *dq, void *dk, void *dv, int B,
                                            int H, int f, int h, int w, int d, int b1, int b2,
                                            int tiles, int iters, monarch_dtype dtype,
                                            monarch_stream_t stream);

/*
 * Forward pass on HOST buffers: q, k, v, out are host pointers (pinned memory
 * gives full PCIe bandwidth; pageable memory works but is slower).  Device
 * copies of the inputs and output and the workspace are taken with
 * cudaMallocAsync on `stream`; the call enqueues host-to-device copies, the
 * forward pass and the device-to-host copy of `out`, then releases the device
 * memory, all on `stream`.  `out` is valid once the stream has synchronised.
 * Source: as monarch_attn_fwd (host buffers: no counterpart in the pages).
 */
MONARCH_API monarch_status monarch_attn_fwd_host(const void *q, const void *k, const void *v, void *out,
                                     int B, int H, int f, int h, int w, int d, int b1, int b2,
                                     int tiles, int iters, monarch_dtype dtype,
                                     monarch_stream_t stream);

/*
 * Index maps of the method, on the host (int32, computed with the same
 * inline functions the kernels use):
 *   u_of_n[n] = n / b2, v_of_n[n] = n % b2, perm[n] = v*b1 + u   (each N entries),
 *   tile_begin[g] = floor(g*b1/tiles) for g = 0..tiles        (tiles + 1 entries).
 * Any output pointer may be NULL to skip it.
 * Source: explainer page, "Monarch矩阵" (the permutation between the two
 * block-diagonal factors), "创新一" (N = f*h*w in blocks of (f*h, w)) and
 * "创新二" (tiles of the block rows).
 */
MONARCH_API monarch_status monarch_index_maps(int f, int h, int w, int b1, int b2, int tiles,
                                  int32_t *u_of_n, int32_t *v_of_n, int32_t *perm,
                                  int32_t *tile_begin);

/*
 * The same maps computed by a kernel on the device into device buffers
 * (sizes as above; NULL skips a map), enqueued on `stream`.
 * Source: as monarch_index_maps.
 */
MONARCH_API monarch_status monarch_index_maps_device(int f, int h, int w, int b1, int b2, int tiles,
                                         int32_t *u_of_n, int32_t *v_of_n, int32_t *perm,
                                         int32_t *tile_begin, monarch_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears the device-side status word of
 * the current device.  Kernels that wait on barriers bound every wait; when one
 * gives up it records MONARCH_ERR_TIMEOUT there and the kernel returns early
 * (its output is then incomplete).  Returns MONARCH_OK if no wait gave up,
 * MONARCH_ERR_CUDA if the synchronisation failed.
 * Source: no counterpart in the pages (failure detection of this library).
 */
MONARCH_API monarch_status monarch_last_device_status(monarch_stream_t stream);

/*
 * Test hook: the iteration limit of the device-side bounded waits (spins on an
 * mbarrier).  0 restores the default.  Takes effect for launches enqueued after
 * the call, on every device.  Returns the previous limit.
 * Source: no counterpart in the pages (a test facility of this library).
 */
MONARCH_API long long monarch_set_wait_limit(long long spins);

/*
 * Test hook: fault injection for the bounded waits.  While on (on != 0), the
 * MMA-issuing warp of every tensor-core kernel launched afterwards first waits
 * on a barrier that nothing ever completes.  The wait gives up after the wait
 * limit, records MONARCH_ERR_TIMEOUT in the status word and the kernel takes
 * its abort path: every other role stops waiting, the kernel waits for its own
 * copies and tensor-core work in flight, frees its tensor memory and returns,
 * leaving the output incomplete.  Nothing faults, traps or hangs.  Affects
 * launches enqueued after the call, on every device.  Returns the previous
 * setting.  (No counterpart in the pages: a test facility of this library.)
 */
MONARCH_API int monarch_debug_inject_stall(int on);

/*
 * Benchmark hook: per-kernel timing.  While enabled (on != 0), every kernel
 * launch of the forward and backward passes is bracketed by CUDA events recorded on its launch
 * stream; the launches themselves are unchanged.  Disabling keeps the counters.
 * Source: no counterpart in the pages (a measurement facility).
 */
MONARCH_API monarch_status monarch_profile_enable(int on);

/*
 * Waits for the recorded events, adds their durations to per-kernel counters
 * and copies, for each kernel family k < max_kernels, the total milliseconds
 * (ms[k]) and launch count (launches[k]) since the previous call, then resets
 * the counters.  Either array may be NULL.  Returns the number of kernel
 * families (the valid k), or -1 if waiting on an event failed.
 * Source: no counterpart in the pages (a measurement facility).
 */
MONARCH_API int monarch_profile_collect(double *ms, long long *launches, int max_kernels);

/* Name of kernel family k (static string), or NULL if k is out of range.
 * Source: no counterpart in the pages. */
MONARCH_API const char *monarch_profile_kernel_name(int k);

/* Static, NUL-terminated description of a status code.
 * Source: no counterpart in the pages. */
MONARCH_API const char *monarch_status_string(monarch_status status);

/*
 * Which kernel family a call with these arguments dispatches to:
 * 0 = generic SIMT kernels (any supported shape, float32 or bfloat16),
 * 1 = sm_100a tensor-core kernels (bfloat16, d = 128, b2 <= 128, the R-step's
 *     shared-memory plan fits; any iteration count),
 * -1 = the arguments fail validation.  Pure host function.
 * Source: no counterpart in the pages (dispatch of this library).
 */
MONARCH_API int monarch_attn_path(int B, int H, int f, int h, int w, int d, int b1, int b2, int tiles,
                      int iters, monarch_dtype dtype);

#ifdef __cplusplus
}
#endif

#endif /* MONARCH_ATTN_H */
