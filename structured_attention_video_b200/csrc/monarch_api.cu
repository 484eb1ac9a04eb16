// monarch_api.cu -- the C ABI declared in include/monarch_attn.h: argument
// validation, workspace sizing and carving, dispatch to the kernel families,
// the host-buffer entry point and the device status word.
#include "monarch_common.cuh"
#include "monarch_sm100.cuh"

#include <cuda.h>

#include <atomic>
#include <map>
#include <math.h>
#include <mutex>
#include <vector>

namespace monarch {

// The device status word (one per device that loads the library).
__device__ int g_device_status = 0;

namespace {

std::atomic<long long> g_wait_limit{kDefaultWaitLimit};
std::atomic<int> g_inject_stall{0};
std::mutex g_dev_mutex;
constexpr int kMaxDevices = 64;
bool g_pool_configured[kMaxDevices] = {false};
SymbolAddressCache g_status_cache;

// The status word of the current context (see SymbolAddressCache).
int *status_word_on_current_device() {
    void *ptr = nullptr;
    return g_status_cache.lookup(g_device_status, &ptr) == cudaSuccess ? (int *)ptr : nullptr;
}

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

template <typename Fn> Fn driver_fn(const char *name) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<Fn>(ptr);
}

// Stream-ordered allocations of the entry points that allocate come from the
// device's default memory pool; keeping freed memory in the pool (instead of
// returning it at every synchronisation) makes repeated calls cheap.
void configure_pool_once() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return;
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (g_pool_configured[dev]) return;
    cudaMemPool_t pool;
    if (cudaDeviceGetDefaultMemPool(&pool, dev) == cudaSuccess) {
        uint64_t keep = UINT64_MAX;
        cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    }
    g_pool_configured[dev] = true;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

bool current_context_id(unsigned long long *id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
        get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    });
    if (!get_current || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

namespace {

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

monarch_status validate_shape(int B, int H, int f, int h, int w, int d, int b1, int b2, int tiles,
                              int iters, monarch_dtype dtype, Problem *p) {
    if (B < 1 || H < 1 || f < 1 || h < 1 || w < 1 || d < 1 || b1 < 1 || b2 < 1)
        return MONARCH_ERR_INVALID_ARG;
    if (dtype != MONARCH_F32 && dtype != MONARCH_BF16) return MONARCH_ERR_INVALID_ARG;
    const int64_t N = (int64_t)f * h * w;
    if (N > (1LL << 30) || (int64_t)b1 * b2 != N) return MONARCH_ERR_SHAPE;
    if (tiles < 1 || tiles > b1 || iters < 1 || iters > 1000) return MONARCH_ERR_SHAPE;
    if ((int64_t)B * H > (1LL << 24)) return MONARCH_ERR_SHAPE;
    if ((int64_t)B * H * tiles >= (1LL << 31)) return MONARCH_ERR_SHAPE;   // unit indices
    if (d != 32 && d != 64 && d != 128) return MONARCH_ERR_UNSUPPORTED;
    // every grid of the generic kernels must fit in 2^31 - 1 blocks
    const int64_t BHt = (int64_t)B * H * tiles;
    const int64_t grid_r = BHt * b1 * ((b2 + 7) / 8);
    const int64_t grid_l = BHt * b2 * ((tile_max_rows(b1, tiles) + 7) / 8);
    const int64_t grid_w = BHt * b2 * ((b1 + 7) / 8);
    if (grid_r >= (1LL << 31) || grid_l >= (1LL << 31) || grid_w >= (1LL << 31))
        return MONARCH_ERR_SHAPE;
    p->B = B;
    p->H = H;
    p->BH = B * H;
    p->N = (int)N;
    p->d = d;
    p->b1 = b1;
    p->b2 = b2;
    p->tiles = tiles;
    p->iters = iters;
    p->scale = (float)(1.0 / sqrt((double)d));
    p->unit_begin = 0;
    p->unit_end = B * H * tiles;
    p->Nk = p->N;
    p->b1k = b1;
    p->layout = kLayoutBHND;
    p->key_tiles = 0;
    return MONARCH_OK;
}

namespace {

// Either reading of the tiles: query rows (tiles in [1, b1]) or key columns
// (tiles in [1, b2]); see Problem::key_tiles.
monarch_status validate_tiled(int B, int H, int f, int h, int w, int d, int b1, int b2, int tiles,
                              int iters, monarch_dtype dtype, monarch_tile_axis axis, Problem *p) {
    if (axis == MONARCH_TILE_QUERY_ROWS)
        return validate_shape(B, H, f, h, w, d, b1, b2, tiles, iters, dtype, p);
    if (axis != MONARCH_TILE_KEY_COLUMNS) return MONARCH_ERR_INVALID_ARG;
    monarch_status st = validate_shape(B, H, f, h, w, d, b1, b2, 1, iters, dtype, p);
    if (st != MONARCH_OK) return st;
    if (tiles < 1 || tiles > b2) return MONARCH_ERR_SHAPE;
    const int64_t BHt = (int64_t)B * H * tiles;
    if (BHt >= (1LL << 31)) return MONARCH_ERR_SHAPE;
    if (BHt * b1 * ((b2 + 7) / 8) >= (1LL << 31) || (int64_t)B * H * b2 * ((b1 + 7) / 8) >= (1LL << 31) ||
        BHt * b2 * ((b1 + 7) / 8) >= (1LL << 31))
        return MONARCH_ERR_SHAPE;
    p->tiles = tiles;
    p->unit_end = (int)BHt;
    p->key_tiles = 1;
    return MONARCH_OK;
}

}  // namespace

namespace {

// The chunk-and-cache form: queries over fq frames, keys and values over fk,
// b1*b2 = fq*h*w and b1k*b2 = fk*h*w.
monarch_status validate_kv(int B, int H, int fq, int fk, int h, int w, int d, int b1, int b1k,
                           int b2, int tiles, int iters, monarch_dtype dtype, Problem *p) {
    monarch_status st = validate_shape(B, H, fq, h, w, d, b1, b2, tiles, iters, dtype, p);
    if (st != MONARCH_OK) return st;
    if (fk < 1 || b1k < 1) return MONARCH_ERR_INVALID_ARG;
    const int64_t Nk = (int64_t)fk * h * w;
    if (Nk > (1LL << 30) || (int64_t)b1k * b2 != Nk) return MONARCH_ERR_SHAPE;
    const int64_t BHt = (int64_t)B * H * tiles;
    if (BHt * b1k * ((b2 + 7) / 8) >= (1LL << 31) || BHt * b2 * ((b1k + 7) / 8) >= (1LL << 31))
        return MONARCH_ERR_SHAPE;
    p->Nk = (int)Nk;
    p->b1k = b1k;
    return MONARCH_OK;
}

}  // namespace

namespace {

int choose_path(const Problem &p, monarch_dtype dtype) {
    return sm100_supports(p, dtype) ? 1 : 0;
}

size_t workspace_bytes_for(const Problem &p, monarch_dtype dtype, int path, bool &overflow) {
    if (path == 1) return sm100_workspace_bytes(p, overflow);
    return generic_workspace_bytes(p, overflow);
}

monarch_status run_forward(const Problem &p, monarch_dtype dtype, const void *q, const void *k,
                           const void *v, void *out, void *ws, cudaStream_t stream) {
    const int path = choose_path(p, dtype);
    cudaError_t e;
    if (path == 1) {
        int *status = status_word_on_current_device();
        if (!status) return MONARCH_ERR_CUDA;
        e = sm100_forward(p, q, k, v, out, ws, status, g_wait_limit.load(),
                          g_inject_stall.load(), stream);
    } else {
        e = generic_forward(p, dtype, q, k, v, out, generic_workspace_carve(p, ws), stream);
    }
    return e == cudaSuccess ? MONARCH_OK : MONARCH_ERR_CUDA;
}

// ---- optional per-kernel timing ------------------------------------------
struct PendingTiming {
    int id, device;
    cudaEvent_t start, stop;
};
std::mutex g_prof_mutex;
std::atomic<bool> g_prof_on{false};
std::vector<PendingTiming> g_pending;
std::map<int, std::vector<cudaEvent_t>> g_event_pool;   // per device
double g_prof_ms[K_COUNT] = {0};
long long g_prof_launches[K_COUNT] = {0};

cudaEvent_t take_event(int device) {
    {
        std::lock_guard<std::mutex> lock(g_prof_mutex);
        auto &pool = g_event_pool[device];
        if (!pool.empty()) {
            cudaEvent_t e = pool.back();
            pool.pop_back();
            return e;
        }
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

}  // namespace

ProfileScope::ProfileScope(KernelId id, cudaStream_t stream) : id_(id), stream_(stream) {
    if (!g_prof_on.load(std::memory_order_relaxed)) return;
    int dev = 0;
    cudaGetDevice(&dev);
    cudaEvent_t e = take_event(dev);
    if (e && cudaEventRecord(e, stream) == cudaSuccess) start_ = e;
}

ProfileScope::~ProfileScope() {
    if (!start_) return;
    int dev = 0;
    cudaGetDevice(&dev);
    cudaEvent_t e = take_event(dev);
    if (!e) return;
    cudaEventRecord(e, stream_);
    std::lock_guard<std::mutex> lock(g_prof_mutex);
    g_pending.push_back({(int)id_, dev, (cudaEvent_t)start_, e});
}

}  // namespace monarch

using namespace monarch;

extern "C" {

size_t monarch_attn_workspace_bytes(int B, int H, int f, int h, int w, int d, int b1, int b2,
                                    int tiles, int iters, monarch_dtype dtype) {
    Problem p;
    if (validate_shape(B, H, f, h, w, d, b1, b2, tiles, iters, dtype, &p) != MONARCH_OK) return 0;
    bool overflow = false;
    const size_t n = workspace_bytes_for(p, dtype, choose_path(p, dtype), overflow);
    return overflow ? 0 : n;
}

int monarch_attn_path(int B, int H, int f, int h, int w, int d, int b1, int b2, int tiles,
                      int iters, monarch_dtype dtype) {
    Problem p;
    if (validate_shape(B, H, f, h, w, d, b1, b2, tiles, iters, dtype, &p) != MONARCH_OK) return -1;
    return choose_path(p, dtype);
}

monarch_status monarch_attn_fwd_ws(const void *q, const void *k, const void *v, void *out, int B,
                                   int H, int f, int h, int w, int d, int b1, int b2, int tiles,
                                   int iters, monarch_dtype dtype, void *workspace,
                                   size_t ws_bytes, monarch_stream_t stream) {
    if (!q || !k || !v || !out || !workspace) return MONARCH_ERR_INVALID_ARG;
    Problem p;
    monarch_status st = validate_shape(B, H, f, h, w, d, b1, b2, tiles, iters, dtype, &p);
    if (st != MONARCH_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        ((uintptr_t)workspace & 255u))
        return MONARCH_ERR_ALIGN;
    bool overflow = false;
    const size_t need = workspace_bytes_for(p, dtype, choose_path(p, dtype), overflow);
    if (overflow) return MONARCH_ERR_SHAPE;
    if (ws_bytes < need) return MONARCH_ERR_NO_MEMORY;
    return run_forward(p, dtype, q, k, v, out, workspace, (cudaStream_t)stream);
}

monarch_status monarch_attn_fwd_layout_ws(const void *q, const void *k, const void *v, void *out,
                                          int B, int H, int f, int h, int w, int d, int b1,
                                          int b2, int tiles, int iters, monarch_dtype dtype,
                                          monarch_layout layout, void *workspace,
                                          size_t ws_bytes, monarch_stream_t stream) {
    if (!q || !k || !v || !out || !workspace) return MONARCH_ERR_INVALID_ARG;
    if (layout != MONARCH_LAYOUT_BHND && layout != MONARCH_LAYOUT_BNHD)
        return MONARCH_ERR_INVALID_ARG;
    Problem p;
    monarch_status st = validate_shape(B, H, f, h, w, d, b1, b2, tiles, iters, dtype, &p);
    if (st != MONARCH_OK) return st;
    p.layout = layout == MONARCH_LAYOUT_BNHD ? kLayoutBNHD : kLayoutBHND;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        ((uintptr_t)workspace & 255u))
        return MONARCH_ERR_ALIGN;
    bool overflow = false;
    const size_t need = workspace_bytes_for(p, dtype, choose_path(p, dtype), overflow);
    if (overflow) return MONARCH_ERR_SHAPE;
    if (ws_bytes < need) return MONARCH_ERR_NO_MEMORY;
    return run_forward(p, dtype, q, k, v, out, workspace, (cudaStream_t)stream);
}

size_t monarch_attn_tiled_workspace_bytes(int B, int H, int f, int h, int w, int d, int b1,
                                           int b2, int tiles, int iters, monarch_dtype dtype,
                                           monarch_tile_axis axis) {
    Problem p;
    if (validate_tiled(B, H, f, h, w, d, b1, b2, tiles, iters, dtype, axis, &p) != MONARCH_OK)
        return 0;
    bool overflow = false;
    const size_t n = workspace_bytes_for(p, dtype, choose_path(p, dtype), overflow);
    return overflow ? 0 : n;
}

int monarch_attn_tiled_path(int B, int H, int f, int h, int w, int d, int b1, int b2, int tiles,
                            int iters, monarch_dtype dtype, monarch_tile_axis axis) {
    Problem p;
    if (validate_tiled(B, H, f, h, w, d, b1, b2, tiles, iters, dtype, axis, &p) != MONARCH_OK)
        return -1;
    return choose_path(p, dtype);
}

monarch_status monarch_attn_fwd_tiled_ws(const void *q, const void *k, const void *v, void *out,
                                         int B, int H, int f, int h, int w, int d, int b1, int b2,
                                         int tiles, int iters, monarch_dtype dtype,
                                         monarch_tile_axis axis, monarch_layout layout,
                                         void *workspace, size_t ws_bytes,
                                         monarch_stream_t stream) {
    if (!q || !k || !v || !out || !workspace) return MONARCH_ERR_INVALID_ARG;
    if (layout != MONARCH_LAYOUT_BHND && layout != MONARCH_LAYOUT_BNHD)
        return MONARCH_ERR_INVALID_ARG;
    Problem p;
    monarch_status st = validate_tiled(B, H, f, h, w, d, b1, b2, tiles, iters, dtype, axis, &p);
    if (st != MONARCH_OK) return st;
    p.layout = layout == MONARCH_LAYOUT_BNHD ? kLayoutBNHD : kLayoutBHND;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        ((uintptr_t)workspace & 255u))
        return MONARCH_ERR_ALIGN;
    bool overflow = false;
    const size_t need = workspace_bytes_for(p, dtype, choose_path(p, dtype), overflow);
    if (overflow) return MONARCH_ERR_SHAPE;
    if (ws_bytes < need) return MONARCH_ERR_NO_MEMORY;
    return run_forward(p, dtype, q, k, v, out, workspace, (cudaStream_t)stream);
}

monarch_status monarch_attn_fwd_units_ws(const void *q, const void *k, const void *v, void *out,
                                         int B, int H, int f, int h, int w, int d, int b1, int b2,
                                         int tiles, int iters, monarch_dtype dtype, int unit_begin,
                                         int unit_end, void *workspace, size_t ws_bytes,
                                         monarch_stream_t stream) {
    if (!q || !k || !v || !out || !workspace) return MONARCH_ERR_INVALID_ARG;
    Problem p;
    monarch_status st = validate_shape(B, H, f, h, w, d, b1, b2, tiles, iters, dtype, &p);
    if (st != MONARCH_OK) return st;
    if (unit_begin < 0 || unit_end > p.unit_end || unit_begin > unit_end) return MONARCH_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        ((uintptr_t)workspace & 255u))
        return MONARCH_ERR_ALIGN;
    bool overflow = false;
    const size_t need = workspace_bytes_for(p, dtype, choose_path(p, dtype), overflow);
    if (overflow) return MONARCH_ERR_SHAPE;
    if (ws_bytes < need) return MONARCH_ERR_NO_MEMORY;
    if (unit_begin == unit_end) return MONARCH_OK;   // nothing to compute
    p.unit_begin = unit_begin;
    p.unit_end = unit_end;
    return run_forward(p, dtype, q, k, v, out, workspace, (cudaStream_t)stream);
}

size_t monarch_attn_kv_workspace_bytes(int B, int H, int fq, int fk, int h, int w, int d,
                                       int b1, int b1k, int b2, int tiles, int iters,
                                       monarch_dtype dtype) {
    Problem p;
    if (validate_kv(B, H, fq, fk, h, w, d, b1, b1k, b2, tiles, iters, dtype, &p) != MONARCH_OK)
        return 0;
    bool overflow = false;
    const size_t n = workspace_bytes_for(p, dtype, choose_path(p, dtype), overflow);
    return overflow ? 0 : n;
}

int monarch_attn_kv_path(int B, int H, int fq, int fk, int h, int w, int d, int b1, int b1k,
                         int b2, int tiles, int iters, monarch_dtype dtype) {
    Problem p;
    if (validate_kv(B, H, fq, fk, h, w, d, b1, b1k, b2, tiles, iters, dtype, &p) != MONARCH_OK)
        return -1;
    return choose_path(p, dtype);
}

monarch_status monarch_attn_fwd_kv_ws(const void *q, const void *k, const void *v, void *out,
                                      int B, int H, int fq, int fk, int h, int w, int d, int b1,
                                      int b1k, int b2, int tiles, int iters, monarch_dtype dtype,
                                      void *workspace, size_t ws_bytes, monarch_stream_t stream) {
    if (!q || !k || !v || !out || !workspace) return MONARCH_ERR_INVALID_ARG;
    Problem p;
    monarch_status st = validate_kv(B, H, fq, fk, h, w, d, b1, b1k, b2, tiles, iters, dtype, &p);
    if (st != MONARCH_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        ((uintptr_t)workspace & 255u))
        return MONARCH_ERR_ALIGN;
    bool overflow = false;
    const size_t need = workspace_bytes_for(p, dtype, choose_path(p, dtype), overflow);
    if (overflow) return MONARCH_ERR_SHAPE;
    if (ws_bytes < need) return MONARCH_ERR_NO_MEMORY;
    return run_forward(p, dtype, q, k, v, out, workspace, (cudaStream_t)stream);
}

monarch_status monarch_attn_fwd(const void *q, const void *k, const void *v, void *out, int B,
                                int H, int f, int h, int w, int d, int b1, int b2, int tiles,
                                int iters, monarch_dtype dtype, monarch_stream_t stream) {
    if (!q || !k || !v || !out) return MONARCH_ERR_INVALID_ARG;
    Problem p;
    monarch_status st = validate_shape(B, H, f, h, w, d, b1, b2, tiles, iters, dtype, &p);
    if (st != MONARCH_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return MONARCH_ERR_ALIGN;
    bool overflow = false;
    const size_t need = workspace_bytes_for(p, dtype, choose_path(p, dtype), overflow);
    if (overflow) return MONARCH_ERR_SHAPE;
    configure_pool_once();
    void *ws = nullptr;
    if (cudaMallocAsync(&ws, need, (cudaStream_t)stream) != cudaSuccess) {
        cudaGetLastError();
        return MONARCH_ERR_NO_MEMORY;
    }
    st = run_forward(p, dtype, q, k, v, out, ws, (cudaStream_t)stream);
    if (cudaFreeAsync(ws, (cudaStream_t)stream) != cudaSuccess && st == MONARCH_OK)
        st = MONARCH_ERR_CUDA;
    return st;
}

// Backward pass of one iteration (generic SIMT kernels): see the header.
size_t monarch_attn_bwd_workspace_bytes(int B, int H, int f, int h, int w, int d, int b1, int b2,
                                        int tiles, int iters, monarch_dtype dtype) {
    Problem p;
    if (validate_shape(B, H, f, h, w, d, b1, b2, tiles, iters, dtype, &p) != MONARCH_OK ||
        iters != 1)
        return 0;
    bool overflow = false;
    const size_t n = backward_workspace_bytes(p, dtype, overflow);
    return overflow ? 0 : n;
}

monarch_status monarch_attn_bwd_ws(const void *q, const void *k, const void *v, const void *dy,
                                   void *dq, void *dk, void *dv, int B, int H, int f, int h,
                                   int w, int d, int b1, int b2, int tiles, int iters,
                                   monarch_dtype dtype, void *workspace, size_t ws_bytes,
                                   monarch_stream_t stream) {
    if (!q || !k || !v || !dy || !dq || !dk || !dv || !workspace) return MONARCH_ERR_INVALID_ARG;
    Problem p;
    monarch_status st = validate_shape(B, H, f, h, w, d, b1, b2, tiles, iters, dtype, &p);
    if (st != MONARCH_OK) return st;
    if (iters != 1) return MONARCH_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dy) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv) || ((uintptr_t)workspace & 255u))
        return MONARCH_ERR_ALIGN;
    bool overflow = false;
    const size_t need = backward_workspace_bytes(p, dtype, overflow);
    if (overflow) return MONARCH_ERR_SHAPE;
    if (ws_bytes < need) return MONARCH_ERR_NO_MEMORY;
    int *status = status_word_on_current_device();
    return generic_backward(p, dtype, q, k, v, dy, dq, dk, dv, workspace, status,
                            g_wait_limit.load(), (cudaStream_t)stream) == cudaSuccess
               ? MONARCH_OK
               : MONARCH_ERR_CUDA;
}

monarch_status monarch_attn_bwd(const void *q, const void *k, const void *v, const void *dy,
                                void *dq, void *dk, void *dv, int B, int H, int f, int h, int w,
                                int d, int b1, int b2, int tiles, int iters, monarch_dtype dtype,
                                monarch_stream_t stream) {
    const size_t need = monarch_attn_bwd_workspace_bytes(B, H, f, h, w, d, b1, b2, tiles, iters,
                                                         dtype);
    if (need == 0) {
        Problem p;
        monarch_status st = validate_shape(B, H, f, h, w, d, b1, b2, tiles, iters, dtype, &p);
        return st != MONARCH_OK ? st : (iters != 1 ? MONARCH_ERR_UNSUPPORTED : MONARCH_ERR_SHAPE);
    }
    if (!q || !k || !v || !dy || !dq || !dk || !dv) return MONARCH_ERR_INVALID_ARG;
    configure_pool_once();
    void *ws = nullptr;
    if (cudaMallocAsync(&ws, need, (cudaStream_t)stream) != cudaSuccess) {
        cudaGetLastError();
        return MONARCH_ERR_NO_MEMORY;
    }
    monarch_status st = monarch_attn_bwd_ws(q, k, v, dy, dq, dk, dv, B, H, f, h, w, d, b1, b2,
                                            tiles, iters, dtype, ws, need, stream);
    if (cudaFreeAsync(ws, (cudaStream_t)stream) != cudaSuccess && st == MONARCH_OK)
        st = MONARCH_ERR_CUDA;
    return st;
}

monarch_status monarch_attn_fwd_host(const void *q, const void *k, const void *v, void *out,
                                     int B, int H, int f, int h, int w, int d, int b1, int b2,
                                     int tiles, int iters, monarch_dtype dtype,
                                     monarch_stream_t stream) {
    if (!q || !k || !v || !out) return MONARCH_ERR_INVALID_ARG;
    Problem p;
    monarch_status st = validate_shape(B, H, f, h, w, d, b1, b2, tiles, iters, dtype, &p);
    if (st != MONARCH_OK) return st;
    bool overflow = false;
    const size_t need = workspace_bytes_for(p, dtype, choose_path(p, dtype), overflow);
    if (overflow) return MONARCH_ERR_SHAPE;
    const size_t es = dtype == MONARCH_BF16 ? 2 : 4;
    const size_t tensor = (size_t)p.BH * p.N * p.d * es;
    const size_t slot = align256(tensor);
    cudaStream_t s = (cudaStream_t)stream;
    configure_pool_once();
    char *dev = nullptr;
    if (cudaMallocAsync((void **)&dev, 4 * slot + need, s) != cudaSuccess) {
        cudaGetLastError();
        return MONARCH_ERR_NO_MEMORY;
    }
    char *dq = dev, *dk = dev + slot, *dv = dev + 2 * slot, *dout = dev + 3 * slot;
    void *ws = dev + 4 * slot;
    if (cudaMemcpyAsync(dq, q, tensor, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(dk, k, tensor, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(dv, v, tensor, cudaMemcpyHostToDevice, s) != cudaSuccess) {
        st = MONARCH_ERR_CUDA;
    } else {
        st = run_forward(p, dtype, dq, dk, dv, dout, ws, s);
        if (st == MONARCH_OK &&
            cudaMemcpyAsync(out, dout, tensor, cudaMemcpyDeviceToHost, s) != cudaSuccess)
            st = MONARCH_ERR_CUDA;
    }
    if (cudaFreeAsync(dev, s) != cudaSuccess && st == MONARCH_OK) st = MONARCH_ERR_CUDA;
    return st;
}

monarch_status monarch_index_maps(int f, int h, int w, int b1, int b2, int tiles, int32_t *u_of_n,
                                  int32_t *v_of_n, int32_t *perm, int32_t *tile_lo) {
    const int64_t N = (int64_t)f * h * w;
    if (f < 1 || h < 1 || w < 1 || b1 < 1 || b2 < 1) return MONARCH_ERR_INVALID_ARG;
    if (N > (1LL << 30) || (int64_t)b1 * b2 != N || tiles < 1 || tiles > b1)
        return MONARCH_ERR_SHAPE;
    for (int64_t n = 0; n < N; n++) {
        const int u = block_row(n, b2), v = block_col(n, b2);
        if (u_of_n) u_of_n[n] = u;
        if (v_of_n) v_of_n[n] = v;
        if (perm) perm[n] = (int32_t)shuffle(u, v, b1);
    }
    if (tile_lo)
        for (int g = 0; g <= tiles; g++) tile_lo[g] = tile_begin(g, b1, tiles);
    return MONARCH_OK;
}

monarch_status monarch_index_maps_device(int f, int h, int w, int b1, int b2, int tiles,
                                         int32_t *u_of_n, int32_t *v_of_n, int32_t *perm,
                                         int32_t *tile_lo, monarch_stream_t stream) {
    const int64_t N = (int64_t)f * h * w;
    if (f < 1 || h < 1 || w < 1 || b1 < 1 || b2 < 1) return MONARCH_ERR_INVALID_ARG;
    if (N > (1LL << 30) || (int64_t)b1 * b2 != N || tiles < 1 || tiles > b1)
        return MONARCH_ERR_SHAPE;
    cudaError_t e = index_maps_device((int)N, b1, b2, tiles, u_of_n, v_of_n, perm, tile_lo,
                                      (cudaStream_t)stream);
    return e == cudaSuccess ? MONARCH_OK : MONARCH_ERR_CUDA;
}

monarch_status monarch_last_device_status(monarch_stream_t stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MONARCH_ERR_CUDA;
    int *status = status_word_on_current_device();
    if (!status) return MONARCH_ERR_CUDA;
    int value = 0, zero = 0;
    if (cudaMemcpy(&value, status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
        return MONARCH_ERR_CUDA;
    return (monarch_status)value;
}

long long monarch_set_wait_limit(long long spins) {
    return g_wait_limit.exchange(spins > 0 ? spins : kDefaultWaitLimit);
}

int monarch_debug_inject_stall(int on) { return g_inject_stall.exchange(on != 0 ? 1 : 0); }

monarch_status monarch_profile_enable(int on) {
    g_prof_on.store(on != 0);
    return MONARCH_OK;
}

int monarch_profile_collect(double *ms, long long *launches, int max_kernels) {
    std::vector<PendingTiming> pending;
    {
        std::lock_guard<std::mutex> lock(g_prof_mutex);
        pending.swap(g_pending);
    }
    bool ok = true;
    int prev = 0;
    cudaGetDevice(&prev);
    for (const PendingTiming &t : pending) {
        float el = 0.f;
        cudaSetDevice(t.device);
        if (cudaEventSynchronize(t.stop) != cudaSuccess ||
            cudaEventElapsedTime(&el, t.start, t.stop) != cudaSuccess)
            ok = false;
        std::lock_guard<std::mutex> lock(g_prof_mutex);
        g_prof_ms[t.id] += el;
        g_prof_launches[t.id] += 1;
        g_event_pool[t.device].push_back(t.start);
        g_event_pool[t.device].push_back(t.stop);
    }
    cudaSetDevice(prev);
    std::lock_guard<std::mutex> lock(g_prof_mutex);
    for (int kk = 0; kk < K_COUNT && kk < max_kernels; kk++) {
        if (ms) ms[kk] = g_prof_ms[kk];
        if (launches) launches[kk] = g_prof_launches[kk];
    }
    for (int kk = 0; kk < K_COUNT; kk++) {
        g_prof_ms[kk] = 0;
        g_prof_launches[kk] = 0;
    }
    return ok ? (int)K_COUNT : -1;
}

const char *monarch_profile_kernel_name(int k) {
    static const char *names[K_COUNT] = {"qbar_mean_kernel",     "rstep_kernel",
                                         "lstep_kernel",         "qbar_weighted_kernel",
                                         "tc_qbar_kernel",       "tc_rstep_kernel",
                                         "tc_lstep_kernel",      "tc_lstat_kernel",
                                         "tc_qagg_kernel", "bwd_lstep_kernels",
                                         "bwd_rstep_kernels",    "tc_bwd_dq_kernel<0>",
                                         "tc_bwd_dkz_kernel",    "tc_bwd_dq_kernel<1>",
                                         "tc_bwd_r_kernel",      "tc_bwd_dqbar+combine"};
    return (k >= 0 && k < K_COUNT) ? names[k] : nullptr;
}

const char *monarch_status_string(monarch_status status) {
    switch (status) {
        case MONARCH_OK: return "ok";
        case MONARCH_ERR_INVALID_ARG: return "invalid argument";
        case MONARCH_ERR_SHAPE: return "inconsistent or too large shape";
        case MONARCH_ERR_ALIGN: return "pointer not 16-byte aligned";
        case MONARCH_ERR_UNSUPPORTED: return "unsupported head dimension";
        case MONARCH_ERR_NO_MEMORY: return "workspace allocation failed or too small";
        case MONARCH_ERR_CUDA: return "CUDA error";
        case MONARCH_ERR_TIMEOUT: return "device-side wait timed out";
        case MONARCH_ERR_SCRATCH_LIMIT:
            return "problem needs more scratch than the no-allocation entry point's static buffer";
    }
    return "unknown status";
}

}  // extern "C"
