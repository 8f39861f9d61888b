// hsa_api.cu -- the extern "C" entry points declared in include/hsa.h:
// argument checks, workspace carving, and the kernel sequence of each call.
#include <algorithm>
#include <atomic>
#include <climits>
#include <cstring>

#include "hsa_internal.cuh"

namespace hsa {

// ------------------------------------------------------------------ wait limit
static std::atomic<uint64_t> g_wait_ns{0};  // 0: the default

uint64_t wait_limit_ns() {
    const uint64_t v = g_wait_ns.load(std::memory_order_relaxed);
    return v ? v : kDefaultWaitNs;
}

// ------------------------------------------------------------------ checks
static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

hsa_status_t check_shape(const hsa_shape_t *s, bool decode) {
    if (!s) return HSA_ERR_INVALID_ARG;
    if (s->B < 0 || s->L < 0 || s->h_q < 1 || s->h_kv < 1 || s->d < 1 || s->S < 1 || s->K < 1)
        return HSA_ERR_INVALID_ARG;
    if (s->h_q % s->h_kv != 0) return HSA_ERR_INVALID_ARG;
    if (s->dtype != HSA_F32 && s->dtype != HSA_BF16) return HSA_ERR_INVALID_ARG;
    if (s->S != 16 && s->S != 32 && s->S != 64 && s->S != 128) return HSA_ERR_UNSUPPORTED;
    if (s->d != 64 && s->d != 128) return HSA_ERR_UNSUPPORTED;
    if (s->K > kMaxK || s->h_q / s->h_kv > kMaxG) return HSA_ERR_UNSUPPORTED;
    // entries pack t * 16 + slot into int32; list offsets are int32
    if ((int64_t)s->L * 16 >= ((int64_t)1 << 31) || (int64_t)s->L * s->K >= ((int64_t)1 << 31))
        return HSA_ERR_UNSUPPORTED;
    if ((int64_t)s->B * s->h_kv > 65535 && !decode) return HSA_ERR_UNSUPPORTED;  // grid.y
    return HSA_OK;
}

// all pointers in the list must be non-null and 16-byte aligned
static bool ptrs_ok(std::initializer_list<const void *> ps) {
    for (const void *p : ps)
        if (!p || !aligned16(p)) return false;
    return true;
}
static bool opt_ok(const void *p) { return !p || aligned16(p); }

// ------------------------------------------------------------------ workspace
struct Carver {
    char *base;
    size_t off = kWsHeader;
    template <typename T> T *take(size_t count) {
        T *p = base ? reinterpret_cast<T *>(base + off) : nullptr;
        off += round_up((int64_t)(count * sizeof(T)), 256);
        return p;
    }
};

struct FwdWs {
    float *kbar;
    int32_t *idx;
    float *w;
    __nv_bfloat16 *kb_hi, *kb_lo;  // split pooled keys for the tensor-core scores
    bool tc;             // chunk-major tensor-core path
    int32_t *entries;    // per (b, g): nW windows x W*K (token, slot) entries, bucket by bucket
    float *entw;         //   and their weights
    int32_t *bucket_hist;  // [J][blocks][nc] per token block chunk counts -> positions
    AttendPlan plan;
    __half *acc;         // fp16 output-accumulator ring, scaled (chunk-major path)
    size_t zero_bytes;   // the plan counters: cleared by one memset per call
};

// token->chunk lists of the chunk-major passes (with the entries' weights if `weights`)
static void carve_lists(Carver &c, const Shape &sh, BwdWs &inv, bool weights) {
    const int ntb = (int)ceil_div(sh.L, kInvTokBlock);
    inv.hist = c.take<int32_t>((size_t)sh.B * sh.hkv * ntb * sh.nc);
    inv.chunk_off = c.take<int32_t>((size_t)sh.B * sh.hkv * (sh.nc + 1));
    inv.seg_off = c.take<int32_t>((size_t)sh.B * sh.hkv * (sh.nc + 1));
    inv.entries = c.take<int32_t>((size_t)sh.B * sh.hkv * sh.L * sh.K);
    inv.entw = weights ? c.take<float>((size_t)sh.B * sh.hkv * sh.L * sh.K) : nullptr;
}

// work plan of the chunk-major passes: windows, units of up to `unit_tiles` tiles, queue
static void carve_plan(Carver &c, const Shape &sh, AttendPlan &P, int unit_tiles, int acc_bytes) {
    P.B = sh.B; P.L = sh.L; P.hq = sh.hq; P.hkv = sh.hkv; P.D = sh.d; P.K = sh.K; P.G = sh.G;
    P.nc = sh.nc; P.ntb = (int)ceil_div(sh.L, kInvTokBlock);
    P.W = (int)std::min<int64_t>(attend_window(sh.G, sh.d, acc_bytes), round_up(std::max(sh.L, 1), kInvTokBlock));
    P.nW = (int)ceil_div(sh.L, P.W); P.J = sh.B * sh.hkv * P.nW; P.TT = 128 / sh.G;
    P.unit_tiles = unit_tiles;
    P.unit_prefix = c.take<int32_t>((size_t)P.J * (sh.nc + 1));
    P.win_units = c.take<int32_t>((size_t)P.J);
    P.win_tiles = c.take<int32_t>((size_t)P.J);
    P.win_ncomb = c.take<int32_t>((size_t)P.J);
    P.seg_start = c.take<int32_t>((size_t)P.J + 1);
    P.counters = c.take<int32_t>(plan_counter_count(P.J));
    // work units <= tiles <= L*K/TT + nc per window, summed over (b, g)
    P.max_items = (int)std::min<int64_t>(
        ((int64_t)sh.B * sh.hkv * ((int64_t)sh.L * sh.K / P.TT + (int64_t)P.nW * sh.nc) + 16),
        (int64_t)INT32_MAX / 4);
    P.items = c.take<int4>((size_t)2 * P.max_items);
    P.win_cap = 0;
    P.ent_stride = (int64_t)sh.L * sh.K;
}

static FwdWs carve_fwd(const Shape &sh, void *ws, size_t *bytes) {
    Carver c{static_cast<char *>(ws)};
    FwdWs f{};
    f.kbar = c.take<float>((size_t)sh.B * sh.hkv * sh.nc * sh.d);
    f.idx = c.take<int32_t>((size_t)sh.B * sh.L * sh.hkv * sh.K);
    f.w = c.take<float>((size_t)sh.B * sh.L * sh.hkv * sh.K);
    if (select_tc_supported(sh)) {
        f.kb_hi = c.take<__nv_bfloat16>((size_t)sh.B * sh.hkv * sh.nc * sh.d);
        f.kb_lo = c.take<__nv_bfloat16>((size_t)sh.B * sh.hkv * sh.nc * sh.d);
    }
    f.tc = attend_tc_supported(sh);
    if (f.tc) {
        // bucket plan: each window owns a fixed slice of the entries and of the queue
        AttendPlan &P = f.plan;
        P.B = sh.B; P.L = sh.L; P.hq = sh.hq; P.hkv = sh.hkv; P.D = sh.d; P.K = sh.K; P.G = sh.G;
        P.nc = sh.nc; P.ntb = (int)ceil_div(sh.L, kInvTokBlock);
        P.W = (int)std::min<int64_t>(attend_window(sh.G, sh.d, kFwdAccBytes), round_up(std::max(sh.L, 1), kInvTokBlock));
        P.nW = (int)ceil_div(sh.L, P.W); P.J = sh.B * sh.hkv * P.nW; P.TT = 128 / sh.G;
        P.unit_tiles = kUnitTiles;
        P.ent_stride = (int64_t)P.nW * P.W * sh.K;
        // units of a window <= its tiles <= W*K/TT + nc (one ragged tile per bucket)
        P.win_cap = (int)std::min<int64_t>((int64_t)P.W * sh.K / P.TT + sh.nc, INT32_MAX / 4);
        P.max_items = (int)std::min<int64_t>((int64_t)P.J * P.win_cap, INT32_MAX / 4);
        f.entries = c.take<int32_t>((size_t)sh.B * sh.hkv * P.ent_stride);
        f.entw = c.take<float>((size_t)sh.B * sh.hkv * P.ent_stride);
        P.unit_prefix = nullptr;
        P.win_units = c.take<int32_t>((size_t)P.J);
        P.win_tiles = c.take<int32_t>((size_t)P.J);
        P.win_ncomb = c.take<int32_t>((size_t)P.J);
        P.seg_start = c.take<int32_t>((size_t)P.J + 1);
        P.items = c.take<int4>((size_t)2 * P.J * P.win_cap);
        f.bucket_hist = c.take<int32_t>(bucket_hist_elems(P));
        const size_t z0 = c.off;
        P.counters = c.take<int32_t>(plan_counter_count(P.J));
        f.zero_bytes = c.off - z0;
        f.acc = c.take<__half>(attend_acc_elems(P.W, sh.G, sh.d));
    }
    if (bytes) *bytes = c.off;
    return f;
}

struct BwdAll {
    BwdWs b;
    bool tc;          // chunk-major tensor-core path
    AttendPlan plan;
    __half *acc;      // fp16 dq accumulator ring, scaled (tensor-core path)
    float *dw;        // [B,L,h_kv,K] gradients of the chunk weights (tensor-core path)
};

constexpr int kBwdUnitTiles = 16;  // backward work units: up to 16 tiles (one dK/dV flush each)

static BwdAll carve_bwd(const Shape &sh, void *ws, size_t *bytes) {
    Carver c{static_cast<char *>(ws)};
    BwdAll r{};
    BwdWs &b = r.b;
    r.tc = bwd_tc_supported(sh) && sh.nc > 0;
    b.dkbar = c.take<float>((size_t)sh.B * sh.hkv * sh.nc * sh.d);
    b.delta = r.tc ? nullptr : c.take<float>((size_t)sh.B * sh.L * sh.hq * sh.K);
    b.dk_acc = c.take<float>((size_t)sh.B * sh.hkv * sh.L * sh.d);
    b.dv_acc = c.take<float>((size_t)sh.B * sh.hkv * sh.L * sh.d);
    carve_lists(c, sh, b, r.tc);
    if (r.tc) {
        r.dw = c.take<float>((size_t)sh.B * sh.L * sh.hkv * sh.K);
        carve_plan(c, sh, r.plan, kBwdUnitTiles, kBwdAccBytes);
        r.acc = c.take<__half>(attend_acc_elems(r.plan.W, sh.G, sh.d));
    }
    if (bytes) *bytes = c.off;
    return r;
}

static size_t ws_size(const Shape &sh, int op) {
    size_t bytes = kWsHeader;
    switch (op) {
        case HSA_OP_POOL:
        case HSA_OP_DECODE:
            return bytes;
        case HSA_OP_SELECT:
            if (select_tc_supported(sh))
                bytes += 2 * round_up((int64_t)sizeof(__nv_bfloat16) * sh.B * sh.hkv * sh.nc * sh.d, 256);
            return bytes;
        case HSA_OP_FWD:
            carve_fwd(sh, nullptr, &bytes);
            return bytes;
        case HSA_OP_BWD:
            carve_bwd(sh, nullptr, &bytes);
            return bytes;
        default:
            return 0;
    }
}

static hsa_status_t check_ws(const Shape &sh, int op, void *ws, size_t ws_bytes) {
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return HSA_ERR_INVALID_ARG;
    if (ws_bytes < ws_size(sh, op)) return HSA_ERR_WORKSPACE;
    return HSA_OK;
}

static hsa_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? HSA_OK : HSA_ERR_CUDA; }

// A problem with no tokens reads and writes nothing: its tensors may be empty
// (null data pointers); only the workspace status word is cleared.
static hsa_status_t empty_call(const Shape &sh, int op, void *ws, size_t ws_bytes, cudaStream_t st) {
    hsa_status_t s = check_ws(sh, op, ws, ws_bytes);
    if (s != HSA_OK) return s;
    return cuda_status(cudaMemsetAsync(ws, 0, sizeof(DevStatus), st));
}

static cudaError_t clear_status(void *ws, cudaStream_t st) {
    return cudaMemsetAsync(ws, 0, sizeof(DevStatus), st);
}

// selection (a2-a4): tensor-core scores for bf16 inputs, CUDA cores otherwise
static cudaError_t run_select(const Shape &sh, const void *q_slc, const float *kbar, __nv_bfloat16 *hi,
                              __nv_bfloat16 *lo, int32_t *idx, float *w, DevStatus *ds, cudaStream_t st);

// run a launcher inside a timing bracket of `kind` covering `n` kernel launches
template <typename F> static cudaError_t timed(int kind, int n, cudaStream_t st, F &&f) {
    TimedLaunch tl(kind, n, st);
    return f();
}

static cudaError_t run_select(const Shape &sh, const void *q_slc, const float *kbar, __nv_bfloat16 *hi,
                              __nv_bfloat16 *lo, int32_t *idx, float *w, DevStatus *ds, cudaStream_t st) {
    TimedLaunch tl(HSA_K_SELECT, 1, st);
    if (hi && lo) return launch_select_tc(sh, q_slc, kbar, hi, lo, idx, w, ds, st);
    return launch_select_simt(sh, q_slc, kbar, idx, w, ds, st);
}

}  // namespace hsa

using namespace hsa;

extern "C" {

size_t hsa_workspace_size(const hsa_shape_t *shape, int op) {
    if (check_shape(shape, op == HSA_OP_DECODE) != HSA_OK) return 0;
    return ws_size(make_shape(*shape), op);
}

hsa_status_t hsa_pool(const hsa_shape_t *shape, const void *k, float *kbar, void *ws, size_t ws_bytes,
                      void *stream) {
    hsa_status_t s = check_shape(shape, false);
    if (s != HSA_OK) return s;
    const Shape sh = make_shape(*shape);
    if ((int64_t)sh.B * sh.L == 0) return empty_call(sh, HSA_OP_POOL, ws, ws_bytes, static_cast<cudaStream_t>(stream));
    if (!ptrs_ok({k, kbar})) return HSA_ERR_INVALID_ARG;
    if ((s = check_ws(sh, HSA_OP_POOL, ws, ws_bytes)) != HSA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    DevStatus *ds = static_cast<DevStatus *>(ws);
    cudaError_t e = clear_status(ws, st);
    if (e == cudaSuccess) e = timed(HSA_K_POOL, 1, st, [&] { return launch_pool(sh, k, kbar, ds, st); });
    return cuda_status(e);
}

hsa_status_t hsa_select(const hsa_shape_t *shape, const void *q_slc, const void *k, float *kbar,
                        int32_t *idx, float *w, void *ws, size_t ws_bytes, void *stream) {
    hsa_status_t s = check_shape(shape, false);
    if (s != HSA_OK) return s;
    const Shape sh = make_shape(*shape);
    if ((int64_t)sh.B * sh.L == 0) return empty_call(sh, HSA_OP_SELECT, ws, ws_bytes, static_cast<cudaStream_t>(stream));
    if (!ptrs_ok({q_slc, k, kbar, idx, w})) return HSA_ERR_INVALID_ARG;
    if ((s = check_ws(sh, HSA_OP_SELECT, ws, ws_bytes)) != HSA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    DevStatus *ds = static_cast<DevStatus *>(ws);
    __nv_bfloat16 *hi = nullptr, *lo = nullptr;
    if (select_tc_supported(sh)) {
        Carver c{static_cast<char *>(ws)};
        hi = c.take<__nv_bfloat16>((size_t)sh.B * sh.hkv * sh.nc * sh.d);
        lo = c.take<__nv_bfloat16>((size_t)sh.B * sh.hkv * sh.nc * sh.d);
    }
    cudaError_t e = clear_status(ws, st);
    PoolExtras px;  // the pooling pass also writes the bf16 split the tensor-core scores use
    px.hi = hi;
    px.lo = lo;
    if (e == cudaSuccess) e = timed(HSA_K_POOL, 1, st, [&] { return launch_pool(sh, k, kbar, ds, st, px); });
    if (e == cudaSuccess) e = run_select(sh, q_slc, kbar, hi, lo, idx, w, ds, st);
    return cuda_status(e);
}

// attention + fusion (a5-a6) for a given selection f.idx / f.w: tensor-core chunk-major
// path (inversion, plan, attend) for the shapes it takes, CUDA cores otherwise
// given_sel: a caller-given selection (hsa_attend); otherwise the forward's own,
// whose pooling pass has already cleared the plan counters and written max|v|
static cudaError_t run_attend(const Shape &sh, const void *q, const void *k, const void *v, FwdWs &f, void *o,
                              float *lse, bool given_sel, DevStatus *ds, cudaStream_t st) {
    cudaError_t e = cudaSuccess;
    if (!f.tc) {
        if (e == cudaSuccess)
            e = timed(HSA_K_ATTEND_SIMT, 1, st, [&] { return launch_attend_simt(sh, q, k, v, f.idx, f.w, o, lse, ds, st); });
        return e;
    }
    // chunk-major tensor-core path: bucket the selection by (window, chunk), queue the
    // work units, attend.  The forward's pooling pass has cleared the plan counters
    // already (and written max|v|); a caller-given selection clears them here.
    if (e == cudaSuccess && given_sel) e = cudaMemsetAsync(f.plan.counters, 0, f.zero_bytes, st);
    if (e == cudaSuccess)
        e = timed(HSA_K_INVERT, sh.nc > 0 ? 3 : 1, st, [&] {
            return launch_bucket_plan(sh, f.idx, f.w, f.plan, f.bucket_hist, f.entries, f.entw, ds, st);
        });
    if (e == cudaSuccess)  // the used accumulator slots start at zero (the kernel re-zeroes them after use)
        e = cudaMemsetAsync(f.acc, 0,
                            sizeof(__half) * std::min<size_t>(attend_acc_elems(f.plan.W, sh.G, sh.d),
                                                             (size_t)f.plan.J * f.plan.W * sh.G * sh.d),
                            st);
    if (e == cudaSuccess && lse)
        e = cudaMemsetAsync(lse, 0, sizeof(float) * (size_t)sh.B * sh.L * sh.hq * sh.K, st);
    if (e == cudaSuccess && given_sel)  // the accumulators' power-of-two scale comes from max|v|
        e = timed(HSA_K_PLAN, 1, st, [&] { return launch_vmax(sh, v, f.plan.counters + 3 * f.plan.J + 1, st); });
    if (e == cudaSuccess && given_sel)  // weights not from stick-breaking: their row sums may exceed 1
        e = timed(HSA_K_PLAN, 1, st, [&] { return launch_wsum(sh, f.idx, f.w, f.plan.counters + 3 * f.plan.J + 2, st); });
    if (e == cudaSuccess)
        e = timed(HSA_K_ATTEND_TC, 1, st, [&] {
            return launch_attend_tc(sh, f.plan, f.entries, f.entw, q, k, v, f.acc, o, lse, ds, st);
        });
    return e;
}

hsa_status_t hsa_fwd(const hsa_shape_t *shape, const void *q, const void *k, const void *v,
                     const void *q_slc, void *o, float *lse, int32_t *idx, float *w, float *kbar,
                     void *ws, size_t ws_bytes, void *stream) {
    hsa_status_t s = check_shape(shape, false);
    if (s != HSA_OK) return s;
    const Shape sh = make_shape(*shape);
    if ((int64_t)sh.B * sh.L == 0) return empty_call(sh, HSA_OP_FWD, ws, ws_bytes, static_cast<cudaStream_t>(stream));
    if (!ptrs_ok({q, k, v, q_slc, o}) || !opt_ok(lse) || !opt_ok(idx) || !opt_ok(w) || !opt_ok(kbar))
        return HSA_ERR_INVALID_ARG;
    if ((s = check_ws(sh, HSA_OP_FWD, ws, ws_bytes)) != HSA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    DevStatus *ds = static_cast<DevStatus *>(ws);
    FwdWs f = carve_fwd(sh, ws, nullptr);
    if (kbar) f.kbar = kbar;
    if (idx) f.idx = idx;
    if (w) f.w = w;
    cudaError_t e = clear_status(ws, st);
    PoolExtras px;  // the bf16 split for the tensor-core scores, max|v| for the accumulators' scale
    px.hi = f.kb_hi;
    px.lo = f.kb_lo;
    if (f.tc) {
        if (e == cudaSuccess) e = cudaMemsetAsync(f.plan.counters, 0, f.zero_bytes, st);
        px.v = v;
        px.vmax_bits = f.plan.counters + 3 * f.plan.J + 1;
    }
    if (e == cudaSuccess) e = timed(HSA_K_POOL, 1, st, [&] { return launch_pool(sh, k, f.kbar, ds, st, px); });
    if (e == cudaSuccess) e = run_select(sh, q_slc, f.kbar, f.kb_hi, f.kb_lo, f.idx, f.w, ds, st);
    if (e == cudaSuccess) e = run_attend(sh, q, k, v, f, o, lse, false, ds, st);
    return cuda_status(e);
}

hsa_status_t hsa_attend(const hsa_shape_t *shape, const void *q, const void *k, const void *v,
                        const int32_t *idx, const float *w, void *o, float *lse, void *ws, size_t ws_bytes,
                        void *stream) {
    hsa_status_t s = check_shape(shape, false);
    if (s != HSA_OK) return s;
    const Shape sh = make_shape(*shape);
    if ((int64_t)sh.B * sh.L == 0) return empty_call(sh, HSA_OP_FWD, ws, ws_bytes, static_cast<cudaStream_t>(stream));
    if (!ptrs_ok({q, k, v, idx, w, o}) || !opt_ok(lse)) return HSA_ERR_INVALID_ARG;
    if ((s = check_ws(sh, HSA_OP_FWD, ws, ws_bytes)) != HSA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    DevStatus *ds = static_cast<DevStatus *>(ws);
    FwdWs f = carve_fwd(sh, ws, nullptr);
    f.idx = const_cast<int32_t *>(idx);  // read only from here on
    f.w = const_cast<float *>(w);
    cudaError_t e = clear_status(ws, st);
    if (e == cudaSuccess) e = run_attend(sh, q, k, v, f, o, lse, true, ds, st);
    return cuda_status(e);
}

// The address a kernel reads `p` through: device (or managed) memory as is,
// page-locked host memory through its mapped device address.  Pageable host
// memory has no such address and is refused before any launch.
static bool device_view(const void *p, const void **dp) {
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        (void)cudaGetLastError();  // a plain host pointer: clear the sticky-free error state
        return false;
    }
    if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) {
        *dp = p;
        return true;
    }
    if (a.type == cudaMemoryTypeHost && a.devicePointer) {
        *dp = a.devicePointer;
        return aligned16(*dp);
    }
    return false;
}

hsa_status_t hsa_decode_multi(const hsa_shape_t *shape, int32_t n_layers, const void *q, const void *q_slc,
                              const void *k_cache, const void *v_cache, const float *kbar, void *o,
                              int32_t *idx, float *w, void *ws, size_t ws_bytes, void *stream) {
    hsa_status_t s = check_shape(shape, true);
    if (s != HSA_OK) return s;
    if (n_layers < 1 || n_layers > HSA_MAX_LAYERS) return HSA_ERR_INVALID_ARG;
    const Shape sh = make_shape(*shape);
    if (sh.B == 0) return empty_call(sh, HSA_OP_DECODE, ws, ws_bytes, static_cast<cudaStream_t>(stream));
    if (!ptrs_ok({q, q_slc, o}) || !opt_ok(idx) || !opt_ok(w)) return HSA_ERR_INVALID_ARG;
    // with no complete cached chunk the caches and the index are never read
    if (sh.nc > 0 && !ptrs_ok({k_cache, v_cache, kbar})) return HSA_ERR_INVALID_ARG;
    if ((s = check_ws(sh, HSA_OP_DECODE, ws, ws_bytes)) != HSA_OK) return s;
    const void *kc = k_cache, *vc = v_cache;
    if (sh.nc > 0 && (!device_view(k_cache, &kc) || !device_view(v_cache, &vc))) return HSA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    DevStatus *ds = static_cast<DevStatus *>(ws);
    const bool cluster = decode_cluster_supported(sh, n_layers);
    cudaError_t e = clear_status(ws, st);
    if (e == cudaSuccess)
        e = timed(HSA_K_DECODE, cluster ? 1 : n_layers, st, [&] {
            if (cluster)
                return launch_decode_cluster(sh, n_layers, q, q_slc, kc, vc, kbar, o, idx, w, ds, st);
            // very long caches, or more layers x heads than the cluster's shared memory holds:
            // token-major kernel, one launch per layer (each repeats the selection)
            const size_t lbytes = (size_t)sh.B * sh.hq * sh.d * (sh.bf16 ? 2 : 4);
            cudaError_t r = cudaSuccess;
            for (int l = 0; l < n_layers && r == cudaSuccess; ++l)
                r = launch_decode_simt(sh, static_cast<const char *>(q) + l * lbytes, q_slc, kc, vc, kbar,
                                       static_cast<char *>(o) + l * lbytes, idx, w, ds, st);
            return r;
        });
    return cuda_status(e);
}

hsa_status_t hsa_decode(const hsa_shape_t *shape, const void *q, const void *q_slc,
                        const void *k_cache, const void *v_cache, const float *kbar, void *o,
                        int32_t *idx, float *w, void *ws, size_t ws_bytes, void *stream) {
    return hsa_decode_multi(shape, 1, q, q_slc, k_cache, v_cache, kbar, o, idx, w, ws, ws_bytes, stream);
}

hsa_status_t hsa_bwd(const hsa_shape_t *shape, const void *q, const void *k, const void *v,
                     const void *q_slc, const void *dO, const float *lse, const int32_t *idx,
                     const float *w, const float *kbar, void *dq, void *dk, void *dv,
                     void *dq_slc, void *ws, size_t ws_bytes, void *stream) {
    hsa_status_t s = check_shape(shape, false);
    if (s != HSA_OK) return s;
    const Shape sh = make_shape(*shape);
    if ((int64_t)sh.B * sh.L == 0) return empty_call(sh, HSA_OP_BWD, ws, ws_bytes, static_cast<cudaStream_t>(stream));
    if (!ptrs_ok({q, k, v, q_slc, dO, lse, idx, w, dq, dk, dv, dq_slc})) return HSA_ERR_INVALID_ARG;
    if (sh.nc > 0 && !ptrs_ok({kbar})) return HSA_ERR_INVALID_ARG;
    if ((s = check_ws(sh, HSA_OP_BWD, ws, ws_bytes)) != HSA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    DevStatus *ds = static_cast<DevStatus *>(ws);
    BwdAll all = carve_bwd(sh, ws, nullptr);
    BwdWs &b = all.b;
    cudaError_t e = clear_status(ws, st);
    const size_t acc_bytes = sizeof(float) * (size_t)sh.B * sh.hkv * sh.L * sh.d;
    if (e == cudaSuccess && sh.nc > 0)
        e = cudaMemsetAsync(b.dkbar, 0, sizeof(float) * (size_t)sh.B * sh.hkv * sh.nc * sh.d, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(b.dk_acc, 0, acc_bytes, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(b.dv_acc, 0, acc_bytes, st);
    if (all.tc) {
        // one chunk-major pass on the tensor cores (dq, dw, dk, dv), then the
        // stick-breaking backward and the finishing pass on CUDA cores
        const AttendPlan &P = all.plan;
        if (e == cudaSuccess) e = timed(HSA_K_INVERT, 4, st, [&] { return launch_invert(sh, idx, w, b, ds, st); });
        if (e == cudaSuccess) e = timed(HSA_K_PLAN, 3, st, [&] { return launch_plan(sh, b, P, st); });
        if (e == cudaSuccess) e = cudaMemsetAsync(P.counters, 0, sizeof(int32_t) * plan_counter_count(P.J), st);
        if (e == cudaSuccess)
            e = cudaMemsetAsync(all.acc, 0,
                                sizeof(__half) * std::min<size_t>(attend_acc_elems(P.W, sh.G, sh.d),
                                                                 (size_t)P.J * P.W * sh.G * sh.d),
                                st);
        if (e == cudaSuccess)  // magnitude bounds for the dq accumulators' power-of-two scale
            e = timed(HSA_K_PLAN, 3, st, [&] {
                int32_t *mb = P.counters + 3 * P.J + 1;
                cudaError_t e2 = launch_rownorm_max(v, (int64_t)sh.B * sh.hkv * sh.L, sh.d, mb, st);
                if (e2 == cudaSuccess) e2 = launch_rownorm_max(dO, (int64_t)sh.B * sh.L * sh.hq, sh.d, mb + 1, st);
                if (e2 == cudaSuccess) e2 = launch_vmax(sh, k, mb + 2, st);
                return e2;
            });
        if (e == cudaSuccess)
            e = timed(HSA_K_BWD_TC, 1, st, [&] {
                return launch_bwd_tc(sh, P, b, q, k, v, dO, lse, all.dw, all.acc, dq, b.dk_acc, b.dv_acc, ds, st);
            });
        if (e == cudaSuccess)
            e = timed(HSA_K_BWD_SEL, 3, st, [&] {
                cudaError_t e2 = launch_bwd_select(sh, q_slc, idx, w, all.dw, kbar, dq_slc, b.dkbar, b, st);
                return e2 == cudaSuccess ? launch_bwd_finish(sh, b, dk, dv, st) : e2;
            });
        return cuda_status(e);
    }
    if (e == cudaSuccess)
        e = timed(HSA_K_BWD1, 1, st, [&] {
            return launch_bwd_phase1(sh, q, q_slc, k, v, dO, lse, idx, w, kbar, dq, dq_slc, b, ds, st);
        });
    if (e == cudaSuccess) e = timed(HSA_K_INVERT, sh.nc > 0 ? 4 : 0, st, [&] { return launch_invert(sh, idx, nullptr, b, ds, st); });
    if (e == cudaSuccess)
        e = timed(HSA_K_BWD2, sh.nc > 0 ? 2 : 1, st, [&] { return launch_bwd_phase2(sh, q, k, v, dO, lse, w, dk, dv, b, ds, st); });
    return cuda_status(e);
}

hsa_status_t hsa_set_wait_limit_ns(uint64_t ns) {
    g_wait_ns.store(ns, std::memory_order_relaxed);
    return HSA_OK;
}

hsa_status_t hsa_device_status(const void *ws, int32_t *code_out, void *stream) {
    if (!ws || !code_out) return HSA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    DevStatus h;
    cudaError_t e = cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return HSA_ERR_CUDA;
    *code_out = h.code;
    return HSA_OK;
}

const char *hsa_status_string(int32_t code) {
    switch (code) {
        case HSA_OK: return "ok";
        case HSA_ERR_INVALID_ARG: return "invalid argument";
        case HSA_ERR_UNSUPPORTED: return "unsupported shape";
        case HSA_ERR_WORKSPACE: return "workspace too small";
        case HSA_ERR_CUDA: return "CUDA launch or API error";
        case HSA_ERR_TIMEOUT: return "device wait timed out";
        case HSA_ERR_DEVICE_CHECK: return "device-side input check failed";
        default: return "unknown status";
    }
}

}  // extern "C"
