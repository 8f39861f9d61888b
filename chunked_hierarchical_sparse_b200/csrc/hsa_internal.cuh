// hsa_internal.cuh -- shared device helpers and launcher declarations of the
// HSA CUDA library.  Nothing here is visible through the C ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hsa.h"

namespace hsa {

constexpr int kChunk = 64;     // S of the tensor-core kernels (the pages' chunk size)
constexpr int kMaxS = 128;     // chunk sizes 16, 32, 64 and 128 run on the CUDA-core kernels
constexpr int kMaxK = 16;      // top-K bound
constexpr int kMaxG = 16;      // query heads per KV group bound
constexpr size_t kWsHeader = 256;

// ---------------------------------------------------------------- status word
// The first bytes of every workspace: code (first error wins) and details.
struct DevStatus {
    int32_t code;
    int32_t where;  // kernel id that reported
    int32_t a, b;   // details (e.g. the offending index)
};

enum KernelId : int32_t {
    kKPool = 1, kKSelect = 2, kKAttendSimt = 3, kKDecode = 4, kKBwd1 = 5, kKInvert = 6,
    kKBwd2 = 7, kKAttendTc = 8, kKFinal = 9, kKSelectTc = 10, kKBwdTc = 11
};

__device__ __forceinline__ void report(DevStatus *st, int32_t code, int32_t where, int32_t a,
                                       int32_t b) {
    if (atomicCAS(&st->code, 0, code) == 0) {
        st->where = where;
        st->a = a;
        st->b = b;
    }
}

// ---------------------------------------------------------------- element access
template <typename T> struct Elem;
template <> struct Elem<float> {
    __device__ __forceinline__ static float load(const float *p) { return *p; }
    __device__ __forceinline__ static void store(float *p, float v) { *p = v; }
};
template <> struct Elem<__nv_bfloat16> {
    __device__ __forceinline__ static float load(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
    __device__ __forceinline__ static void store(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }
};

__host__ __device__ constexpr inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ constexpr inline int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

// ---------------------------------------------------------------- shapes
struct Shape {
    int B, L, hq, hkv, d, S, K, G, nc;
    bool bf16;
};

inline Shape make_shape(const hsa_shape_t &s) {
    Shape r;
    r.B = s.B; r.L = s.L; r.hq = s.h_q; r.hkv = s.h_kv; r.d = s.d; r.S = s.S; r.K = s.K;
    r.G = s.h_kv > 0 ? s.h_q / s.h_kv : 0;
    r.nc = s.S > 0 ? s.L / s.S : 0;
    r.bf16 = s.dtype == HSA_BF16;
    return r;
}

// Host-side validation of a problem shape shared by every entry point: INVALID_ARG
// for inconsistent values, UNSUPPORTED for valid shapes that are not built.
hsa_status_t check_shape(const hsa_shape_t *s, bool decode);

// Bound on one wait inside the persistent kernels (attention, selection, backward), in
// nanoseconds of wall-clock time: 2 s unless hsa_set_wait_limit_ns changed it (a
// testing aid for the failure path).  Passed to the kernels as an argument; the waits
// that let a CTA's own copies and MMAs finish before it exits keep kDrainWaitNs.
uint64_t wait_limit_ns();
constexpr uint64_t kDefaultWaitNs = 2000000000ull;
constexpr uint64_t kDrainWaitNs = 2000000000ull;

// ---------------------------------------------------------------- launch helpers
// Raise a kernel's dynamic shared-memory limit to `bytes` once (cached per
// kernel, so repeated calls -- and calls during stream capture -- make no
// runtime API call once the limit has been set).
cudaError_t set_smem_once(const void *func, size_t bytes);

// ---------------------------------------------------------------- timing
// RAII bracket: records a CUDA event pair around the launches made in its
// scope when hsa_timing_enable(1) is in force (see timing.cu).
class TimedLaunch {
  public:
    TimedLaunch(int kind, int nlaunch, cudaStream_t st);
    ~TimedLaunch();
    TimedLaunch(const TimedLaunch &) = delete;
    TimedLaunch &operator=(const TimedLaunch &) = delete;

  private:
    int kind_, nlaunch_;
    cudaStream_t st_;
    cudaEvent_t a_ = nullptr, b_ = nullptr;
    bool active_ = false;
};

// ---------------------------------------------------------------- launchers
// All launchers enqueue on `st` and return the launch's cudaError_t.
// Optional outputs of the pooling pass (bf16 inputs): the bf16 hi/lo split of the
// pooled keys, and max|v| over the complete chunks of v max-ed into *vmax_bits.
struct PoolExtras {
    __nv_bfloat16 *hi = nullptr, *lo = nullptr;
    const void *v = nullptr;
    int32_t *vmax_bits = nullptr;
};
cudaError_t launch_pool(const Shape &sh, const void *k, float *kbar, DevStatus *ds, cudaStream_t st,
                        const PoolExtras &x = PoolExtras{});

cudaError_t launch_select_simt(const Shape &sh, const void *q_slc, const float *kbar, int32_t *idx,
                               float *w, DevStatus *ds, cudaStream_t st);

cudaError_t launch_attend_simt(const Shape &sh, const void *q, const void *k, const void *v,
                               const int32_t *idx, const float *w, void *o, float *lse,
                               DevStatus *ds, cudaStream_t st);

// Decode: shape.L = P.  idx_out / w_out may point into the workspace.
cudaError_t launch_decode_simt(const Shape &sh, const void *q, const void *q_slc, const void *kc,
                               const void *vc, const float *kbar, void *o, int32_t *idx_out,
                               float *w_out, DevStatus *ds, cudaStream_t st);

// Decode on a thread-block cluster per (b, g) (DSMEM exchange of scores and partials).
// NL layers' queries q [NL,B,h_q,d] share the step's selection and chunk reads; o [NL,B,h_q,d].
bool decode_cluster_supported(const Shape &sh, int NL);
cudaError_t launch_decode_cluster(const Shape &sh, int NL, const void *q, const void *q_slc, const void *kc,
                                  const void *vc, const float *kbar, void *o, int32_t *idx_out, float *w_out,
                                  DevStatus *ds, cudaStream_t st);

// Backward pieces.
struct BwdWs {
    float *dkbar;     // [B,hkv,nc,d] fp32 accumulator (zeroed by the launcher)
    float *delta;     // [B,L,hq,K]  dO . O_k per (token, head, slot)
    float *dk_acc;    // [B,hkv,L,d] fp32 accumulators (zeroed by the launcher)
    float *dv_acc;
    int32_t *hist;    // [B,hkv,ntb,nc] per token-block counts -> offsets
    int32_t *chunk_off;  // [B,hkv,nc+1] CSR offsets into entries (per (b,g) base)
    int32_t *seg_off;    // [B,hkv,nc+1] phase-2 segment offsets (kBwdSeg entries each)
    int32_t *entries;    // [B,hkv, L*K] packed t*16 + slot, sorted by t per chunk
    float *entw;         // [B,hkv, L*K] the entries' stick-breaking weights (forward only, else null)
};

cudaError_t launch_bwd_phase1(const Shape &sh, const void *q, const void *q_slc, const void *k,
                              const void *v, const void *dO, const float *lse, const int32_t *idx,
                              const float *w, const float *kbar, void *dq, void *dq_slc,
                              const BwdWs &ws, DevStatus *ds, cudaStream_t st);

// w (nullable): when given, the entries' weights are gathered into ws.entw.
cudaError_t launch_invert(const Shape &sh, const int32_t *idx, const float *w, const BwdWs &ws, DevStatus *ds,
                          cudaStream_t st);

cudaError_t launch_bwd_phase2(const Shape &sh, const void *q, const void *k, const void *v,
                              const void *dO, const float *lse, const float *w, void *dk, void *dv,
                              const BwdWs &ws, DevStatus *ds, cudaStream_t st);

// tokens per histogram block of the inversion: the scatter walks a block's tokens
// in order (one warp); the histogram holds ceil(L / block) x n_c counts per (b, g)
constexpr int kInvTokBlock = 128;
constexpr int kBwdSeg = 32;        // list entries per phase-2 block

// ---------------------------------------------------------------- chunk-major forward plan
constexpr int kUnitTiles = 4;      // forward: tiles of one chunk per work unit (one K/V load)
constexpr int kCombTokens = 16;    // tokens per combine item
// Accumulators of the chunk-major passes: a ring of kRing window slots, each
// a [W tokens][G heads][d] block of scaled fp16 sums that the tiles of one
// window reduce their weighted outputs (forward) or dq rows (backward) into
// (two 32 MiB slots: the ring stays resident in L2 next to the K/V and query
// working set; smaller slots and a third slot were measured slower at 64K).
constexpr int kRing = 2;
constexpr size_t kAccSlotBudget = size_t(32) << 20;
constexpr int kMaxWindow = 16384;  // tokens per window at most

struct AttendPlan {
    int B, L, hq, hkv, D, K, G, nc, ntb, W, nW, J, TT;
    int unit_tiles;        // tiles per work unit (at most; one K/V load per unit)
    int32_t *unit_prefix;  // [J][nc+1] work units per (window, chunk), exclusive prefix
    int32_t *win_units;    // [J]
    int32_t *win_tiles;    // [J]
    int32_t *win_ncomb;    // [J]
    int32_t *seg_start;    // [J+1] queue segment starts (the units of window s)
    int32_t *counters;     // [3J+4] tiles_done[J], comb_done[J], comb_head[J], a done count, bounds (zeroed per call)
    int4 *items;           // [2 per queue item] descriptors
    int max_items;         // capacity of `items`
    // Layout of the lists and the queue.  win_cap == 0: the queue is contiguous in
    // queue order and each (b, g) owns L*K entries.  win_cap > 0 (the forward's
    // bucket plan): window j's units sit at items[j*win_cap ...], queue position q
    // of window j is seg_start[j] + its unit index, and each window owns W*K
    // entries of its (b, g), ent_stride = nW*W*K entries per (b, g).
    int win_cap;
    int64_t ent_stride;
};

// Forward bucket plan (k_bucket.cu): entries/entw [B*h_kv][nW*W*K], per-block
// chunk histograms hist [bucket_hist_elems(P)]; fills the plan's queue (win_cap
// layout), per-window counts and seg_start.  The plan counters must be zero on entry.
size_t bucket_hist_elems(const AttendPlan &P);
cudaError_t launch_bucket_plan(const Shape &sh, const int32_t *idx, const float *w, const AttendPlan &P,
                               int32_t *hist, int32_t *entries, float *entw, DevStatus *ds, cudaStream_t st);

// tiles_done[J], comb_done[J], comb_head[J], then three words of magnitude bounds as
// float bits: forward max|v|; backward max row norm of v, of dO, and max|k|
inline size_t plan_counter_count(int J) { return 3 * (size_t)J + 4; }

// queue item descriptor (two int4): {type, j, c, e0} {e1, t0, t1, 0}
//   type 0: work unit, chunk c, entries [e0, e1) of its bucket, tiles [t0, t1)
// Combine items are not queued: once every tile of window j is stored, the
// combine warps of all CTAs claim window j's items from comb_head[j].

// window length (tokens) of the chunk-major passes: a multiple of 256 such that
// one window's accumulators (W * G * d elements of `esize` bytes) fit in kAccSlotBudget
inline int attend_window(int G, int d, int esize) {
    const int64_t per_tok = (int64_t)G * d * esize;
    int64_t w = (int64_t)(kAccSlotBudget / per_tok) / kInvTokBlock * kInvTokBlock;
    if (w < kInvTokBlock) w = kInvTokBlock;
    if (w > kMaxWindow) w = kMaxWindow;
    return (int)w;
}

// elements of the accumulator ring of one call
inline size_t attend_acc_elems(int W, int G, int d) { return (size_t)kRing * W * G * d; }

// Both rings hold fp16 sums scaled by a power of two 2^-e at or above a bound of
// every partial sum: the forward's by max|v| (a partial sum of w_k * softmax-
// averages of v), the backward's dq by 2 max||dO_row|| max||v_row|| max|k| / sqrt(d).
constexpr int kFwdAccBytes = 2, kBwdAccBytes = 2;

bool select_tc_supported(const Shape &sh);
// Chunk selection with tensor-core scores; hi/lo: [B,hkv,nc,d] the bf16 split of
// kbar written by the pooling pass.
cudaError_t launch_select_tc(const Shape &sh, const void *q_slc, const float *kbar, __nv_bfloat16 *hi,
                             __nv_bfloat16 *lo, int32_t *idx, float *w, DevStatus *ds, cudaStream_t st);

cudaError_t launch_plan(const Shape &sh, const BwdWs &inv, const AttendPlan &plan, cudaStream_t st);
bool attend_tc_supported(const Shape &sh);
// entries/entw: the bucket plan's lists (plan.ent_stride entries per (b, g))
cudaError_t launch_attend_tc(const Shape &sh, const AttendPlan &plan, const int32_t *entries, const float *entw,
                             const void *q, const void *k, const void *v, __half *acc, void *o, float *lse,
                             DevStatus *ds, cudaStream_t st);
// max|v| over the whole value tensor, as float bits, max-ed into *bits (zeroed by the caller)
cudaError_t launch_vmax(const Shape &sh, const void *v, int32_t *bits, cudaStream_t st);
cudaError_t launch_wsum(const Shape &sh, const int32_t *idx, const float *w, int32_t *bits, cudaStream_t st);

// Chunk-major backward on the tensor cores (d = 128, G in {8, 16}): dq (via the
// plan's window ring `acc`), dw [B,L,hkv,K], and dK / dV added into the fp32
// accumulators of `inv` (dk_acc / dv_acc).  inv.entw must hold the entries' weights.
bool bwd_tc_supported(const Shape &sh);
cudaError_t launch_bwd_tc(const Shape &sh, const AttendPlan &plan, const BwdWs &inv, const void *q, const void *k,
                          const void *v, const void *dO, const float *lse, float *dw, __half *acc, void *dq,
                          float *dk_acc, float *dv_acc, DevStatus *ds, cudaStream_t st);
// max L2 norm over the rows (of d bf16 values) of x, as float bits max-ed into *bits
cudaError_t launch_rownorm_max(const void *x, int64_t rows, int d, int32_t *bits, cudaStream_t st);
// Stick-breaking backward from dw: dq_slc, and dkbar (added into, fp32).
cudaError_t launch_bwd_select(const Shape &sh, const void *q_slc, const int32_t *idx, const float *w, float *dw,
                              const float *kbar, void *dq_slc, float *dkbar, const BwdWs &inv, cudaStream_t st);
// dk = dk_acc + dkbar_c / S, dv = dv_acc, in the input dtype.
cudaError_t launch_bwd_finish(const Shape &sh, const BwdWs &ws, void *dk, void *dv, cudaStream_t st);

}  // namespace hsa
