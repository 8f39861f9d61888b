// k_select_tc.cu -- chunk selection with the score GEMM on the tensor cores.
//
// Cited page: "Hardware-aligned Hierarchical Sparse Attention for Efficient
// Long-term Memory Access" (paper notes), §HSA "Chunk Selection" (each token's
// selection query against every chunk's mean-pooled key, a top-K per query
// group) and §HSA second stage (stick-breaking weights from the scores).
//
// A CTA owns 128 consecutive tokens of one (b, g).  Their selection queries
// (bf16, exact) form the A tile; the fp32 pooled keys are split into two bf16
// terms, kbar = hi + lo with hi = bf16(kbar), lo = bf16(kbar - hi), so
//   q . kbar  ~=  q . hi + q . lo      (two tcgen05 MMAs into one fp32 TMEM tile)
// with a residual of ~2^-16 of |kbar| per element -- far below the score gaps
// that decide the top-K.  Chunk tiles of 64 pooled keys are streamed by TMA
// into two stages; tile i is scored into TMEM buffer i % 2.
//
// Top-K: two epilogue warpgroups, one per TMEM buffer, so group e sees the
// tiles i = e, e + 2, ... in increasing chunk order.  A thread owns one token
// row and keeps a descending list of its group's best chunks in registers.
// Because the chunks reach a group in increasing index order, a new chunk
// beats an equal score already listed (ties go to the higher index), so the
// filter against the current K-th best theta is one compare, x >= theta, and
// a 32-chunk slice whose maximum is below theta is skipped after one warp vote.
// A surviving chunk is inserted at its position (a popcount of parallel
// compares) with a predicated shift.  At the end group 1 hands its list to
// group 0 through shared memory, group 0 merges it (full score-then-index
// order), lists the K chunks most-recent-first and forms the stick-breaking
// weights.
#include <math_constants.h>

#include <algorithm>

#include "hsa_internal.cuh"
#include "sm100.cuh"

namespace hsa {

using namespace sm100;

namespace {

constexpr int kSelThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2-5 and 6-9 the two epilogue groups
constexpr int kSelN = 64;         // chunks per tile (two CTAs fit per SM)
constexpr uint64_t kSelWaitNs = 2000000000ull;

template <int D> struct SelSmem {
    static constexpr int NH = D / 64;
    static constexpr int QBYTES = NH * 128 * 128;     // 128 tokens x D bf16
    static constexpr int BHALF = kSelN * 128;         // kSelN chunks x 64 bf16
    static constexpr int BBYTES = 2 * NH * BHALF;     // hi + lo
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_B = OFF_Q + QBYTES;      // 2 stages; group 1's lists after the last tile
    static constexpr int OFF_BAR = OFF_B + 2 * BBYTES;
    static constexpr int BYTES = OFF_BAR + 16 * 8 + 64;
    static constexpr int ALLOC = BYTES + 1024;
};
static_assert(2 * SelSmem<64>::BBYTES >= 128 * 16 * 8, "group lists do not fit in the tile stages");

// The sorted list: KM (score, chunk) slots, best first.  The first KM - K slots
// hold +inf sentinels that nothing displaces, so slot KM - 1 is always the
// K-th best (a fixed register, no dynamic indexing).
template <int KM> struct TopList {
    float s[KM];
    int c[KM];

    __device__ __forceinline__ void init(int K) {
#pragma unroll
        for (int i = 0; i < KM; ++i) {
            const bool sent = i < KM - K;
            s[i] = sent ? CUDART_INF_F : -CUDART_INF_F;
            c[i] = sent ? 0x7fffffff : -1;
        }
    }
    __device__ __forceinline__ float theta() const { return s[KM - 1]; }

    // place (x, cx) at slot p, shifting slots p.. down by one (the last falls off)
    __device__ __forceinline__ void put(int p, float x, int cx) {
#pragma unroll
        for (int k = KM - 1; k >= 1; --k) {
            const bool sh = k > p, eq = k == p;
            s[k] = sh ? s[k - 1] : (eq ? x : s[k]);
            c[k] = sh ? c[k - 1] : (eq ? cx : c[k]);
        }
        s[0] = (p == 0) ? x : s[0];
        c[0] = (p == 0) ? cx : c[0];
    }
    // a chunk with a higher index than every listed one, x >= theta()
    __device__ __forceinline__ void insert_newest(float x, int cx) {
        int p = 0;
#pragma unroll
        for (int k = 0; k < KM; ++k) p += s[k] > x ? 1 : 0;
        put(p, x, cx);
    }
    // any chunk: score first, then the higher index
    __device__ __forceinline__ void insert_any(float x, int cx) {
        if (!(x > s[KM - 1] || (x == s[KM - 1] && cx > c[KM - 1]))) return;
        int p = 0;
#pragma unroll
        for (int k = 0; k < KM; ++k) p += (s[k] > x || (s[k] == x && c[k] > cx)) ? 1 : 0;
        put(p, x, cx);
    }
};

// v[e] for a lane-varying e in [0, 32), by a select tree on e's bits (stays in registers)
__device__ __forceinline__ float pick32(const float (&v)[32], int e) {
    float t16[16], t8[8], t4[4];
#pragma unroll
    for (int i = 0; i < 16; ++i) t16[i] = (e & 1) ? v[2 * i + 1] : v[2 * i];
#pragma unroll
    for (int i = 0; i < 8; ++i) t8[i] = (e & 2) ? t16[2 * i + 1] : t16[2 * i];
#pragma unroll
    for (int i = 0; i < 4; ++i) t4[i] = (e & 4) ? t8[2 * i + 1] : t8[2 * i];
    const float t2a = (e & 8) ? t4[1] : t4[0], t2b = (e & 8) ? t4[3] : t4[2];
    return (e & 16) ? t2b : t2a;
}

// one 32-chunk slice [c0, c0 + 32) of this row's raw scores v (chunks < ne eligible)
template <int KM>
__device__ __forceinline__ void scan_slice(TopList<KM> &tl, const float (&v)[32], int c0, int ne) {
    float m8[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m8[i] = fmaxf(fmaxf(v[4 * i], v[4 * i + 1]), fmaxf(v[4 * i + 2], v[4 * i + 3]));
    const float vmax = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
    const bool any = c0 < ne && vmax >= tl.theta();
    if (!__any_sync(0xffffffffu, any)) return;
    uint32_t m = 0;
    if (any) {
        const float th = tl.theta();
        const int nel = ne - c0;  // eligible chunks in the slice (may exceed 32)
#pragma unroll
        for (int e = 0; e < 32; ++e) m |= (v[e] >= th && e < nel) ? (1u << e) : 0u;
    }
    while (m) {
        const int e = __ffs(m) - 1;
        m &= m - 1;
        const float x = pick32(v, e);
        if (x >= tl.theta()) tl.insert_newest(x, c0 + e);
    }
}

}  // namespace

template <int D, int KM>
__global__ void __launch_bounds__(kSelThreads, KM <= 8 ? 2 : 1) select_tc_kernel(
    const __grid_constant__ CUtensorMap tm_qs, const __grid_constant__ CUtensorMap tm_hi,
    const __grid_constant__ CUtensorMap tm_lo, int32_t *__restrict__ idx, float *__restrict__ wout,
    int L, int hkv, int nc, int K, DevStatus *ds) {
    using SL = SelSmem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + SL::OFF_BAR);
    uint64_t *q_full = bar;
    uint64_t *b_full = bar + 1;     // [2]
    uint64_t *b_empty = bar + 3;    // [2]
    uint64_t *a_full = bar + 5;     // [2]  TMEM buffer e scored (MMA -> group e)
    uint64_t *a_empty = bar + 7;    // [2]  TMEM buffer e read (group e -> MMA)
    uint64_t *mma_done = bar + 9;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + SL::OFF_BAR + 16 * 8);
    volatile int *fail = reinterpret_cast<volatile int *>(sm + SL::OFF_BAR + 16 * 8 + 16);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // token blocks late in the sequence score the most chunks: they are issued first
    const int nbg = gridDim.x / ((L + 127) / 128);
    const int bg = blockIdx.x % nbg, b = bg / hkv, g = bg % hkv;
    const int t0 = ((L + 127) / 128 - 1 - (int)blockIdx.x / nbg) * 128;
    const int tlast = min(t0 + 128, L) - 1;
    const int ne_max = min(tlast / kChunk, nc);
    const int ntiles = (ne_max + kSelN - 1) / kSelN;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&b_full[i], 1); mbar_init(&b_empty[i], 1);
            mbar_init(&a_full[i], 1); mbar_init(&a_empty[i], 4);
        }
        mbar_init(mma_done, 1);
        *fail = 0;
        mbar_fence_init();
    }
    if (warp == 1) { tmem_alloc(tmem_slot, 2 * kSelN); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // every lane waits (converged, sleeping in try_wait); the warp's verdict is a vote
    auto warp_wait = [&](uint64_t *bb, uint32_t par) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bb, par, kSelWaitNs));
    };

    if (warp == 0) {
        // -------------------------------------------------- TMA producer
        bool ok = true;
        if (ntiles > 0 && lane == 0) {
            mbar_arrive_expect_tx(q_full, SL::QBYTES);
#pragma unroll
            for (int h = 0; h < SL::NH; ++h)
                tma_load_3d(sm + SL::OFF_Q + h * 128 * 128, &tm_qs, h * 64, g, b * L + t0, q_full);
        }
        for (int i = 0; i < ntiles && ok; ++i) {
            const int s = i & 1;
            if (i >= 2 && !warp_wait(&b_empty[s], ((i >> 1) - 1) & 1)) { ok = false; break; }
            if (lane == 0) {
                mbar_arrive_expect_tx(&b_full[s], SL::BBYTES);
                const int row = bg * nc + i * kSelN;
                uint8_t *dst = sm + SL::OFF_B + s * SL::BBYTES;
#pragma unroll
                for (int h = 0; h < SL::NH; ++h) {
                    tma_load_2d(dst + h * SL::BHALF, &tm_hi, h * 64, row, &b_full[s]);
                    tma_load_2d(dst + (SL::NH + h) * SL::BHALF, &tm_lo, h * 64, row, &b_full[s]);
                }
            }
            __syncwarp();
        }
        if (!ok && lane == 0) {
            *fail = 1;
            report(ds, HSA_ERR_TIMEOUT, kKSelectTc, 1, t0);
            // let the loads already issued land before the CTA can go away (bounded)
            for (int i = max(0, ntiles - 2); i < ntiles; ++i) mbar_wait(&b_full[i & 1], (i >> 1) & 1, kSelWaitNs);
        }
    } else if (warp == 1) {
        // -------------------------------------------------- MMA issuer
        constexpr uint32_t idesc = idesc_bf16_f32(128, kSelN, false, false);
        bool ok = true;
        if (ntiles > 0 && !warp_wait(q_full, 0)) ok = false;
        for (int i = 0; i < ntiles && ok; ++i) {
            const int s = i & 1;
            if (!warp_wait(&b_full[s], (i >> 1) & 1)) { ok = false; break; }
            if (i >= 2 && !warp_wait(&a_empty[s], ((i >> 1) - 1) & 1)) { ok = false; break; }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t qa = smem_u32(sm + SL::OFF_Q);
                const uint32_t bb = smem_u32(sm + SL::OFF_B + s * SL::BBYTES);
                const uint32_t dcol = tmem + s * kSelN;
#pragma unroll
                for (int part = 0; part < 2; ++part)  // hi then lo
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const int h = ks >> 2, kk = ks & 3;
                        mma_bf16_ss(dcol, smem_desc_sw128(qa + h * 128 * 128 + kk * 32, 16, 1024),
                                    smem_desc_sw128(bb + (part * SL::NH + h) * SL::BHALF + kk * 32, 16, 1024), idesc,
                                    (part | ks) != 0);
                    }
                mma_commit(&a_full[s]);
                mma_commit(&b_empty[s]);
            }
            __syncwarp();
        }
        if (!ok && lane == 0) { *fail = 1; report(ds, HSA_ERR_TIMEOUT, kKSelectTc, 2, t0); }
        if (lane == 0) { mma_commit(mma_done); mbar_wait(mma_done, 0, kSelWaitNs); }
        __syncwarp();
    } else {
        // -------------------------------------------------- two epilogue groups, one token row per thread
        const int eg = (warp - 2) >> 2;   // group = TMEM buffer = tile parity
        const int wq = warp & 3;          // TMEM lane quadrant of this warp
        const int r = wq * 32 + lane;
        const int t = t0 + r;
        const int ne = (t < L) ? min(t / kChunk, nc) : 0;
        const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16) + eg * kSelN;
        TopList<KM> tl;
        tl.init(K);
        bool ok = true;
        for (int i = eg; i < ntiles; i += 2) {
            if (!warp_wait(&a_full[eg], (i >> 1) & 1)) { ok = false; break; }
            tc_fence_after();
            float v0[32], v1[32];
            tmem_ld32(lane_base, v0);
            tmem_ld32(lane_base + 32, v1);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            mbar_arrive_lane0(&a_empty[eg], lane);  // the buffer is free for tile i + 2
            scan_slice(tl, v0, i * kSelN, ne);
            scan_slice(tl, v1, i * kSelN + 32, ne);
        }
        if (!ok) { *fail = 1; if (lane == 0) report(ds, HSA_ERR_TIMEOUT, kKSelectTc, 3, t0); }
        // group 1 hands its list over in the tile stages, once the MMA warp's final
        // commit shows that every MMA (and so every tile load) has completed
        float *ls = reinterpret_cast<float *>(sm + SL::OFF_B);
        int *lc = reinterpret_cast<int *>(sm + SL::OFF_B) + 128 * KM;
        if (eg == 1) {
            if (!warp_wait(mma_done, 0)) { *fail = 1; if (lane == 0) report(ds, HSA_ERR_TIMEOUT, kKSelectTc, 4, t0); }
#pragma unroll
            for (int k = 0; k < KM; ++k) { ls[k * 128 + r] = tl.s[k]; lc[k * 128 + r] = tl.c[k]; }
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (eg == 0 && !*fail && t < L) {
#pragma unroll
            for (int k = 0; k < KM; ++k) {
                const int c1 = lc[k * 128 + r];
                if (c1 >= 0 && c1 != 0x7fffffff) tl.insert_any(ls[k * 128 + r], c1);
            }
            // most-recent-first: order the chosen chunks by descending index (empty = -1 last)
#pragma unroll
            for (int k = 0; k < KM; ++k)
                if (k < KM - K) { tl.c[k] = -1; tl.s[k] = 0.f; }  // sentinels
#pragma unroll
            for (int a = 0; a < KM; ++a)
#pragma unroll
                for (int k = 0; k + 1 < KM - a; ++k) {
                    const bool sw = tl.c[k] < tl.c[k + 1];
                    const float s0 = tl.s[k], s1 = tl.s[k + 1];
                    const int i0 = tl.c[k], i1 = tl.c[k + 1];
                    tl.s[k] = sw ? s1 : s0; tl.s[k + 1] = sw ? s0 : s1;
                    tl.c[k] = sw ? i1 : i0; tl.c[k + 1] = sw ? i0 : i1;
                }
            const float scale = 1.0f / sqrtf((float)D);
            float keep = 1.f;
            const int64_t o = (((int64_t)b * L + t) * hkv + g) * K;
#pragma unroll
            for (int k = 0; k < KM; ++k) {
                if (k < K) {
                    if (tl.c[k] >= 0) {
                        const float sg = 1.0f / (1.0f + expf(-tl.s[k] * scale));
                        idx[o + k] = tl.c[k];
                        wout[o + k] = sg * keep;
                        keep *= (1.f - sg);
                    } else {
                        idx[o + k] = -1;
                        wout[o + k] = 0.f;
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 2 * kSelN);
}

namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn sel_encode() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}
bool map_bf16(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims, const cuuint64_t *strides,
              const cuuint32_t *box) {
    EncodeTiledFn enc = sel_encode();
    if (!enc) return false;
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_sel(const Shape &sh, const void *q_slc, const float *kbar, __nv_bfloat16 *hi,
                       __nv_bfloat16 *lo, int32_t *idx, float *w, DevStatus *ds, cudaStream_t st) {
    CUtensorMap mq, mh, ml;
    // q_slc [B*L, h_kv, d] viewed 3D: (d, h_kv, B*L); box (64, 1, 128 tokens)
    const cuuint64_t qd[3] = {(cuuint64_t)D, (cuuint64_t)sh.hkv, (cuuint64_t)sh.B * sh.L};
    const cuuint64_t qsd[2] = {(cuuint64_t)D * 2, (cuuint64_t)sh.hkv * D * 2};
    const cuuint32_t qb[3] = {64, 1, 128};
    const cuuint64_t kd[2] = {(cuuint64_t)D, (cuuint64_t)std::max<int64_t>(1, (int64_t)sh.B * sh.hkv * sh.nc)};
    const cuuint64_t ksd[1] = {(cuuint64_t)D * 2};
    const cuuint32_t kb[2] = {64, kSelN};
    if (!map_bf16(&mq, q_slc, 3, qd, qsd, qb) || !map_bf16(&mh, hi, 2, kd, ksd, kb) ||
        !map_bf16(&ml, lo, 2, kd, ksd, kb))
        return cudaErrorInvalidValue;
    const size_t smem = SelSmem<D>::ALLOC;
    const unsigned grid = (unsigned)(ceil_div(sh.L, 128) * sh.B * sh.hkv);  // 1D: (token block desc, b*hkv + g)
    cudaError_t e;
    if (sh.K <= 8) {
        if ((e = set_smem_once((const void *)select_tc_kernel<D, 8>, smem)) != cudaSuccess) return e;
        select_tc_kernel<D, 8><<<grid, kSelThreads, smem, st>>>(mq, mh, ml, idx, w, sh.L, sh.hkv, sh.nc, sh.K, ds);
    } else {
        if ((e = set_smem_once((const void *)select_tc_kernel<D, 16>, smem)) != cudaSuccess) return e;
        select_tc_kernel<D, 16><<<grid, kSelThreads, smem, st>>>(mq, mh, ml, idx, w, sh.L, sh.hkv, sh.nc, sh.K, ds);
    }
    return cudaGetLastError();
}
}  // namespace

bool select_tc_supported(const Shape &sh) {
    return sh.bf16 && (sh.d == 64 || sh.d == 128) && sel_encode() != nullptr;
}

cudaError_t launch_select_tc(const Shape &sh, const void *q_slc, const float *kbar, __nv_bfloat16 *hi,
                             __nv_bfloat16 *lo, int32_t *idx, float *w, DevStatus *ds, cudaStream_t st) {
    if (sh.B == 0 || sh.L == 0) return cudaSuccess;
    if (sh.d == 128) return launch_sel<128>(sh, q_slc, kbar, hi, lo, idx, w, ds, st);
    return launch_sel<64>(sh, q_slc, kbar, hi, lo, idx, w, ds, st);
}

}  // namespace hsa
