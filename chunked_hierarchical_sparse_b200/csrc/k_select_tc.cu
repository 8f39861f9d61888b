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
// into two stages and scored into two TMEM buffers.
//
// Top-K, one token row per epilogue thread, in two passes over the row: the
// tiles are scored twice (the tensor cores have time to spare; the CUDA-core
// work per score is what bounds this kernel).
//   pass 1  the maximum of each of 16 column stripes (chunk index mod 16) over
//           the whole row.  K of the stripes hold a score at least as large as
//           the K-th largest stripe maximum tau, so the row's K-th best is >= tau;
//           for these inputs only ~2% of the scores reach tau;
//   pass 2  the scores >= tau are appended to the row's candidate buffer in
//           shared memory; they arrive in increasing chunk order.
// The buffer is then inserted into a sorted list.  A candidate always has a
// higher index than everything listed, so it beats an equal listed score
// (ties go to the higher index) and the insertion compares scores only.  A
// buffer that fills is inserted early and the threshold raised to the list's
// K-th best.  At the end the K chunks are listed most-recent-first and the
// stick-breaking weights are formed.
#include <float.h>
#include <math_constants.h>

#include <algorithm>

#include "hsa_internal.cuh"
#include "sm100.cuh"

namespace hsa {

using namespace sm100;

namespace {

constexpr int kSelThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue (one TMEM lane quadrant each)
constexpr int kSelN = 64;         // chunks per tile
constexpr int kStripes = 16;      // column stripes of pass 1 (>= K)
constexpr int kCap = 12;          // candidate buffer entries per row

template <int D> struct SelSmem {
    static constexpr int NH = D / 64;
    static constexpr int QBYTES = NH * 128 * 128;     // 128 tokens x D bf16
    static constexpr int BHALF = kSelN * 128;         // kSelN chunks x 64 bf16
    static constexpr int BBYTES = 2 * NH * BHALF;     // hi + lo
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_B = OFF_Q + QBYTES;      // 2 stages
    static constexpr int OFF_CS = OFF_B + 2 * BBYTES; // [kCap][128] candidate scores
    static constexpr int OFF_CC = OFF_CS + kCap * 128 * 4;  // [kCap][128] candidate chunks
    static constexpr int OFF_BAR = OFF_CC + kCap * 128 * 4;
    static constexpr int BYTES = OFF_BAR + 16 * 8 + 64;
    static constexpr int ALLOC = BYTES + 1024;
};
static_assert(2 * (SelSmem<128>::ALLOC + 1024) <= 228 * 1024, "two selection CTAs must fit one SM");

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
    // a chunk with a higher index than every listed one: it beats equal scores.
    // Top-down pass: the element being placed moves down while it beats the slot.
    __device__ __forceinline__ void insert_newest(float x, int cx) {
#pragma unroll
        for (int k = 0; k < KM; ++k) {
            const bool sw = x >= s[k];
            const float ts = s[k];
            const int tc = c[k];
            s[k] = sw ? x : ts;
            c[k] = sw ? cx : tc;
            x = sw ? ts : x;
            cx = sw ? tc : cx;
        }
    }
};

// ascending sort of KS floats (bitonic network, static indices)
template <int KS> __device__ __forceinline__ void sort_asc(float (&a)[KS]) {
#pragma unroll
    for (int k = 2; k <= KS; k <<= 1)
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1)
#pragma unroll
            for (int i = 0; i < KS; ++i) {
                const int l = i ^ j;
                if (l > i) {
                    const bool up = (i & k) == 0;
                    const float lo = fminf(a[i], a[l]), hi = fmaxf(a[i], a[l]);
                    a[i] = up ? lo : hi;
                    a[l] = up ? hi : lo;
                }
            }
}

// v[e] for a lane-varying e in [0, 32), by a select tree on e's bits (stays in registers)
__device__ __forceinline__ float pick32(const float *v, int e) {
    float t16[16], t8[8], t4[4];
#pragma unroll
    for (int i = 0; i < 16; ++i) t16[i] = (e & 1) ? v[2 * i + 1] : v[2 * i];
#pragma unroll
    for (int i = 0; i < 8; ++i) t8[i] = (e & 2) ? t16[2 * i + 1] : t16[2 * i];
#pragma unroll
    for (int i = 0; i < 4; ++i) t4[i] = (e & 4) ? t8[2 * i + 1] : t8[2 * i];
    const float ta = (e & 8) ? t4[1] : t4[0], tb = (e & 8) ? t4[3] : t4[2];
    return (e & 16) ? tb : ta;
}

}  // namespace

template <int D, int KM>
__global__ void __launch_bounds__(kSelThreads, 2) select_tc_kernel(
    const __grid_constant__ CUtensorMap tm_qs, const __grid_constant__ CUtensorMap tm_hi,
    const __grid_constant__ CUtensorMap tm_lo, int32_t *__restrict__ idx, float *__restrict__ wout,
    int L, int hkv, int nc, int K, DevStatus *ds, uint64_t wait_ns) {
    using SL = SelSmem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + SL::OFF_BAR);
    uint64_t *q_full = bar;
    uint64_t *b_full = bar + 1;     // [2]  tile stage loaded (TMA -> MMA)
    uint64_t *b_empty = bar + 3;    // [2]  tile stage read (MMA -> TMA)
    uint64_t *a_full = bar + 5;     // [2]  TMEM buffer holds a scored tile (MMA -> epilogue)
    uint64_t *a_empty = bar + 7;    // [2]  TMEM buffer read (epilogue -> MMA)
    uint64_t *mma_done = bar + 9;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + SL::OFF_BAR + 16 * 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // token blocks late in the sequence score the most chunks: they are issued first
    const int nbg = gridDim.x / ((L + 127) / 128);
    const int bg = blockIdx.x % nbg, b = bg / hkv, g = bg % hkv;
    const int t0 = ((L + 127) / 128 - 1 - (int)blockIdx.x / nbg) * 128;
    const int tlast = min(t0 + 128, L) - 1;
    const int ne_max = min(tlast / kChunk, nc);
    const int ntiles = (ne_max + kSelN - 1) / kSelN;
    const int nsteps = 2 * ntiles;  // every tile scored twice: pass 1, then pass 2

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&b_full[i], 1); mbar_init(&b_empty[i], 1);
            mbar_init(&a_full[i], 1); mbar_init(&a_empty[i], 4);
        }
        mbar_init(mma_done, 1);
        mbar_fence_init();
    }
    if (warp == 1) { tmem_alloc(tmem_slot, 2 * kSelN); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // every lane waits (converged, sleeping in try_wait); the warp decides by a vote
    auto warp_wait = [&](uint64_t *bb, uint32_t par) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bb, par, wait_ns));
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
        int issued = 0;
        for (int i = 0; i < nsteps && ok; ++i) {
            const int s = i & 1;
            if (i >= 2 && !warp_wait(&b_empty[s], ((i >> 1) - 1) & 1)) { ok = false; break; }
            if (lane == 0) {
                mbar_arrive_expect_tx(&b_full[s], SL::BBYTES);
                const int row = bg * nc + (i % ntiles) * kSelN;
                uint8_t *dst = sm + SL::OFF_B + s * SL::BBYTES;
#pragma unroll
                for (int h = 0; h < SL::NH; ++h) {
                    tma_load_2d(dst + h * SL::BHALF, &tm_hi, h * 64, row, &b_full[s]);
                    tma_load_2d(dst + (SL::NH + h) * SL::BHALF, &tm_lo, h * 64, row, &b_full[s]);
                }
            }
            issued = i + 1;
            __syncwarp();
        }
        if (!ok && lane == 0) {
            report(ds, HSA_ERR_TIMEOUT, kKSelectTc, 1, t0);
            // let the loads already issued land before the CTA can go away (bounded)
            for (int i = max(0, issued - 2); i < issued; ++i) mbar_wait(&b_full[i & 1], (i >> 1) & 1, kDrainWaitNs);
        }
    } else if (warp == 1) {
        // -------------------------------------------------- MMA issuer
        constexpr uint32_t idesc = idesc_bf16_f32(128, kSelN, false, false);
        bool ok = true;
        if (ntiles > 0 && !warp_wait(q_full, 0)) ok = false;
        for (int i = 0; i < nsteps && ok; ++i) {
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
        if (!ok && lane == 0) report(ds, HSA_ERR_TIMEOUT, kKSelectTc, 2, t0);
        if (lane == 0) { mma_commit(mma_done); mbar_wait(mma_done, 0, kDrainWaitNs); }
        __syncwarp();
    } else {
        // -------------------------------------------------- epilogue: one token row per thread
        const int wq = warp & 3;          // TMEM lane quadrant of this warp
        const int r = wq * 32 + lane;
        const int t = t0 + r;
        const int ne = (t < L) ? min(t / kChunk, nc) : 0;
        const int ne_warp = __reduce_min_sync(0xffffffffu, (unsigned)ne);  // chunks < ne_warp: eligible in every lane
        float *cs = reinterpret_cast<float *>(sm + SL::OFF_CS) + r;  // candidate i at cs[i * 128]
        int *cc = reinterpret_cast<int *>(sm + SL::OFF_CC) + r;
        TopList<KM> tl;
        tl.init(K);
        int n = 0;  // buffered candidates
        auto flush = [&]() {
            for (int i = 0; i < n; ++i) {
                const float x = cs[i * 128];
                if (x >= tl.theta()) tl.insert_newest(x, cc[i * 128]);
            }
            n = 0;
        };
        float st[kStripes];
#pragma unroll
        for (int j = 0; j < kStripes; ++j) st[j] = -CUDART_INF_F;
        float thr = CUDART_INF_F;
        bool ok = true;
        for (int i = 0; i < nsteps; ++i) {
            const int s = i & 1;
            const int cb = (i % ntiles) * kSelN;
            const bool full = cb + kSelN <= ne_warp;  // every chunk of the tile eligible in every lane
            if (!warp_wait(&a_full[s], (i >> 1) & 1)) { ok = false; break; }
            tc_fence_after();
            float v[64];
            tmem_ld32(tmem + ((uint32_t)(wq * 32) << 16) + s * kSelN, *reinterpret_cast<float(*)[32]>(&v[0]));
            tmem_ld32(tmem + ((uint32_t)(wq * 32) << 16) + s * kSelN + 32, *reinterpret_cast<float(*)[32]>(&v[32]));
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            mbar_arrive_lane0(&a_empty[s], lane);  // the buffer is free for step i + 2
            if (!full) {
#pragma unroll
                for (int e = 0; e < 64; ++e) v[e] = cb + e < ne ? v[e] : -CUDART_INF_F;
            }
            if (i < ntiles) {
                // ---- pass 1: stripe maxima
#pragma unroll
                for (int e = 0; e < 64; ++e) st[e % kStripes] = fmaxf(st[e % kStripes], v[e]);
                if (i == ntiles - 1) {  // tau: the K-th largest stripe maximum = the least of the top K
                    sort_asc<kStripes>(st);
                    thr = CUDART_INF_F;
#pragma unroll
                    for (int j = 0; j < kStripes; ++j) thr = fminf(thr, j >= kStripes - K ? st[j] : CUDART_INF_F);
                    // fewer than K eligible chunks leave tau = -inf: every finite (eligible)
                    // score is a candidate, the masked -inf ones are not
                    thr = fmaxf(thr, -FLT_MAX);
                }
            } else {
                // ---- pass 2: buffer every score >= thr (ineligible ones are -inf)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t m = 0;
#pragma unroll
                    for (int e = 0; e < 32; ++e) m |= (v[hf * 32 + e] >= thr) ? (1u << e) : 0u;
                    if (n + __popc(m) > kCap) {  // rare: insert the buffer, raise the threshold
                        flush();
                        thr = fmaxf(thr, tl.theta());
#pragma unroll
                        for (int e = 0; e < 32; ++e) m &= (v[hf * 32 + e] >= thr) ? 0xffffffffu : ~(1u << e);
                        while (__popc(m) > kCap) {  // still too many: insert directly, lowest chunks first
                            const int e = __ffs(m) - 1;
                            m &= m - 1;
                            const float x = pick32(v + hf * 32, e);
                            if (x >= tl.theta()) tl.insert_newest(x, cb + hf * 32 + e);
                        }
                    }
                    while (m) {
                        const int e = __ffs(m) - 1;
                        m &= m - 1;
                        cs[n * 128] = pick32(v + hf * 32, e);
                        cc[n * 128] = cb + hf * 32 + e;
                        ++n;
                    }
                }
            }
        }
        if (!ok && lane == 0) report(ds, HSA_ERR_TIMEOUT, kKSelectTc, 3, t0);
        if (ok && t < L) {
            flush();
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
        select_tc_kernel<D, 8><<<grid, kSelThreads, smem, st>>>(mq, mh, ml, idx, w, sh.L, sh.hkv, sh.nc, sh.K, ds,
                                                                wait_limit_ns());
    } else {
        if ((e = set_smem_once((const void *)select_tc_kernel<D, 16>, smem)) != cudaSuccess) return e;
        select_tc_kernel<D, 16><<<grid, kSelThreads, smem, st>>>(mq, mh, ml, idx, w, sh.L, sh.hkv, sh.nc, sh.K, ds,
                                                                 wait_limit_ns());
    }
    return cudaGetLastError();
}
}  // namespace

bool select_tc_supported(const Shape &sh) {
    return sh.bf16 && sh.S == kChunk && (sh.d == 64 || sh.d == 128) && sel_encode() != nullptr;
}

cudaError_t launch_select_tc(const Shape &sh, const void *q_slc, const float *kbar, __nv_bfloat16 *hi,
                             __nv_bfloat16 *lo, int32_t *idx, float *w, DevStatus *ds, cudaStream_t st) {
    if (sh.B == 0 || sh.L == 0) return cudaSuccess;
    if (sh.d == 128) return launch_sel<128>(sh, q_slc, kbar, hi, lo, idx, w, ds, st);
    return launch_sel<64>(sh, q_slc, kbar, hi, lo, idx, w, ds, st);
}

}  // namespace hsa
