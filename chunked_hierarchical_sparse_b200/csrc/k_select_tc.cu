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
// that decide the top-K.  Chunk tiles of 128 pooled keys are streamed by TMA;
// each epilogue thread owns one token row, reads its 128 scores from TMEM and
// keeps a sorted top-K (16 register slots) updated only when a score beats
// its current K-th best.  Afterwards the K chunks are put most-recent-first
// and the stick-breaking weights are formed.
#include <math_constants.h>

#include <algorithm>

#include "hsa_internal.cuh"
#include "sm100.cuh"

namespace hsa {

using namespace sm100;


namespace {

constexpr int kSelThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kSelN = 64;         // chunks per tile (two CTAs fit per SM)
constexpr uint64_t kSelWaitNs = 2000000000ull;

template <int D> struct SelSmem {
    static constexpr int NH = D / 64;
    static constexpr int QBYTES = NH * 128 * 128;     // 128 tokens x D bf16
    static constexpr int BHALF = kSelN * 128;         // kSelN chunks x 64 bf16
    static constexpr int BBYTES = 2 * NH * BHALF;     // hi + lo
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_B = OFF_Q + QBYTES;      // 2 stages
    static constexpr int OFF_BAR = OFF_B + 2 * BBYTES;
    static constexpr int BYTES = OFF_BAR + 16 * 8 + 64;
    static constexpr int ALLOC = BYTES + 1024;
};

__device__ __forceinline__ bool sel_beats(float s1, int c1, float s2, int c2) {
    return s1 > s2 || (s1 == s2 && c1 > c2);
}

}  // namespace

// kbar fp32 -> (hi, lo) bf16
__global__ void kbar_split_kernel(const float *__restrict__ kbar, __nv_bfloat16 *__restrict__ hi,
                                  __nv_bfloat16 *__restrict__ lo, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float x = kbar[i];
        const __nv_bfloat16 h = __float2bfloat16_rn(x);
        hi[i] = h;
        lo[i] = __float2bfloat16_rn(x - __bfloat162float(h));
    }
}

template <int D, int KM>
__global__ void __launch_bounds__(kSelThreads, 2) select_tc_kernel(
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
    uint64_t *a_full = bar + 5;     // [2]
    uint64_t *a_empty = bar + 7;    // [2]
    uint64_t *mma_done = bar + 9;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + SL::OFF_BAR + 16 * 8);
    volatile int *wg_flag = reinterpret_cast<volatile int *>(sm + SL::OFF_BAR + 16 * 8 + 16);

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
        mbar_fence_init();
    }
    if (warp == 1) { tmem_alloc(tmem_slot, 2 * kSelN); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto warp_wait = [&](uint64_t *bb, uint32_t par) -> bool {
        int r = 1;
        if (lane == 0) r = mbar_wait(bb, par, kSelWaitNs) ? 1 : 0;
        return __shfl_sync(0xffffffffu, r, 0) != 0;
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
        if (!ok && lane == 0) report(ds, HSA_ERR_TIMEOUT, kKSelectTc, 1, t0);
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
        if (!ok && lane == 0) report(ds, HSA_ERR_TIMEOUT, kKSelectTc, 2, t0);
        if (lane == 0) { mma_commit(mma_done); mbar_wait(mma_done, 0, kSelWaitNs); }
        __syncwarp();
    } else {
        // -------------------------------------------------- epilogue: one token row per thread
        const int wq = warp & 3;
        const int r = wq * 32 + lane;
        const int tid = threadIdx.x - 64;
        const int t = t0 + r;
        const int ne = (t < L) ? min(t / kChunk, nc) : 0;
        const float scale = 1.0f / sqrtf((float)D);
        const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
        // Sorted best-first slots (KM >= K).  The first KM-K slots hold +inf sentinels
        // that nothing displaces, so the last slot is always the K-th best (a
        // fixed register, no dynamic indexing).
        float bs[KM];
        int bc[KM];
#pragma unroll
        for (int i = 0; i < KM; ++i) {
            const bool sent = i < KM - K;
            bs[i] = sent ? CUDART_INF_F : -CUDART_INF_F;
            bc[i] = sent ? 0x7fffffff : -1;
        }
        int wcnt = 0;
        bool ok = true;
        for (int i = 0; i < ntiles; ++i) {
            const int s = i & 1;
            int v = 1;
            if (tid == 0) v = mbar_wait(&a_full[s], (i >> 1) & 1, kSelWaitNs) ? 1 : 0;
            const int slot = (wcnt++) & 1;
            if (tid == 0) wg_flag[slot] = v;
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (!wg_flag[slot]) { ok = false; break; }
            tc_fence_after();
            const int cbase = i * kSelN;
            for (int q4 = 0; q4 < kSelN / 32; ++q4) {
                float sc[32];
                tmem_ld32(lane_base + s * kSelN + q4 * 32, sc);
                tmem_wait_ld();
                const int c0 = cbase + q4 * 32;
                if (c0 == 0) {
                    // the first 32 chunks: nearly all of them enter the (still filling)
                    // list, so take them in order, without extracting each one
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const float x = sc[e] * scale;
                        if (e < ne && sel_beats(x, e, bs[KM - 1], bc[KM - 1])) {
                            float cs = x;
                            int cc = e;
#pragma unroll
                            for (int k = 0; k < KM; ++k) {
                                const bool sw = sel_beats(cs, cc, bs[k], bc[k]);
                                const float ts = bs[k];
                                const int tc = bc[k];
                                bs[k] = sw ? cs : ts;
                                bc[k] = sw ? cc : tc;
                                cs = sw ? ts : cs;
                                cc = sw ? tc : cc;
                            }
                        }
                    }
                    continue;
                }
                // cheap pass: which of the 32 candidates beat the current K-th best?
                uint32_t m = 0;
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    sc[e] *= scale;
                    if (c0 + e < ne && sel_beats(sc[e], c0 + e, bs[KM - 1], bc[KM - 1])) m |= 1u << e;
                }
                // rare pass: insert them one by one (candidate picked by a select tree on
                // the bits of its position, so everything stays in registers)
                while (m) {
                    const int e = __ffs(m) - 1;
                    m &= m - 1;
                    float t16[16], t8[8], t4[4], t2[2];
#pragma unroll
                    for (int i = 0; i < 16; ++i) t16[i] = (e & 1) ? sc[2 * i + 1] : sc[2 * i];
#pragma unroll
                    for (int i = 0; i < 8; ++i) t8[i] = (e & 2) ? t16[2 * i + 1] : t16[2 * i];
#pragma unroll
                    for (int i = 0; i < 4; ++i) t4[i] = (e & 4) ? t8[2 * i + 1] : t8[2 * i];
#pragma unroll
                    for (int i = 0; i < 2; ++i) t2[i] = (e & 8) ? t4[2 * i + 1] : t4[2 * i];
                    const float x = (e & 16) ? t2[1] : t2[0];
                    const int c = c0 + e;
                    if (!sel_beats(x, c, bs[KM - 1], bc[KM - 1])) continue;
                    float cs = x;
                    int cc = c;
#pragma unroll
                    for (int k = 0; k < KM; ++k) {
                        const bool sw = sel_beats(cs, cc, bs[k], bc[k]);
                        const float ts = bs[k];
                        const int tc = bc[k];
                        bs[k] = sw ? cs : ts;
                        bc[k] = sw ? cc : tc;
                        cs = sw ? ts : cs;
                        cc = sw ? tc : cc;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_empty[s]);
        }
        if (!ok && tid == 0) report(ds, HSA_ERR_TIMEOUT, kKSelectTc, 3, t0);
        if (t < L) {
            // most-recent-first: order the chosen chunks by descending index (invalid = -1 last)
#pragma unroll
            for (int k = 0; k < KM; ++k)
                if (k < KM - K) { bc[k] = -1; bs[k] = 0.f; }  // sentinels
#pragma unroll
            for (int a = 0; a < KM; ++a)
#pragma unroll
                for (int k = 0; k + 1 < KM - a; ++k) {
                    const bool sw = bc[k] < bc[k + 1];
                    const float s0 = bs[k], s1 = bs[k + 1];
                    const int i0 = bc[k], i1 = bc[k + 1];
                    bs[k] = sw ? s1 : s0; bs[k + 1] = sw ? s0 : s1;
                    bc[k] = sw ? i1 : i0; bc[k + 1] = sw ? i0 : i1;
                }
            float keep = 1.f;
            const int64_t o = (((int64_t)b * L + t) * hkv + g) * K;
#pragma unroll
            for (int k = 0; k < KM; ++k) {
                if (k < K) {
                    if (bc[k] >= 0) {
                        const float sg = 1.0f / (1.0f + expf(-bs[k]));
                        idx[o + k] = bc[k];
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
    const int64_t n = (int64_t)sh.B * sh.hkv * sh.nc * D;
    if (n > 0) {
        kbar_split_kernel<<<(unsigned)std::min<int64_t>(ceil_div(n, 256), 148 * 8), 256, 0, st>>>(kbar, hi, lo, n);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
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
