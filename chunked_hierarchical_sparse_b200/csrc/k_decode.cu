// k_decode.cu -- the decode step on a thread-block cluster per (b, g).
//
// Cited page: "Hardware-aligned Hierarchical Sparse Attention for Efficient
// Long-term Memory Access" (paper notes), §training/inference "KV Cache
// Offloading": at inference only the chunk-level index stays in fast memory;
// each step scores it with the new token's selection query, keeps the top-K
// chunks and reads only those chunks' K/V.  The new token sits at position P,
// so every complete cached chunk is eligible.
//
// One cluster of kDecCta CTAs per (b, g); the whole step is latency-bound, so
// the work is spread over the cluster and exchanged through distributed
// shared memory instead of global memory:
//   1. CTA r scores its slice of the chunk index (coalesced 512 B rows).
//   2. cluster barrier; every CTA reads all scores over DSMEM and keeps the
//      same top-K (warp 0), orders it most-recent-first, forms the
//      stick-breaking weights.
//   3. CTA r attends the group's G query heads to the chunk of slot r (and
//      r + kDecCta, ...), softmax-off-by-one, and scales by w / Z.
//   4. cluster barrier; CTA r sums its share of the output columns over all
//      CTAs' partial outputs (DSMEM) and writes o; a last barrier keeps every
//      CTA's shared memory alive until all remote reads are done.
#include <cooperative_groups.h>
#include <math_constants.h>

#include "hsa_internal.cuh"
#include "topk_warp.cuh"

namespace cg = cooperative_groups;

namespace hsa {

constexpr int kDecCta = 8;
constexpr int kDecThreads = 128;

template <typename T, int D>
__global__ void __cluster_dims__(kDecCta, 1, 1) __launch_bounds__(kDecThreads)
    decode_cluster_kernel(const T *__restrict__ q, const T *__restrict__ q_slc, const T *__restrict__ kc,
                          const T *__restrict__ vc, const float *__restrict__ kbar, T *__restrict__ o,
                          int32_t *__restrict__ idx_out, float *__restrict__ w_out, int P, int hq, int hkv,
                          int nc, int K, int G) {
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int bg = blockIdx.x / kDecCta, b = bg / hkv, g = bg % hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float scale = 1.0f / sqrtf((float)D);

    extern __shared__ float4 dsm4[];
    float *sm = reinterpret_cast<float *>(dsm4);
    const int per = (nc + kDecCta - 1) / kDecCta;     // chunks scored by each CTA
    float *scores = sm;                               // [per]
    float *part = scores + ((per + 3) & ~3);          // [G][D] partial output of this CTA's slots
    float *Qs = part + kMaxG * D;                     // [G][D]
    float *Ks = Qs + kMaxG * D;                       // [64][D+1]
    float *Vs = Ks + kChunk * (D + 1);                // [64][D]
    float *Pm = Vs + kChunk * D;                      // [G][64]
    __shared__ int slot_c[kMaxK];
    __shared__ float slot_w[kMaxK];
    __shared__ float coef[kMaxG];

    // ---- 1. scores of this CTA's chunk slice
    const int c_lo = rank * per, c_hi = min(nc, c_lo + per);
    const float *kb = kbar + (int64_t)bg * nc * D;
    float qv[D / 32];
#pragma unroll
    for (int e = 0; e < D / 32; ++e) qv[e] = Elem<T>::load(q_slc + (int64_t)bg * D + lane + 32 * e);
    for (int c = c_lo + warp; c < c_hi; c += kDecThreads / 32) {
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < D / 32; ++e) acc = fmaf(qv[e], kb[(int64_t)c * D + lane + 32 * e], acc);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) scores[c - c_lo] = acc * scale;
    }
    for (int e = tid; e < G * D; e += kDecThreads)
        Qs[e] = Elem<T>::load(q + ((int64_t)b * hq + (int64_t)g * G) * D + e);
    for (int e = tid; e < kMaxG * D; e += kDecThreads) part[e] = 0.f;
    cluster.sync();

    // ---- 2. top-K over all chunks (every CTA, warp 0), read over DSMEM
    if (warp == 0) {
        float ls = (lane < K) ? -CUDART_INF_F : CUDART_INF_F;
        int lc = (lane < K) ? -1 : 0x7fffffff;
        for (int c0 = 0; c0 < nc; c0 += 64) {
            const int ca = c0 + lane, cb = c0 + lane + 32;
            float sa = 0.f, sb = 0.f;
            if (ca < nc) sa = cluster.map_shared_rank(scores, ca / per)[ca % per];
            if (cb < nc) sb = cluster.map_shared_rank(scores, cb / per)[cb % per];
            topk_merge(K, sa, ca < nc ? ca : -1, sb, cb < nc ? cb : -1, ls, lc);
        }
        if (lane >= K) { ls = -CUDART_INF_F; lc = -1; }
        int sc_; float sw, ss;
        topk_finish(K, ls, lc, sc_, sw, ss);
        if (lane < K) {
            slot_c[lane] = sc_;
            slot_w[lane] = sw;
            if (rank == 0) {
                if (idx_out) idx_out[(int64_t)bg * K + lane] = sc_;
                if (w_out) w_out[(int64_t)bg * K + lane] = sw;
            }
        }
    }
    __syncthreads();

    // ---- 3. attention to the chunks of this CTA's slots
    const T *kbase = kc + (int64_t)bg * P * D;
    const T *vbase = vc + (int64_t)bg * P * D;
    for (int kk = rank; kk < K; kk += kDecCta) {
        const int c = slot_c[kk];
        if (c < 0) break;  // valid slots form a prefix
        const float wk = slot_w[kk];
        __syncthreads();
        for (int e = tid * 4; e < kChunk * D; e += kDecThreads * 4) {
            // 4 consecutive elements of one row (D is a multiple of 4)
            const int i = e / D, j = e % D;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                Ks[i * (D + 1) + j + u] = Elem<T>::load(kbase + (int64_t)c * kChunk * D + e + u);
                Vs[e + u] = Elem<T>::load(vbase + (int64_t)c * kChunk * D + e + u);
            }
        }
        __syncthreads();
        for (int e = tid; e < G * kChunk; e += kDecThreads) {
            const int h = e / kChunk, i = e % kChunk;
            const float *qh = Qs + h * D;
            const float *ki = Ks + i * (D + 1);
            float acc = 0.f;
#pragma unroll 8
            for (int j = 0; j < D; ++j) acc = fmaf(qh[j], ki[j], acc);
            Pm[e] = acc * scale;
        }
        __syncthreads();
        for (int h = warp; h < G; h += kDecThreads / 32) {
            const float x0 = Pm[h * kChunk + lane], x1 = Pm[h * kChunk + lane + 32];
            float m = fmaxf(0.f, fmaxf(x0, x1));
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
            const float e0 = expf(x0 - m), e1 = expf(x1 - m);
            float z = e0 + e1;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
            z += expf(-m);
            Pm[h * kChunk + lane] = e0;
            Pm[h * kChunk + lane + 32] = e1;
            if (lane == 0) coef[h] = wk / z;
        }
        __syncthreads();
        for (int e = tid; e < G * D; e += kDecThreads) {
            const int h = e / D, j = e % D;
            const float *ph = Pm + h * kChunk;
            float acc = 0.f;
#pragma unroll 8
            for (int i = 0; i < kChunk; ++i) acc = fmaf(ph[i], Vs[i * D + j], acc);
            part[e] = fmaf(coef[h], acc, part[e]);
        }
    }
    cluster.sync();

    // ---- 4. sum the partial outputs of the cluster (DSMEM), this CTA's column share
    const int ncol = G * D;
    const int cper = (ncol + kDecCta - 1) / kDecCta;
    for (int e = rank * cper + tid; e < min(ncol, (rank + 1) * cper); e += kDecThreads) {
        float acc = 0.f;
#pragma unroll
        for (int r = 0; r < kDecCta; ++r) acc += cluster.map_shared_rank(part, r)[e];
        Elem<T>::store(o + ((int64_t)b * hq + (int64_t)g * G) * D + e, acc);
    }
    cluster.sync();
}

size_t decode_cluster_smem(int nc, int d) {
    const int per = (nc + kDecCta - 1) / kDecCta;
    return sizeof(float) * ((size_t)((per + 3) & ~3) + 2 * (size_t)kMaxG * d + (size_t)kChunk * (d + 1) +
                            (size_t)kChunk * d + (size_t)kMaxG * kChunk);
}

template <typename T, int D>
static cudaError_t decode_launch(const Shape &sh, const void *q, const void *q_slc, const void *kc, const void *vc,
                                 const float *kbar, void *o, int32_t *idx_out, float *w_out, cudaStream_t st) {
    const size_t smem = decode_cluster_smem(sh.nc, D);
    cudaError_t e = set_smem_once((const void *)decode_cluster_kernel<T, D>, smem);
    if (e != cudaSuccess) return e;
    decode_cluster_kernel<T, D><<<(unsigned)(sh.B * sh.hkv * kDecCta), kDecThreads, smem, st>>>(
        (const T *)q, (const T *)q_slc, (const T *)kc, (const T *)vc, kbar, (T *)o, idx_out, w_out, sh.L, sh.hq,
        sh.hkv, sh.nc, sh.K, sh.G);
    return cudaGetLastError();
}

bool decode_cluster_supported(const Shape &sh) {
    return (sh.d == 64 || sh.d == 128) && sh.G <= kMaxG && sh.K <= kMaxK &&
           decode_cluster_smem(sh.nc, sh.d) <= 200 * 1024;
}

cudaError_t launch_decode_cluster(const Shape &sh, const void *q, const void *q_slc, const void *kc,
                                  const void *vc, const float *kbar, void *o, int32_t *idx_out, float *w_out,
                                  DevStatus *, cudaStream_t st) {
    if (sh.B == 0) return cudaSuccess;
    if (sh.bf16)
        return sh.d == 128 ? decode_launch<__nv_bfloat16, 128>(sh, q, q_slc, kc, vc, kbar, o, idx_out, w_out, st)
                           : decode_launch<__nv_bfloat16, 64>(sh, q, q_slc, kc, vc, kbar, o, idx_out, w_out, st);
    return sh.d == 128 ? decode_launch<float, 128>(sh, q, q_slc, kc, vc, kbar, o, idx_out, w_out, st)
                       : decode_launch<float, 64>(sh, q, q_slc, kc, vc, kbar, o, idx_out, w_out, st);
}

}  // namespace hsa
