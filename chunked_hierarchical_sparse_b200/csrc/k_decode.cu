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
//   2. cluster barrier; every CTA reads all scores over DSMEM and selects
//      the same top-K with all its threads: a threshold (the K-th best of the
//      per-thread bests) leaves a few survivors, which are ranked pairwise;
//      warp 0 orders the K most-recent-first and forms the stick-breaking
//      weights.
//   3. CTA r attends the group's G query heads to the chunk of slot r (and
//      r + kDecCta, ...), softmax-off-by-one, and scales by w / Z.
//   4. cluster barrier; CTA r sums its share of the output columns over all
//      CTAs' partial outputs (DSMEM) and writes o; a last barrier keeps every
//      CTA's shared memory alive until all remote reads are done.
#include <cooperative_groups.h>
#include <type_traits>
#include <math_constants.h>

#include "hsa_internal.cuh"
#include "topk_warp.cuh"

namespace cg = cooperative_groups;

namespace hsa {


constexpr int kDecCta = 8;
constexpr int kDecThreads = 128;

// The chunk's K (to a padded [64][D+1] fp32 tile) and V (to [64][D] fp32): every
// thread issues all of its 16-byte loads before the first store.
template <typename T, int D>
__device__ __forceinline__ void load_chunk(const T *__restrict__ kc, const T *__restrict__ vc, float *Ks, float *Vs,
                                           int tid) {
    constexpr int EPV = 16 / sizeof(T);                  // elements per 16-byte vector
    constexpr int NV = kChunk * D / EPV / kDecThreads;   // vectors per thread and tensor
    constexpr int NB = NV < 8 ? NV : 8;                  // vectors in flight per batch
#pragma unroll 1
    for (int u0 = 0; u0 < NV; u0 += NB) {
    uint4 rk[NB], rv[NB];
#pragma unroll
    for (int u = 0; u < NB; ++u) {
        rk[u] = __ldcs(reinterpret_cast<const uint4 *>(kc) + tid + (u0 + u) * kDecThreads);
        rv[u] = __ldcs(reinterpret_cast<const uint4 *>(vc) + tid + (u0 + u) * kDecThreads);
    }
#pragma unroll
    for (int u = 0; u < NB; ++u) {
        const int e = (tid + (u0 + u) * kDecThreads) * EPV;  // first element; the vector stays in one row
        const int i = e / D, j = e % D;
        const T *pk = reinterpret_cast<const T *>(&rk[u]);
        const T *pv = reinterpret_cast<const T *>(&rv[u]);
#pragma unroll
        for (int x = 0; x < EPV; ++x) {
            Ks[i * (D + 1) + j + x] = Elem<T>::load(pk + x);
            Vs[e + x] = Elem<T>::load(pv + x);
        }
    }
    }
}

// ---------------------------------------------------------------- bf16 tensor-core tile
// Pitches (bf16 elements) of the shared tiles of the bf16 path, padded so that the
// fragment loads of a warp hit 32 different banks.
template <int D> struct DecTile {
    static constexpr int QP = D + 8;   // Q16 [16][QP]: the G query heads (rows >= G zero)
    static constexpr int KP = D + 8;   // K16 [64][KP]
    static constexpr int VP = D + 8;   // V16 [64][VP] (row-major; read transposed by ldmatrix)
};

__device__ __forceinline__ uint32_t ld_b32(const __nv_bfloat16 *p) { return *reinterpret_cast<const uint32_t *>(p); }

// D[16x8] += A[16x16] B[16x8], bf16 operands, fp32 accumulators (one warp)
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// The chunk's K and V to K16 / V16 (row-major, padded rows), 16-byte loads issued first.
template <int D>
__device__ __forceinline__ void load_chunk16(const __nv_bfloat16 *__restrict__ kc, const __nv_bfloat16 *__restrict__ vc,
                                             __nv_bfloat16 *K16, __nv_bfloat16 *V16, int tid) {
    using DT = DecTile<D>;
    constexpr int NV = kChunk * D / 8 / kDecThreads;  // 16-byte vectors per thread and tensor
    uint4 rk[NV], rv[NV];
#pragma unroll
    for (int u = 0; u < NV; ++u) {
        rk[u] = __ldcs(reinterpret_cast<const uint4 *>(kc) + tid + u * kDecThreads);
        rv[u] = __ldcs(reinterpret_cast<const uint4 *>(vc) + tid + u * kDecThreads);
    }
#pragma unroll
    for (int u = 0; u < NV; ++u) {
        const int e = (tid + u * kDecThreads) * 8;
        const int i = e / D, j = e % D;
        *reinterpret_cast<uint4 *>(K16 + i * DT::KP + j) = rk[u];
        *reinterpret_cast<uint4 *>(V16 + i * DT::VP + j) = rv[u];
    }
}

// One selected chunk on the tensor cores: every warp computes the G x 64 scores
// (heads padded to 16 rows), applies softmax-off-by-one in registers, and adds
// w / Z * P V for its quarter of the d columns into part[G][D].
template <int D>
__device__ __forceinline__ void attend_chunk16(const __nv_bfloat16 *Q16, const __nv_bfloat16 *K16,
                                               const __nv_bfloat16 *V16, float *part, int G, float wk,
                                               float scale, int warp, int lane) {
    using DT = DecTile<D>;
    const int g = lane >> 2, t = lane & 3;
    float sacc[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a[4];
        a[0] = ld_b32(Q16 + g * DT::QP + kk * 16 + 2 * t);
        a[1] = ld_b32(Q16 + (g + 8) * DT::QP + kk * 16 + 2 * t);
        a[2] = ld_b32(Q16 + g * DT::QP + kk * 16 + 2 * t + 8);
        a[3] = ld_b32(Q16 + (g + 8) * DT::QP + kk * 16 + 2 * t + 8);
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            uint32_t bb[2];
            bb[0] = ld_b32(K16 + (n * 8 + g) * DT::KP + kk * 16 + 2 * t);
            bb[1] = ld_b32(K16 + (n * 8 + g) * DT::KP + kk * 16 + 2 * t + 8);
            mma_16816(sacc[n], a, bb);
        }
    }
    // rows g (elements 0, 1) and g + 8 (elements 2, 3); a row's 64 keys live in the 4 lanes of equal g
    float m0 = 0.f, m1 = 0.f;  // the off-by-one term is a logit of 0
#pragma unroll
    for (int n = 0; n < 8; ++n) {
        m0 = fmaxf(m0, fmaxf(sacc[n][0], sacc[n][1]) * scale);
        m1 = fmaxf(m1, fmaxf(sacc[n][2], sacc[n][3]) * scale);
    }
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, off));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, off));
    }
    float z0 = 0.f, z1 = 0.f;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
        sacc[n][0] = expf(sacc[n][0] * scale - m0);
        sacc[n][1] = expf(sacc[n][1] * scale - m0);
        sacc[n][2] = expf(sacc[n][2] * scale - m1);
        sacc[n][3] = expf(sacc[n][3] * scale - m1);
        z0 += sacc[n][0] + sacc[n][1];
        z1 += sacc[n][2] + sacc[n][3];
    }
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
        z0 += __shfl_xor_sync(0xffffffffu, z0, off);
        z1 += __shfl_xor_sync(0xffffffffu, z1, off);
    }
    const float cf0 = wk / (z0 + expf(-m0)), cf1 = wk / (z1 + expf(-m1));
    // O = P V for this warp's D/4 columns; P's fragments come straight from the scores'
    constexpr int NT = D / 32;
    float oacc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        uint32_t a[4];
        a[0] = pack_bf16(sacc[2 * kk][0], sacc[2 * kk][1]);
        a[1] = pack_bf16(sacc[2 * kk][2], sacc[2 * kk][3]);
        a[2] = pack_bf16(sacc[2 * kk + 1][0], sacc[2 * kk + 1][1]);
        a[3] = pack_bf16(sacc[2 * kk + 1][2], sacc[2 * kk + 1][3]);
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int d0 = warp * (D / 4) + n * 8;
            // B fragment of V[keys 16kk.., columns d0..d0+7]: two 8x8 tiles read transposed
            // (lanes 0-7 address the rows of the first tile, lanes 8-15 those of the second)
            uint32_t bb[2];
            const uint32_t addr = (uint32_t)__cvta_generic_to_shared(V16 + (kk * 16 + (lane & 15)) * DT::VP + d0);
            asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
                         : "=r"(bb[0]), "=r"(bb[1]) : "r"(addr));
            mma_16816(oacc[n], a, bb);
        }
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const int d0 = warp * (D / 4) + n * 8 + 2 * t;
        if (g < G) {
            part[g * D + d0] += cf0 * oacc[n][0];
            part[g * D + d0 + 1] += cf0 * oacc[n][1];
        }
        if (g + 8 < G) {
            part[(g + 8) * D + d0] += cf1 * oacc[n][2];
            part[(g + 8) * D + d0 + 1] += cf1 * oacc[n][3];
        }
    }
}

// Sorts one (score, chunk) pair per lane across the warp, best first under `beats`
// (bitonic network over the 32 lanes).
__device__ __forceinline__ void warp_sort_best_first(float &s, int &c, int lane) {
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            const float os = __shfl_xor_sync(0xffffffffu, s, j);
            const int oc = __shfl_xor_sync(0xffffffffu, c, j);
            const bool keep_better = ((lane & j) == 0) == ((lane & k) == 0);
            if (keep_better == beats(os, oc, s, c)) { s = os; c = oc; }
        }
}

template <typename T, int D>
__global__ void __cluster_dims__(kDecCta, 1, 1) __launch_bounds__(kDecThreads)
    decode_cluster_kernel(const T *__restrict__ q, const T *__restrict__ q_slc, const T *__restrict__ kc,
                          const T *__restrict__ vc, const float *__restrict__ kbar, T *__restrict__ o,
                          int32_t *__restrict__ idx_out, float *__restrict__ w_out, int P, int hq, int hkv,
                          int nc, int K, int G, int NL, int64_t lstride) {
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int bg = blockIdx.x / kDecCta, b = bg / hkv, g = bg % hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float scale = 1.0f / sqrtf((float)D);

    extern __shared__ float4 dsm4[];
    float *sm = reinterpret_cast<float *>(dsm4);
    const int per = (nc + kDecCta - 1) / kDecCta;     // chunks scored by each CTA
    float *scores = sm;                               // [per]
    float *part = scores + ((per + 3) & ~3);          // [NL][G][D] partial outputs of this CTA's slots
    float *Qs = part + NL * kMaxG * D;                // [G][D] one layer's queries
    float *Ks = Qs + kMaxG * D;                       // [64][D+1]
    float *Vs = Ks + kChunk * (D + 1);                // [64][D]
    float *Pm = Vs + kChunk * D;                      // [G][64]
    const int ncr = (nc + 3) & ~3;
    float *allsc = Pm + kMaxG * kChunk;               // [nc] every chunk's score (top-K stage)
    float *surv_s = allsc + ncr;                      // [nc] candidates not beaten by the threshold
    int *surv_c = reinterpret_cast<int *>(surv_s + ncr);
    __shared__ float tmax_s[kDecThreads];
    __shared__ int tmax_c[kDecThreads];
    __shared__ float top_s[kMaxK];
    __shared__ int top_c[kMaxK];
    __shared__ int n_surv;
    __shared__ int slot_c[kMaxK];
    __shared__ float slot_w[kMaxK];
    __shared__ float coef[kMaxG];

    // ---- 1. scores of this CTA's chunk slice
    const int c_lo = rank * per, c_hi = min(nc, c_lo + per);
    const float *kb = kbar + (int64_t)bg * nc * D;
    float qv[D / 32];
#pragma unroll
    for (int e = 0; e < D / 32; ++e) qv[e] = Elem<T>::load(q_slc + (int64_t)bg * D + lane + 32 * e);
    // each warp takes 8 chunks at a time: all 8 rows of k-bar are loaded before any is used
    constexpr int kCB = 8;
    for (int c0 = c_lo + warp * kCB; c0 < c_hi; c0 += kDecThreads / 32 * kCB) {
        float kv[kCB][D / 32];
#pragma unroll
        for (int u = 0; u < kCB; ++u)
#pragma unroll
            for (int e = 0; e < D / 32; ++e)
                kv[u][e] = (c0 + u < c_hi) ? kb[(int64_t)(c0 + u) * D + lane + 32 * e] : 0.f;
#pragma unroll
        for (int u = 0; u < kCB; ++u) {
            float acc = 0.f;
#pragma unroll
            for (int e = 0; e < D / 32; ++e) acc = fmaf(qv[e], kv[u][e], acc);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (lane == 0 && c0 + u < c_hi) scores[c0 + u - c_lo] = acc * scale;
        }
    }
    constexpr bool kTc = std::is_same<T, __nv_bfloat16>::value;  // bf16: tensor-core chunk tiles
    __nv_bfloat16 *Q16 = reinterpret_cast<__nv_bfloat16 *>(Qs);
    __nv_bfloat16 *K16 = reinterpret_cast<__nv_bfloat16 *>(Ks);
    __nv_bfloat16 *V16 = reinterpret_cast<__nv_bfloat16 *>(Vs);
    // queries of layer l (all layers share this step's selection and chunks)
    auto load_q = [&](int l) {
        const T *ql = q + (int64_t)l * lstride + ((int64_t)b * hq + (int64_t)g * G) * D;
        if constexpr (kTc) {
            for (int e = tid; e < 16 * D / 8; e += kDecThreads) {  // heads padded to the MMA's 16 rows
                const int h = e / (D / 8), j = (e % (D / 8)) * 8;
                *reinterpret_cast<uint4 *>(Q16 + h * DecTile<D>::QP + j) =
                    (h < G) ? *reinterpret_cast<const uint4 *>(ql + (int64_t)h * D + j) : make_uint4(0, 0, 0, 0);
            }
        } else {
            for (int e = tid; e < G * D; e += kDecThreads)  // a few 2-byte loads per thread, all independent
                Qs[e] = Elem<T>::load(ql + e);
        }
    };
    load_q(0);
    int q_cur = 0;  // the layer whose queries Qs / Q16 hold (block-uniform)
    for (int e = tid; e < NL * kMaxG * D; e += kDecThreads) part[e] = 0.f;
    cluster.sync();

    // ---- 2. top-K over all chunks (every CTA, all threads), scores read over DSMEM.
    // Order: (s1, c1) beats (s2, c2) iff s1 > s2, or s1 == s2 and c1 > c2.
    // 2a. stage every score; each thread keeps the best of its candidates
    float bs = -CUDART_INF_F;
    int bc = -1;
    for (int c = tid; c < nc; c += 2 * kDecThreads) {  // two remote reads in flight at a time
        const int c2 = c + kDecThreads;
        const float s1 = cluster.map_shared_rank(scores, c / per)[c % per];
        const float s2 = (c2 < nc) ? cluster.map_shared_rank(scores, c2 / per)[c2 % per] : -CUDART_INF_F;
        allsc[c] = s1;
        if (beats(s1, c, bs, bc)) { bs = s1; bc = c; }
        if (c2 < nc) {
            allsc[c2] = s2;
            if (beats(s2, c2, bs, bc)) { bs = s2; bc = c2; }
        }
    }
    // 2b. threshold: each warp sorts its 32 per-thread bests, best first (bitonic network
    //     over the lanes); its K-th is a lower bound of the overall K-th best score (the
    //     warp holds K distinct candidates at least as good), and the threshold is the
    //     best of the warps' bounds
    {
        float s = bs;
        int c = bc;
        warp_sort_best_first(s, c, lane);
        if (lane == K - 1) { tmax_s[warp] = s; tmax_c[warp] = c; }
    }
    if (tid == 0) n_surv = 0;
    __syncthreads();
    // 2c. survivors: the candidates that the threshold does not beat
    {
        float ts = tmax_s[0];
        int tc = tmax_c[0];
#pragma unroll
        for (int q = 1; q < kDecThreads / 32; ++q)
            if (beats(tmax_s[q], tmax_c[q], ts, tc)) { ts = tmax_s[q]; tc = tmax_c[q]; }
        for (int c = tid; c < nc; c += kDecThreads) {
            const float sc = allsc[c];
            if (!beats(ts, tc, sc, c)) {
                const int i = atomicAdd(&n_surv, 1);
                surv_s[i] = sc;
                surv_c[i] = c;
            }
        }
    }
    __syncthreads();
    // 2d. the K best survivors, best first: with at most 32 survivors (the usual case)
    //     warp 0 sorts them in registers; otherwise every survivor is ranked pairwise
    const int ns = n_surv;
    if (ns > 32) {
        for (int i = tid; i < ns; i += kDecThreads) {
            const float si = surv_s[i];
            const int ci = surv_c[i];
            int rk = 0;
            for (int j = 0; j < ns; ++j) rk += beats(surv_s[j], surv_c[j], si, ci) ? 1 : 0;
            if (rk < K) { top_s[rk] = si; top_c[rk] = ci; }
        }
        __syncthreads();
    }
    // 2e. warp 0: most-recent-first order and the stick-breaking weights
    if (warp == 0) {
        const int nsel = min(K, ns);
        float ls, lc_s;
        int lc;
        if (ns > 32) {
            ls = (lane < nsel) ? top_s[lane] : -CUDART_INF_F;
            lc = (lane < nsel) ? top_c[lane] : -1;
        } else {
            lc_s = (lane < ns) ? surv_s[lane] : -CUDART_INF_F;
            lc = (lane < ns) ? surv_c[lane] : -1;
            warp_sort_best_first(lc_s, lc, lane);
            ls = (lane < nsel) ? lc_s : -CUDART_INF_F;
            if (lane >= nsel) lc = -1;
        }
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
        if constexpr (kTc) {
            load_chunk16<D>(kbase + (int64_t)c * kChunk * D, vbase + (int64_t)c * kChunk * D, K16, V16, tid);
            __syncthreads();
            for (int l = 0; l < NL; ++l) {  // the chunk is read once and serves every layer
                if (l != q_cur) {
                    __syncthreads();
                    load_q(l);
                    q_cur = l;
                    __syncthreads();
                }
                attend_chunk16<D>(Q16, K16, V16, part + l * kMaxG * D, G, wk, scale, warp, lane);
            }
            continue;
        }
        load_chunk<T, D>(kbase + (int64_t)c * kChunk * D, vbase + (int64_t)c * kChunk * D, Ks, Vs, tid);
        __syncthreads();
        for (int l = 0; l < NL; ++l) {
        if (l != q_cur) {
            load_q(l);
            q_cur = l;
            __syncthreads();
        }
        float *pl = part + l * kMaxG * D;
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
            pl[e] = fmaf(coef[h], acc, pl[e]);
        }
        __syncthreads();  // Qs, Pm and coef are rewritten for the next layer
        }
    }
    cluster.sync();

    // ---- 4. sum the partial outputs of the cluster (DSMEM), this CTA's column share
    const int ncol = G * D, tot = NL * ncol;
    const int cper = (tot + kDecCta - 1) / kDecCta;
    for (int e = rank * cper + tid; e < min(tot, (rank + 1) * cper); e += kDecThreads) {
        const int l = e / ncol, col = e - l * ncol;
        float acc = 0.f;
#pragma unroll
        for (int r = 0; r < kDecCta; ++r) acc += cluster.map_shared_rank(part, r)[l * kMaxG * D + col];
        Elem<T>::store(o + (int64_t)l * lstride + ((int64_t)b * hq + (int64_t)g * G) * D + col, acc);
    }
    cluster.sync();
}


size_t decode_cluster_smem(int nc, int d, int NL) {
    const int per = (nc + kDecCta - 1) / kDecCta;
    const size_t ncr = (size_t)((nc + 3) & ~3);
    return sizeof(float) * ((size_t)((per + 3) & ~3) + (size_t)(NL + 1) * kMaxG * d + (size_t)kChunk * (d + 1) +
                            (size_t)kChunk * d + (size_t)kMaxG * kChunk + 3 * ncr);
}

template <typename T, int D>
static cudaError_t decode_launch(const Shape &sh, int NL, const void *q, const void *q_slc, const void *kc,
                                 const void *vc, const float *kbar, void *o, int32_t *idx_out, float *w_out,
                                 cudaStream_t st) {
    const size_t smem = decode_cluster_smem(sh.nc, D, NL);
    cudaError_t e = set_smem_once((const void *)decode_cluster_kernel<T, D>, smem);
    if (e != cudaSuccess) return e;
    decode_cluster_kernel<T, D><<<(unsigned)(sh.B * sh.hkv * kDecCta), kDecThreads, smem, st>>>(
        (const T *)q, (const T *)q_slc, (const T *)kc, (const T *)vc, kbar, (T *)o, idx_out, w_out, sh.L, sh.hq,
        sh.hkv, sh.nc, sh.K, sh.G, NL, (int64_t)sh.B * sh.hq * D);
    return cudaGetLastError();
}

bool decode_cluster_supported(const Shape &sh, int NL) {
    return (sh.d == 64 || sh.d == 128) && sh.G <= kMaxG && sh.K <= kMaxK && NL >= 1 &&
           decode_cluster_smem(sh.nc, sh.d, NL) <= 200 * 1024;
}

cudaError_t launch_decode_cluster(const Shape &sh, int NL, const void *q, const void *q_slc, const void *kc,
                                  const void *vc, const float *kbar, void *o, int32_t *idx_out, float *w_out,
                                  DevStatus *, cudaStream_t st) {
    if (sh.B == 0) return cudaSuccess;
    if (sh.bf16)
        return sh.d == 128 ? decode_launch<__nv_bfloat16, 128>(sh, NL, q, q_slc, kc, vc, kbar, o, idx_out, w_out, st)
                           : decode_launch<__nv_bfloat16, 64>(sh, NL, q, q_slc, kc, vc, kbar, o, idx_out, w_out, st);
    return sh.d == 128 ? decode_launch<float, 128>(sh, NL, q, q_slc, kc, vc, kbar, o, idx_out, w_out, st)
                       : decode_launch<float, 64>(sh, NL, q, q_slc, kc, vc, kbar, o, idx_out, w_out, st);
}

}  // namespace hsa
