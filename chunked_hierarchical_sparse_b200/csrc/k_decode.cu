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
//   1. CTA r scores its slice of the chunk index (coalesced 512 B rows) and
//      takes the slice's own top-K (a bitonic sort in one warp's registers; a
//      long slice is first cut down by a threshold), then stores that list into
//      every CTA of the cluster (remote shared-memory stores).
//   2. cluster barrier; warp 0 of every CTA sorts the kDecCta lists (the
//      overall top-K is among them) in registers, orders the best K
//      most-recent-first and forms the stick-breaking weights.
//   3. CTA r attends the group's G query heads to the chunk of slot r (and
//      r + kDecCta, ...), softmax-off-by-one, and scales by w / Z.
//   4. CTA r stores its partial output into its own slot of the owner CTA of
//      each output column (remote shared-memory stores); cluster barrier; each
//      CTA sums its columns' slots in rank order (the result does not depend
//      on timing) and writes them.
#include <cooperative_groups.h>
#include <type_traits>
#include <math_constants.h>

#include "hsa_internal.cuh"
#include "topk_warp.cuh"

namespace cg = cooperative_groups;

namespace hsa {


constexpr int kDecCta = 8;
constexpr int kDecThreads = 128;

// shared::cluster address of `p` (this CTA's shared memory) in the CTA of cluster rank `rank`
__device__ __forceinline__ uint32_t dsmem_addr(const void *p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"((uint32_t)__cvta_generic_to_shared(p)), "r"(rank));
    return r;
}
// 8-byte store into another cluster CTA's shared memory
__device__ __forceinline__ void dsmem_st2(uint32_t addr, float x, float y) {
    asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(x), "f"(y) : "memory");
}
// 16-byte store into another cluster CTA's shared memory
__device__ __forceinline__ void dsmem_st4(uint32_t addr, float4 v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w)
                 : "memory");
}

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

// Sorts the 32 E (score, chunk) pairs a warp holds, best first under `beats`:
// element i = 32 e + lane sits in lane `lane`, register e.  Bitonic network: a
// pair that is 32 or more apart lies in one lane, a closer one across lanes.
template <int E>
__device__ __forceinline__ void warp_sort_best_first(float (&s)[E], int (&c)[E], int lane) {
#pragma unroll
    for (int k = 2; k <= 32 * E; k <<= 1)
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j >= 32) {
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const int p = e ^ (j >> 5);
                    if (p <= e) continue;
                    // the lower position keeps the better entry in a block sorted best first
                    const bool up = ((e * 32 + lane) & k) == 0;
                    if (up == beats(s[p], c[p], s[e], c[e])) {
                        const float ts = s[e]; s[e] = s[p]; s[p] = ts;
                        const int tc = c[e]; c[e] = c[p]; c[p] = tc;
                    }
                }
            } else {
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const float os = __shfl_xor_sync(0xffffffffu, s[e], j);
                    const int oc = __shfl_xor_sync(0xffffffffu, c[e], j);
                    const int i = e * 32 + lane;
                    const bool keep_better = ((i & j) == 0) == ((i & k) == 0);
                    if (keep_better == beats(os, oc, s[e], c[e])) { s[e] = os; c[e] = oc; }
                }
            }
        }
}

// The best K (<= 32) of the n entries (s_i, c_i) = (src_s[i], c0 + i), i < n <= 32 E,
// sorted in one warp: lane r < K receives the r-th best ((-inf, -1) past n).
template <int E>
__device__ __forceinline__ void warp_top_of_scores(const float *src_s, int c0, int n, int lane, float &ls, int &lc) {
    float s[E];
    int c[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int i = e * 32 + lane;
        s[e] = i < n ? src_s[i] : -CUDART_INF_F;
        c[e] = i < n ? c0 + i : -1;
    }
    warp_sort_best_first<E>(s, c, lane);
    ls = s[0];
    lc = c[0];
}

// The same for n <= 32 E entries given as (score, chunk bits) pairs.
template <int E>
__device__ __forceinline__ void warp_top_of_pairs(const float2 *src, int n, int lane, float &ls, int &lc) {
    float s[E];
    int c[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int i = e * 32 + lane;
        const float2 v = i < n ? src[i] : make_float2(-CUDART_INF_F, __int_as_float(-1));
        s[e] = v.x;
        c[e] = __float_as_int(v.y);
    }
    warp_sort_best_first<E>(s, c, lane);
    ls = s[0];
    lc = c[0];
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
    const int per4 = (per + 3) & ~3;
    const int tot = NL * G * D;                       // output values of the step (a multiple of 64)
    const int cper = tot / kDecCta;                   // columns owned by each CTA (a multiple of 8)
    // every region below is a multiple of 16 bytes long
    float *scores = sm;                               // [per]
    float *part = scores + per4;                      // [NL][G][D] partial outputs of this CTA's slots
    float *Qs = part + tot;                           // [16][D] one layer's queries
    float *Ks = Qs + kMaxG * D;                       // [64][D+1]
    float *Vs = Ks + kChunk * (D + 1);                // [64][D]
    float *Pm = Vs + kChunk * D;                      // [G][64]
    float *surv_s = Pm + kMaxG * kChunk;              // [per] slice entries not beaten by the threshold
    int *surv_c = reinterpret_cast<int *>(surv_s + per4);
    float *stage = reinterpret_cast<float *>(surv_c + per4);  // [kDecCta][cper] every source's part of my columns
    __shared__ float tmax_s[kDecThreads / 32];
    __shared__ int tmax_c[kDecThreads / 32];
    __shared__ float loc_s[kMaxK];               // a long slice's top-K, best first
    __shared__ int loc_c[kMaxK];
    __shared__ float2 cand[kDecCta * kMaxK];     // every slice's list: (score, chunk bits), written by its CTA
    __shared__ int n_surv;
    __shared__ int slot_c[kMaxK];
    __shared__ float slot_w[kMaxK];
    __shared__ float coef[kMaxG];

    // every CTA of the cluster must be running before its shared memory is written
    // from another: arrive now, wait before the first remote store (after the scores)
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

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
    for (int e = tid; e < tot; e += kDecThreads) part[e] = 0.f;

    // ---- 1b. this slice's top-K, into every CTA's candidate list.  Order: (s1, c1)
    // beats (s2, c2) iff s1 > s2, or s1 == s2 and c1 > c2.  A slice of up to 128
    // chunks is sorted by warp 0 in registers.  A longer one is first cut down: each
    // thread keeps the best of its entries and each warp sorts its 32 bests; a warp's
    // K-th is a lower bound of the slice's K-th best score (the warp holds K distinct
    // entries at least as good), the best of the warps' bounds is the threshold, and
    // the entries it does not beat are ranked pairwise.
    __syncthreads();  // scores[] written
    const int nloc = c_hi - c_lo;
    float ls = -CUDART_INF_F;  // warp 0, lane r < K: the slice's r-th best
    int lc = -1;
    if (nloc <= 128) {
        if (warp == 0) {
            if (nloc <= 32) warp_top_of_scores<1>(scores, c_lo, nloc, lane, ls, lc);
            else if (nloc <= 64) warp_top_of_scores<2>(scores, c_lo, nloc, lane, ls, lc);
            else warp_top_of_scores<4>(scores, c_lo, nloc, lane, ls, lc);
        }
    } else {
        {
            float bs[1] = {-CUDART_INF_F};
            int bc[1] = {-1};
            for (int i = tid; i < nloc; i += kDecThreads)
                if (beats(scores[i], c_lo + i, bs[0], bc[0])) { bs[0] = scores[i]; bc[0] = c_lo + i; }
            warp_sort_best_first<1>(bs, bc, lane);
            if (lane == K - 1) { tmax_s[warp] = bs[0]; tmax_c[warp] = bc[0]; }
        }
        if (tid == 0) n_surv = 0;
        __syncthreads();
        {
            float ts = tmax_s[0];
            int tc = tmax_c[0];
#pragma unroll
            for (int w = 1; w < kDecThreads / 32; ++w)
                if (beats(tmax_s[w], tmax_c[w], ts, tc)) { ts = tmax_s[w]; tc = tmax_c[w]; }
            for (int i = tid; i < nloc; i += kDecThreads)
                if (!beats(ts, tc, scores[i], c_lo + i)) {
                    const int j = atomicAdd(&n_surv, 1);
                    surv_s[j] = scores[i];
                    surv_c[j] = c_lo + i;
                }
            if (tid < K) { loc_s[tid] = -CUDART_INF_F; loc_c[tid] = -1; }  // fewer than K entries in the slice
        }
        __syncthreads();
        {
            const int ns = n_surv;
            for (int i = tid; i < ns; i += kDecThreads) {
                const float si = surv_s[i];
                const int ci = surv_c[i];
                int rk = 0;
                for (int j = 0; j < ns; ++j) rk += beats(surv_s[j], surv_c[j], si, ci) ? 1 : 0;
                if (rk < K) { loc_s[rk] = si; loc_c[rk] = ci; }
            }
        }
        __syncthreads();
        if (warp == 0 && lane < K) { ls = loc_s[lane]; lc = loc_c[lane]; }
    }
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    if (warp == 0 && lane < K) {
#pragma unroll
        for (int r = 0; r < kDecCta; ++r) dsmem_st2(dsmem_addr(&cand[rank * K + lane], (uint32_t)r), ls, __int_as_float(lc));
    }
    cluster.sync();

    // ---- 2. the overall top-K: the best K of the kDecCta slice lists (every CTA
    // sorts the same candidates, so all take the same selection); most-recent-first
    // order and the stick-breaking weights
    if (warp == 0) {
        float ms;
        int mc;
        if (K <= 4) warp_top_of_pairs<1>(cand, kDecCta * K, lane, ms, mc);
        else if (K <= 8) warp_top_of_pairs<2>(cand, kDecCta * K, lane, ms, mc);
        else warp_top_of_pairs<4>(cand, kDecCta * K, lane, ms, mc);
        int sc_; float sw, ss;
        topk_finish(K, ms, mc, sc_, sw, ss);
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
                attend_chunk16<D>(Q16, K16, V16, part + l * G * D, G, wk, scale, warp, lane);
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
        float *pl = part + l * G * D;
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
    // ---- 4. this CTA's partial output stored into its slot at the owners of its
    // columns (the CTAs with a selected chunk are the ranks below n_src; the others
    // hold zeros and send nothing); after the barrier every owner holds all the
    // parts of its columns, and no CTA touches another's shared memory any more
    int n_src = 0;
    while (n_src < kDecCta && n_src < K && slot_c[n_src] >= 0) ++n_src;
    if (rank < n_src) {
        for (int e = 4 * tid; e < tot; e += 4 * kDecThreads) {  // cper is a multiple of 4: one owner per vector
            const int ow = e / cper;
            dsmem_st4(dsmem_addr(stage + rank * cper + (e - ow * cper), (uint32_t)ow),
                      *reinterpret_cast<const float4 *>(part + e));
        }
    }
    cluster.sync();
    const int ncol = G * D;
    for (int i = tid; i < cper; i += kDecThreads) {
        float acc = 0.f;
        for (int r = 0; r < n_src; ++r) acc += stage[r * cper + i];  // rank order
        const int e = rank * cper + i, l = e / ncol, col = e - l * ncol;
        Elem<T>::store(o + (int64_t)l * lstride + ((int64_t)b * hq + (int64_t)g * G) * D + col, acc);
    }
}


size_t decode_cluster_smem(int nc, int d, int NL, int G) {
    const size_t per4 = (size_t)(((nc + kDecCta - 1) / kDecCta + 3) & ~3);
    const size_t tot = (size_t)NL * G * d;
    // scores, survivors (2), part and stage, Q, K, V, P
    return sizeof(float) * (3 * per4 + 2 * tot + (size_t)kMaxG * d + (size_t)kChunk * (d + 1) + (size_t)kChunk * d +
                            (size_t)kMaxG * kChunk);
}

template <typename T, int D>
static cudaError_t decode_launch(const Shape &sh, int NL, const void *q, const void *q_slc, const void *kc,
                                 const void *vc, const float *kbar, void *o, int32_t *idx_out, float *w_out,
                                 cudaStream_t st) {
    const size_t smem = decode_cluster_smem(sh.nc, D, NL, sh.G);
    cudaError_t e = set_smem_once((const void *)decode_cluster_kernel<T, D>, smem);
    if (e != cudaSuccess) return e;
    decode_cluster_kernel<T, D><<<(unsigned)(sh.B * sh.hkv * kDecCta), kDecThreads, smem, st>>>(
        (const T *)q, (const T *)q_slc, (const T *)kc, (const T *)vc, kbar, (T *)o, idx_out, w_out, sh.L, sh.hq,
        sh.hkv, sh.nc, sh.K, sh.G, NL, (int64_t)sh.B * sh.hq * D);
    return cudaGetLastError();
}

bool decode_cluster_supported(const Shape &sh, int NL) {
    return sh.S == kChunk && (sh.d == 64 || sh.d == 128) && sh.G <= kMaxG && sh.K <= kMaxK && NL >= 1 &&
           decode_cluster_smem(sh.nc, sh.d, NL, sh.G) <= 200 * 1024;
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
