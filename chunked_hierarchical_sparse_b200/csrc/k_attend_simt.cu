// k_attend_simt.cu -- token-major softmax-off-by-one chunk attention and
// stick-breaking fusion on CUDA cores, plus the decode step built on it.
//
// Cited page: "Hardware-aligned Hierarchical Sparse Attention for Efficient
// Long-term Memory Access" (paper notes), §kernel: per token the output starts
// at zero, and for each selected chunk the chunk's K/V is brought on chip,
// attention with a softmax-off-by-one is taken inside it, and the result is
// added with the chunk's weight.  This is that token-major order, one block per
// (token, KV group) with the group's query heads together; it serves the fp32
// path and the decode step.  The bf16 prefill path uses the chunk-major
// tensor-core kernel instead.
#include "hsa_internal.cuh"
#include "topk_warp.cuh"

namespace hsa {

constexpr int kAttThreads = 128;

// Shared-memory layout for one (token, group) block; S keys per chunk.
struct AttSmem {
    float *Ks;   // [S][d+1]
    float *Vs;   // [S][d]
    float *Qs;   // [G][d]
    float *P;    // [G][S]
    float *coef; // [G]
};

__host__ __device__ inline size_t att_smem_floats(int d, int G, int S) {
    return (size_t)S * (d + 1) + (size_t)S * d + (size_t)G * d + (size_t)G * S + kMaxG;
}

__device__ inline AttSmem att_carve(float *sm, int d, int G, int S) {
    AttSmem s;
    s.Ks = sm;
    s.Vs = s.Ks + S * (d + 1);
    s.Qs = s.Vs + S * d;
    s.P = s.Qs + G * d;
    s.coef = s.P + G * S;
    return s;
}

// Attend the G query rows (already in s.Qs) to the K slots (chunk ids in
// slot_c[], weights in slot_w[], both in shared memory); accumulate
// o[h][j] for the thread's (h, j) pairs e = tid + 128 * i.
// kv_base points at chunk 0 of this (b, g) in the [.., L, d] K/V layout.
template <typename T, int MAXPER>
__device__ void attend_group(const T *__restrict__ kbase, const T *__restrict__ vbase, int d, int G, int S,
                             int K, const int *slot_c, const float *slot_w, AttSmem s,
                             float (&oacc)[MAXPER], float *lse_out /* [G][K] or null, stride K */) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float scale = 1.0f / sqrtf((float)d);
    for (int kk = 0; kk < K; ++kk) {
        const int c = slot_c[kk];
        if (c < 0) {
            if (lse_out)
                for (int h = tid; h < G; h += kAttThreads) lse_out[h * K + kk] = 0.f;
            continue;
        }
        const float wk = slot_w[kk];
        __syncthreads();
        const T *kc = kbase + (int64_t)c * S * d;
        const T *vc = vbase + (int64_t)c * S * d;
        for (int e = tid; e < S * d; e += kAttThreads) {
            const int i = e / d, j = e % d;
            s.Ks[i * (d + 1) + j] = Elem<T>::load(kc + e);
            s.Vs[e] = Elem<T>::load(vc + e);
        }
        __syncthreads();
        for (int e = tid; e < G * S; e += kAttThreads) {
            const int h = e / S, i = e % S;
            const float *qh = s.Qs + h * d;
            const float *ki = s.Ks + i * (d + 1);
            float acc = 0.f;
            for (int j = 0; j < d; ++j) acc = fmaf(qh[j], ki[j], acc);
            s.P[e] = acc * scale;
        }
        __syncthreads();
        // softmax-off-by-one per head: m = max(0, max x); Z = e^{-m} + sum e^{x-m}
        // (lane takes keys lane, lane + 32, ...)
        for (int h = warp; h < G; h += kAttThreads / 32) {
            float xv[kMaxS / 32];
            float m = 0.f;
#pragma unroll
            for (int u = 0; u < kMaxS / 32; ++u) {
                const int i = lane + 32 * u;
                xv[u] = (i < S) ? s.P[h * S + i] : -CUDART_INF_F;
                m = fmaxf(m, xv[u]);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
            float z = 0.f;
#pragma unroll
            for (int u = 0; u < kMaxS / 32; ++u) {
                const int i = lane + 32 * u;
                if (i < S) {
                    const float ev = expf(xv[u] - m);
                    s.P[h * S + i] = ev;
                    z += ev;
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
            z += expf(-m);
            if (lane == 0) {
                s.coef[h] = wk / z;
                if (lse_out) lse_out[h * K + kk] = m + logf(z);
            }
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < MAXPER; ++i) {
            const int e = tid + kAttThreads * i;
            if (e < G * d) {
                const int h = e / d, j = e % d;
                const float *ph = s.P + h * S;
                float acc = 0.f;
                for (int r = 0; r < S; ++r) acc = fmaf(ph[r], s.Vs[r * d + j], acc);
                oacc[i] = fmaf(s.coef[h], acc, oacc[i]);
            }
        }
    }
}

// One block per (token t, b*hkv + g).
template <typename T, int MAXPER>
__global__ void __launch_bounds__(kAttThreads) attend_simt_kernel(
    const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
    const int32_t *__restrict__ idx, const float *__restrict__ w, T *__restrict__ o,
    float *__restrict__ lse, int L, int hq, int hkv, int d, int S, int nc, int K, int G, DevStatus *ds) {
    extern __shared__ float4 smem4[];
    float *sm = reinterpret_cast<float *>(smem4);
    AttSmem s = att_carve(sm, d, G, S);
    __shared__ int slot_c[kMaxK];
    __shared__ float slot_w[kMaxK];
    const int t = blockIdx.x;
    const int bg = blockIdx.y, b = bg / hkv, g = bg % hkv;
    const int tid = threadIdx.x;
    const int64_t row = (int64_t)b * L + t;
    if (tid < K) {
        int c = idx[(row * hkv + g) * K + tid];
        if (c >= 0 && (c >= nc || c >= t / S)) {
            report(ds, HSA_ERR_DEVICE_CHECK, kKAttendSimt, (int)row, c);
            c = -1;
        }
        slot_c[tid] = c;
        slot_w[tid] = (c >= 0) ? w[(row * hkv + g) * K + tid] : 0.f;
    }
    for (int e = tid; e < G * d; e += kAttThreads)
        s.Qs[e] = Elem<T>::load(q + (row * hq + (int64_t)g * G) * d + e);
    __syncthreads();
    float oacc[MAXPER];
#pragma unroll
    for (int i = 0; i < MAXPER; ++i) oacc[i] = 0.f;
    const T *kbase = k + (int64_t)bg * L * d;
    const T *vbase = v + (int64_t)bg * L * d;
    attend_group<T, MAXPER>(kbase, vbase, d, G, S, K, slot_c, slot_w, s, oacc,
                            lse ? lse + (row * hq + (int64_t)g * G) * K : nullptr);
#pragma unroll
    for (int i = 0; i < MAXPER; ++i) {
        const int e = tid + kAttThreads * i;
        if (e < G * d) Elem<T>::store(o + (row * hq + (int64_t)g * G) * d + e, oacc[i]);
    }
}

template <typename T>
static cudaError_t attend_dispatch(const Shape &sh, const void *q, const void *k, const void *v,
                                   const int32_t *idx, const float *w, void *o, float *lse,
                                   DevStatus *ds, cudaStream_t st) {
    dim3 grid((unsigned)sh.L, (unsigned)(sh.B * sh.hkv));
    const size_t smem = att_smem_floats(sh.d, sh.G, sh.S) * sizeof(float);
    const int per = (int)ceil_div((int64_t)sh.G * sh.d, kAttThreads);
#define HSA_ATT_CASE(N)                                                                          \
    if (per <= N) {                                                                              \
        cudaError_t e = set_smem_once((const void *)attend_simt_kernel<T, N>, smem); \
        if (e != cudaSuccess) return e;                                                          \
        attend_simt_kernel<T, N><<<grid, kAttThreads, smem, st>>>(                               \
            (const T *)q, (const T *)k, (const T *)v, idx, w, (T *)o, lse, sh.L, sh.hq, sh.hkv,  \
            sh.d, sh.S, sh.nc, sh.K, sh.G, ds);                                                  \
        return cudaGetLastError();                                                               \
    }
    HSA_ATT_CASE(2)
    HSA_ATT_CASE(4)
    HSA_ATT_CASE(8)
    HSA_ATT_CASE(16)
#undef HSA_ATT_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_attend_simt(const Shape &sh, const void *q, const void *k, const void *v,
                               const int32_t *idx, const float *w, void *o, float *lse,
                               DevStatus *ds, cudaStream_t st) {
    if (sh.B == 0 || sh.L == 0) return cudaSuccess;
    return sh.bf16 ? attend_dispatch<__nv_bfloat16>(sh, q, k, v, idx, w, o, lse, ds, st)
                   : attend_dispatch<float>(sh, q, k, v, idx, w, o, lse, ds, st);
}

// ------------------------------------------------------------------ decode
// One block per (b, g): score all floor(P/S) cached chunks against the
// selection query (one warp per chunk, lanes along d), keep the top-K with
// warp 0, then attend the group's query heads to the chosen chunks.
template <typename T, int MAXPER>
__global__ void __launch_bounds__(kAttThreads) decode_simt_kernel(
    const T *__restrict__ q, const T *__restrict__ q_slc, const T *__restrict__ kc,
    const T *__restrict__ vc, const float *__restrict__ kbar, T *__restrict__ o,
    int32_t *__restrict__ idx_out, float *__restrict__ w_out, int P, int hq, int hkv, int d, int S, int nc,
    int K, int G) {
    extern __shared__ float4 smem4[];
    float *sm = reinterpret_cast<float *>(smem4);
    AttSmem s = att_carve(sm, d, G, S);
    float *scores = s.coef + kMaxG;  // [nc]
    float *qs = scores + nc;         // [d]
    __shared__ int slot_c[kMaxK];
    __shared__ float slot_w[kMaxK];
    const int bg = blockIdx.x, b = bg / hkv, g = bg % hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float scale = 1.0f / sqrtf((float)d);
    for (int j = tid; j < d; j += kAttThreads) qs[j] = Elem<T>::load(q_slc + (int64_t)bg * d + j);
    for (int e = tid; e < G * d; e += kAttThreads)
        s.Qs[e] = Elem<T>::load(q + ((int64_t)b * hq + (int64_t)g * G) * d + e);
    __syncthreads();
    const float *kb = kbar + (int64_t)bg * nc * d;
    for (int c = warp; c < nc; c += kAttThreads / 32) {
        float acc = 0.f;
        for (int j = lane; j < d; j += 32) acc = fmaf(qs[j], kb[(int64_t)c * d + j], acc);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) scores[c] = acc * scale;
    }
    __syncthreads();
    if (warp == 0) {
        float ls = (lane < K) ? -CUDART_INF_F : CUDART_INF_F;
        int lc = (lane < K) ? -1 : 0x7fffffff;
        for (int c0 = 0; c0 < nc; c0 += 64) {
            const int ca = c0 + lane, cb = c0 + lane + 32;
            topk_merge(K, ca < nc ? scores[ca] : 0.f, ca < nc ? ca : -1, cb < nc ? scores[cb] : 0.f,
                       cb < nc ? cb : -1, ls, lc);
        }
        if (lane >= K) { ls = -CUDART_INF_F; lc = -1; }
        int sc_; float sw, ss;
        topk_finish(K, ls, lc, sc_, sw, ss);
        if (lane < K) {
            slot_c[lane] = sc_;
            slot_w[lane] = sw;
            if (idx_out) idx_out[(int64_t)bg * K + lane] = sc_;
            if (w_out) w_out[(int64_t)bg * K + lane] = sw;
        }
    }
    __syncthreads();
    float oacc[MAXPER];
#pragma unroll
    for (int i = 0; i < MAXPER; ++i) oacc[i] = 0.f;
    attend_group<T, MAXPER>(kc + (int64_t)bg * P * d, vc + (int64_t)bg * P * d, d, G, S, K, slot_c,
                            slot_w, s, oacc, nullptr);
#pragma unroll
    for (int i = 0; i < MAXPER; ++i) {
        const int e = tid + kAttThreads * i;
        if (e < G * d) Elem<T>::store(o + ((int64_t)b * hq + (int64_t)g * G) * d + e, oacc[i]);
    }
}

template <typename T>
static cudaError_t decode_dispatch(const Shape &sh, const void *q, const void *q_slc, const void *kc,
                                   const void *vc, const float *kbar, void *o, int32_t *idx_out,
                                   float *w_out, cudaStream_t st) {
    const size_t smem = (att_smem_floats(sh.d, sh.G, sh.S) + (size_t)sh.nc + sh.d) * sizeof(float);
    const int per = (int)ceil_div((int64_t)sh.G * sh.d, kAttThreads);
#define HSA_DEC_CASE(N)                                                                           \
    if (per <= N) {                                                                               \
        cudaError_t e = set_smem_once((const void *)decode_simt_kernel<T, N>, smem); \
        if (e != cudaSuccess) return e;                                                           \
        decode_simt_kernel<T, N><<<(unsigned)(sh.B * sh.hkv), kAttThreads, smem, st>>>(           \
            (const T *)q, (const T *)q_slc, (const T *)kc, (const T *)vc, kbar, (T *)o, idx_out,   \
            w_out, sh.L, sh.hq, sh.hkv, sh.d, sh.S, sh.nc, sh.K, sh.G);                           \
        return cudaGetLastError();                                                                \
    }
    HSA_DEC_CASE(2)
    HSA_DEC_CASE(4)
    HSA_DEC_CASE(8)
    HSA_DEC_CASE(16)
#undef HSA_DEC_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode_simt(const Shape &sh, const void *q, const void *q_slc, const void *kc,
                               const void *vc, const float *kbar, void *o, int32_t *idx_out,
                               float *w_out, DevStatus *, cudaStream_t st) {
    if (sh.B == 0) return cudaSuccess;
    return sh.bf16 ? decode_dispatch<__nv_bfloat16>(sh, q, q_slc, kc, vc, kbar, o, idx_out, w_out, st)
                   : decode_dispatch<float>(sh, q, q_slc, kc, vc, kbar, o, idx_out, w_out, st);
}

}  // namespace hsa
