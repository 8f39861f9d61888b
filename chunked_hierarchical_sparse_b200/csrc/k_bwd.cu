// k_bwd.cu -- the two-phase backward on CUDA cores.
//
// Cited page: "Hardware-aligned Hierarchical Sparse Attention for Efficient
// Long-term Memory Access" (paper notes), §kernel: phase 1 walks each token's
// K chunks and accumulates the gradients of Q and of the chunk weights w;
// phase 2 walks, for each chunk, every token that selected it and accumulates
// the gradients of K and V.  §HSA "end-to-end learning": the chunk weight's
// gradient reaches the selection score, hence q_slc and the pooled keys.
//
// Per token t, head h in group g, slot k (chunk c, weight w_k), with
// p = softmax-off-by-one(x), x_i = q.k_i/sqrt(d), O_k = sum_i p_i v_i:
//   Delta_{t,h,k} = dO . O_k          dw_k = sum_{h in g} Delta_{t,h,k}
//   dx_i = w_k p_i (dO . v_i - Delta)  dq += dx_i k_i / sqrt(d)
//   dk_i += dx_i q / sqrt(d)           dv_i += w_k p_i dO
//   ds_j = dw_j w_j (1 - sig_j) - sig_j sum_{k>j} dw_k w_k
//   dq_slc += ds_j kbar_{c_j} / sqrt(d);  dkbar_{c_j} += ds_j q_slc / sqrt(d)
//   dk (keys of chunk c) += dkbar_c / S        (mean pooling)
// p is recomputed from the forward's lse: p_i = exp(x_i - lse).
#include <algorithm>
#include <type_traits>

#include "hsa_internal.cuh"

namespace hsa {

constexpr int kB1Threads = 128;

// ------------------------------------------------------------------ phase 1
// One block per (token t, b*hkv + g).
template <typename T, int MAXPER>
__global__ void __launch_bounds__(kB1Threads) bwd_phase1_kernel(
    const T *__restrict__ q, const T *__restrict__ q_slc, const T *__restrict__ k,
    const T *__restrict__ v, const T *__restrict__ dO, const float *__restrict__ lse,
    const int32_t *__restrict__ idx, const float *__restrict__ w, const float *__restrict__ kbar,
    T *__restrict__ dq, T *__restrict__ dq_slc, float *__restrict__ dkbar, float *__restrict__ delta,
    int L, int hq, int hkv, int d, int S, int nc, int K, int G, DevStatus *ds) {
    extern __shared__ float4 smem4[];
    float *sm = reinterpret_cast<float *>(smem4);
    float *Ks = sm;                        // [S][d+1]
    float *Vs = Ks + S * (d + 1);          // [S][d+1]
    float *Qs = Vs + S * (d + 1);          // [G][d]
    float *dOs = Qs + G * d;               // [G][d]
    float *Pm = dOs + G * d;               // [G][S]
    float *dPm = Pm + G * S;               // [G][S]
    float *Dl = dPm + G * S;               // [G]
    __shared__ int slot_c[kMaxK];
    __shared__ float slot_w[kMaxK];
    __shared__ float dw_s[kMaxK];
    __shared__ float ds_s[kMaxK];

    const int t = blockIdx.x, bg = blockIdx.y, b = bg / hkv, g = bg % hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t row = (int64_t)b * L + t;
    const float scale = 1.0f / sqrtf((float)d);
    if (tid < K) {
        int c = idx[(row * hkv + g) * K + tid];
        if (c >= 0 && (c >= nc || c >= t / S)) {
            report(ds, HSA_ERR_DEVICE_CHECK, kKBwd1, (int)row, c);
            c = -1;
        }
        slot_c[tid] = c;
        slot_w[tid] = (c >= 0) ? w[(row * hkv + g) * K + tid] : 0.f;
        dw_s[tid] = 0.f;
    }
    for (int e = tid; e < G * d; e += kB1Threads) {
        Qs[e] = Elem<T>::load(q + (row * hq + (int64_t)g * G) * d + e);
        dOs[e] = Elem<T>::load(dO + (row * hq + (int64_t)g * G) * d + e);
    }
    __syncthreads();
    float dqa[MAXPER];
#pragma unroll
    for (int i = 0; i < MAXPER; ++i) dqa[i] = 0.f;
    const T *kb = k + (int64_t)bg * L * d;
    const T *vb = v + (int64_t)bg * L * d;
    for (int kk = 0; kk < K; ++kk) {
        const int c = slot_c[kk];
        if (c < 0) {
            for (int h = tid; h < G; h += kB1Threads) delta[(row * hq + (int64_t)g * G + h) * K + kk] = 0.f;
            continue;
        }
        const float wk = slot_w[kk];
        __syncthreads();
        for (int e = tid; e < S * d; e += kB1Threads) {
            const int i = e / d, j = e % d;
            Ks[i * (d + 1) + j] = Elem<T>::load(kb + (int64_t)c * S * d + e);
            Vs[i * (d + 1) + j] = Elem<T>::load(vb + (int64_t)c * S * d + e);
        }
        __syncthreads();
        for (int e = tid; e < G * S; e += kB1Threads) {
            const int h = e / S, i = e % S;
            float ax = 0.f, ap = 0.f;
            for (int j = 0; j < d; ++j) {
                ax = fmaf(Qs[h * d + j], Ks[i * (d + 1) + j], ax);
                ap = fmaf(dOs[h * d + j], Vs[i * (d + 1) + j], ap);
            }
            const float l = lse[(row * hq + (int64_t)g * G + h) * K + kk];
            Pm[e] = expf(ax * scale - l);
            dPm[e] = ap;
        }
        __syncthreads();
        // Delta_h = dO_h . O_k,h with O_k,h = sum_i p_i v_i  (one warp per head)
        for (int h = warp; h < G; h += kB1Threads / 32) {
            float acc = 0.f;
            for (int j = lane; j < d; j += 32) {
                float o = 0.f;
                for (int i = 0; i < S; ++i) o = fmaf(Pm[h * S + i], Vs[i * (d + 1) + j], o);
                acc = fmaf(dOs[h * d + j], o, acc);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (lane == 0) {
                Dl[h] = acc;
                delta[(row * hq + (int64_t)g * G + h) * K + kk] = acc;
            }
        }
        __syncthreads();
        if (tid == 0) {
            float sdl = 0.f;
            for (int h = 0; h < G; ++h) sdl += Dl[h];
            dw_s[kk] = sdl;
        }
        for (int e = tid; e < G * S; e += kB1Threads) {
            const int h = e / S;
            dPm[e] = wk * Pm[e] * (dPm[e] - Dl[h]);  // dx
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < MAXPER; ++i) {
            const int e = tid + kB1Threads * i;
            if (e < G * d) {
                const int h = e / d, j = e % d;
                float acc = 0.f;
                for (int r = 0; r < S; ++r) acc = fmaf(dPm[h * S + r], Ks[r * (d + 1) + j], acc);
                dqa[i] = fmaf(acc, scale, dqa[i]);
            }
        }
    }
    __syncthreads();
    // stick-breaking backward (warp 0): recompute s_j = q_slc . kbar_{c_j} / sqrt(d)
    const float *kbg = kbar + (int64_t)bg * nc * d;
    if (warp == 0) {
        float s_j = 0.f;
        const int cj = (lane < K) ? slot_c[lane] : -1;
        for (int jj = 0; jj < K; ++jj) {
            const int c = slot_c[jj];
            if (c < 0) continue;
            float acc = 0.f;
            for (int j = lane; j < d; j += 32)
                acc = fmaf(Elem<T>::load(q_slc + (row * hkv + g) * d + j), kbg[(int64_t)c * d + j], acc);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (lane == jj) s_j = acc * scale;
        }
        const float sg = (cj >= 0) ? 1.0f / (1.0f + expf(-s_j)) : 0.f;
        const float wj = (lane < K) ? slot_w[lane] : 0.f;
        const float dwj = (lane < K) ? dw_s[lane] : 0.f;
        // tail_j = sum_{k>j} dw_k w_k (valid slots are a prefix; empty ones add 0)
        float prod = (cj >= 0) ? dwj * wj : 0.f;
        float incl = prod;  // suffix sum via reversed inclusive scan
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_down_sync(0xffffffffu, incl, off);
            if (lane + off < 32) incl += y;
        }
        const float tail = incl - prod;
        if (lane < K) ds_s[lane] = (cj >= 0) ? dwj * wj * (1.f - sg) - sg * tail : 0.f;
    }
    __syncthreads();
    for (int j = tid; j < d; j += kB1Threads) {
        float acc = 0.f;
        const float qsj = Elem<T>::load(q_slc + (row * hkv + g) * d + j);
        for (int jj = 0; jj < K; ++jj) {
            const int c = slot_c[jj];
            if (c < 0) continue;
            acc = fmaf(ds_s[jj], kbg[(int64_t)c * d + j], acc);
            atomicAdd(dkbar + ((int64_t)bg * nc + c) * d + j, ds_s[jj] * qsj * scale);
        }
        Elem<T>::store(dq_slc + (row * hkv + g) * d + j, acc * scale);
    }
#pragma unroll
    for (int i = 0; i < MAXPER; ++i) {
        const int e = tid + kB1Threads * i;
        if (e < G * d) Elem<T>::store(dq + (row * hq + (int64_t)g * G) * d + e, dqa[i]);
    }
}

template <typename T>
static cudaError_t phase1_dispatch(const Shape &sh, const void *q, const void *q_slc, const void *k,
                                   const void *v, const void *dO, const float *lse,
                                   const int32_t *idx, const float *w, const float *kbar, void *dq,
                                   void *dq_slc, const BwdWs &ws, DevStatus *ds, cudaStream_t st) {
    dim3 grid((unsigned)sh.L, (unsigned)(sh.B * sh.hkv));
    const size_t smem = sizeof(float) * ((size_t)2 * sh.S * (sh.d + 1) + (size_t)2 * sh.G * sh.d +
                                         (size_t)2 * sh.G * sh.S + kMaxG);
    const int per = (int)ceil_div((int64_t)sh.G * sh.d, kB1Threads);
#define HSA_B1_CASE(N)                                                                            \
    if (per <= N) {                                                                               \
        cudaError_t e = set_smem_once((const void *)bwd_phase1_kernel<T, N>, smem); \
        if (e != cudaSuccess) return e;                                                           \
        bwd_phase1_kernel<T, N><<<grid, kB1Threads, smem, st>>>(                                  \
            (const T *)q, (const T *)q_slc, (const T *)k, (const T *)v, (const T *)dO, lse, idx, w, \
            kbar, (T *)dq, (T *)dq_slc, ws.dkbar, ws.delta, sh.L, sh.hq, sh.hkv, sh.d, sh.S, sh.nc, \
            sh.K, sh.G, ds);                                                                      \
        return cudaGetLastError();                                                                \
    }
    HSA_B1_CASE(2)
    HSA_B1_CASE(4)
    HSA_B1_CASE(8)
    HSA_B1_CASE(16)
#undef HSA_B1_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_bwd_phase1(const Shape &sh, const void *q, const void *q_slc, const void *k,
                              const void *v, const void *dO, const float *lse, const int32_t *idx,
                              const float *w, const float *kbar, void *dq, void *dq_slc,
                              const BwdWs &ws, DevStatus *ds, cudaStream_t st) {
    if (sh.B == 0 || sh.L == 0) return cudaSuccess;
    return sh.bf16 ? phase1_dispatch<__nv_bfloat16>(sh, q, q_slc, k, v, dO, lse, idx, w, kbar, dq,
                                                    dq_slc, ws, ds, st)
                   : phase1_dispatch<float>(sh, q, q_slc, k, v, dO, lse, idx, w, kbar, dq, dq_slc,
                                            ws, ds, st);
}

// ------------------------------------------------------------------ phase 2
// Grid (segment, b*hkv): segment z of (b, g) belongs to the chunk c with
// seg_off[c] <= z < seg_off[c+1] and covers list entries
// [off_c + (z - seg_off[c])*SEG, ... + SEG).  A block takes min(S, 64) keys of the chunk
// (blockIdx.z picks the 64-key half of a 128-key chunk), four threads per key: key row
// i = tid/4, column quarter jq = tid%4; the thread keeps its quarter of k_i, v_i and of
// the dk_i, dv_i accumulators in registers.  Partial sums are added into fp32
// accumulators; a finishing kernel adds dkbar/S and rounds.
constexpr int kB2Threads = 256;  // the most threads a block takes (64 keys, 4 per key)
constexpr int kB2Seg = kBwdSeg;

template <typename T, int DQ>
__global__ void __launch_bounds__(kB2Threads) bwd_phase2_kernel(
    const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v, const T *__restrict__ dO,
    const float *__restrict__ lse, const float *__restrict__ w, const float *__restrict__ delta,
    const int32_t *__restrict__ chunk_off, const int32_t *__restrict__ seg_off,
    const int32_t *__restrict__ entries, float *__restrict__ dk_acc, float *__restrict__ dv_acc,
    int L, int hq, int hkv, int S, int nc, int K, int G) {
    constexpr int d = DQ * 4;
    __shared__ float qs[d], dos[d];
    const int z = blockIdx.x, bg = blockIdx.y, b = bg / hkv, g = bg % hkv;
    const int32_t *so = seg_off + (int64_t)bg * (nc + 1);
    if (z >= so[nc]) return;
    int lo = 0, hi = nc - 1;  // last c with so[c] <= z
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (so[mid] <= z) lo = mid; else hi = mid - 1;
    }
    const int c = lo;
    const int32_t *off = chunk_off + (int64_t)bg * (nc + 1);
    const int beg = off[c] + (z - so[c]) * kB2Seg;
    const int end = min(off[c + 1], beg + kB2Seg);
    if (beg >= end) return;
    const int tid = threadIdx.x, i = (tid >> 2) + 64 * (int)blockIdx.z, jq = tid & 3;
    const float scale = 1.0f / sqrtf((float)d);
    const int64_t krow = ((int64_t)bg * L + (int64_t)c * S + i) * d + jq * DQ;
    float kr[DQ], vr[DQ], dka[DQ], dva[DQ];
#pragma unroll
    for (int e = 0; e < DQ; ++e) {
        kr[e] = Elem<T>::load(k + krow + e);
        vr[e] = Elem<T>::load(v + krow + e);
        dka[e] = 0.f;
        dva[e] = 0.f;
    }
    const int32_t *E = entries + (int64_t)bg * L * K;
    for (int p = beg; p < end; ++p) {
        const int ent = E[p];
        const int t = ent >> 4, kk = ent & 15;
        const int64_t row = (int64_t)b * L + t;
        const float wk = w[(row * hkv + g) * K + kk];
        for (int h = g * G; h < (g + 1) * G; ++h) {
            __syncthreads();
            for (int j = tid; j < d; j += blockDim.x) {
                qs[j] = Elem<T>::load(q + (row * hq + h) * d + j);
                dos[j] = Elem<T>::load(dO + (row * hq + h) * d + j);
            }
            __syncthreads();
            float ax = 0.f, ap = 0.f;
#pragma unroll
            for (int e = 0; e < DQ; ++e) {
                ax = fmaf(qs[jq * DQ + e], kr[e], ax);
                ap = fmaf(dos[jq * DQ + e], vr[e], ap);
            }
            ax += __shfl_xor_sync(0xffffffffu, ax, 1);
            ax += __shfl_xor_sync(0xffffffffu, ax, 2);
            ap += __shfl_xor_sync(0xffffffffu, ap, 1);
            ap += __shfl_xor_sync(0xffffffffu, ap, 2);
            const float pi = expf(ax * scale - lse[(row * hq + h) * K + kk]);
            const float dx = wk * pi * (ap - delta[(row * hq + h) * K + kk]);
            const float wp = wk * pi;
#pragma unroll
            for (int e = 0; e < DQ; ++e) {
                dka[e] = fmaf(dx * scale, qs[jq * DQ + e], dka[e]);
                dva[e] = fmaf(wp, dos[jq * DQ + e], dva[e]);
            }
        }
    }
#pragma unroll
    for (int e = 0; e < DQ; ++e) {
        atomicAdd(dk_acc + krow + e, dka[e]);
        atomicAdd(dv_acc + krow + e, dva[e]);
    }
}

// dk = dk_acc + dkbar_c / S; dv = dv_acc; rows of the trailing partial chunk = 0.
// One thread per 4 consecutive values of a row (d is a multiple of 4); 1/S is exact
// (S is a power of two), so the product equals the quotient.
template <typename T>
__device__ __forceinline__ void store4(T *p, float4 v) {
    if constexpr (std::is_same<T, float>::value) {
        *reinterpret_cast<float4 *>(p) = v;
    } else {
        __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
        uint2 u;
        u.x = *reinterpret_cast<uint32_t *>(&a);
        u.y = *reinterpret_cast<uint32_t *>(&b);
        *reinterpret_cast<uint2 *>(p) = u;
    }
}

template <typename T>
__global__ void bwd_finish_kernel(const float *__restrict__ dk_acc, const float *__restrict__ dv_acc,
                                  const float *__restrict__ dkbar, T *__restrict__ dk, T *__restrict__ dv,
                                  int L, int d, int S, int nc, int64_t total) {
    const int d4 = d / 4;
    const float inv_s = 1.0f / (float)S;
    for (int64_t e4 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e4 < total / 4;
         e4 += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = e4 / d4;  // row (b, g, t)
        const int j = (int)(e4 - r * d4) * 4;
        const int t = (int)(r % L);
        const int64_t bg = r / L;
        const int c = t / S;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), bv = a;
        if (c < nc) {
            a = *reinterpret_cast<const float4 *>(dk_acc + e4 * 4);
            const float4 kb = *reinterpret_cast<const float4 *>(dkbar + (bg * nc + c) * d + j);
            a.x += kb.x * inv_s; a.y += kb.y * inv_s; a.z += kb.z * inv_s; a.w += kb.w * inv_s;
            bv = *reinterpret_cast<const float4 *>(dv_acc + e4 * 4);
        }
        store4<T>(dk + e4 * 4, a);
        store4<T>(dv + e4 * 4, bv);
    }
}

template <typename T>
static cudaError_t phase2_dispatch(const Shape &sh, const void *q, const void *k, const void *v,
                                   const void *dO, const float *lse, const float *w, void *dk,
                                   void *dv, const BwdWs &ws, cudaStream_t st) {
    // dk_acc/dv_acc are laid out [B*hkv, nc*S, d]; k/v rows use stride L.
    if (sh.nc > 0) {
        // a (b, g) has at most L*K/SEG + nc segments
        const int maxseg = (int)(ceil_div((int64_t)sh.L * sh.K, kB2Seg) + sh.nc);
        dim3 grid(maxseg, sh.B * sh.hkv, sh.S > 64 ? sh.S / 64 : 1);
        const unsigned nthr = 4 * (unsigned)std::min(sh.S, 64);  // one thread per (key, column quarter)
        if (sh.d == 128)
            bwd_phase2_kernel<T, 32><<<grid, nthr, 0, st>>>(
                (const T *)q, (const T *)k, (const T *)v, (const T *)dO, lse, w, ws.delta, ws.chunk_off,
                ws.seg_off, ws.entries, ws.dk_acc, ws.dv_acc, sh.L, sh.hq, sh.hkv, sh.S, sh.nc, sh.K, sh.G);
        else
            bwd_phase2_kernel<T, 16><<<grid, nthr, 0, st>>>(
                (const T *)q, (const T *)k, (const T *)v, (const T *)dO, lse, w, ws.delta, ws.chunk_off,
                ws.seg_off, ws.entries, ws.dk_acc, ws.dv_acc, sh.L, sh.hq, sh.hkv, sh.S, sh.nc, sh.K, sh.G);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const int64_t total = (int64_t)sh.B * sh.hkv * sh.L * sh.d;
    const int blocks = (int)std::min<int64_t>(ceil_div(total / 4, 256), 148 * 16);
    bwd_finish_kernel<T><<<blocks, 256, 0, st>>>(ws.dk_acc, ws.dv_acc, ws.dkbar, (T *)dk, (T *)dv,
                                                  sh.L, sh.d, sh.S, sh.nc, total);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t finish_dispatch(const Shape &sh, const BwdWs &ws, void *dk, void *dv, cudaStream_t st) {
    const int64_t total = (int64_t)sh.B * sh.hkv * sh.L * sh.d;
    if (total == 0) return cudaSuccess;
    const int blocks = (int)std::min<int64_t>(ceil_div(total / 4, 256), 148 * 16);
    bwd_finish_kernel<T><<<blocks, 256, 0, st>>>(ws.dk_acc, ws.dv_acc, ws.dkbar, (T *)dk, (T *)dv, sh.L, sh.d,
                                                  sh.S, sh.nc, total);
    return cudaGetLastError();
}

cudaError_t launch_bwd_finish(const Shape &sh, const BwdWs &ws, void *dk, void *dv, cudaStream_t st) {
    return sh.bf16 ? finish_dispatch<__nv_bfloat16>(sh, ws, dk, dv, st) : finish_dispatch<float>(sh, ws, dk, dv, st);
}

cudaError_t launch_bwd_phase2(const Shape &sh, const void *q, const void *k, const void *v,
                              const void *dO, const float *lse, const float *w, void *dk, void *dv,
                              const BwdWs &ws, DevStatus *, cudaStream_t st) {
    if (sh.B == 0 || sh.L == 0) return cudaSuccess;
    return sh.bf16 ? phase2_dispatch<__nv_bfloat16>(sh, q, k, v, dO, lse, w, dk, dv, ws, st)
                   : phase2_dispatch<float>(sh, q, k, v, dO, lse, w, dk, dv, ws, st);
}

}  // namespace hsa
