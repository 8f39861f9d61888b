// k_select.cu -- chunk pooling and chunk selection on CUDA cores.
//
// Cited page: "Hardware-aligned Hierarchical Sparse Attention for Efficient
// Long-term Memory Access" (paper notes), §HSA "Chunk Selection": every token
// scores the mean-pooled key of each chunk with its selection query and each
// query group keeps its own top-K; §HSA second stage: stick-breaking weights
// from the sigmoid of the score.  §training/inference: the chunk index is
// floor(L/S) x d per KV head.
#include "hsa_internal.cuh"
#include "topk_warp.cuh"

namespace hsa {

// ------------------------------------------------------------------ pooling
// One warp per (b, g, chunk), four warps per block.  A lane owns VEC = 16 /
// sizeof(T) columns (one 16-byte load per row) and 64 / RS of the chunk's rows
// (RS = 32 / (d / VEC) row parts per warp); it sums them in fp64 with sixteen
// loads in flight, the row parts are combined by shuffles, and the mean is
// rounded once to fp32.  The fp64 sum of 64 bf16 (or fp32) values of one tensor
// is exact, so the result does not depend on the summation order.
//
// With x.hi set (bf16 inputs) the same pass also writes the two-term bf16 split
// of each pooled key (hi = bf16(kbar), lo = bf16(kbar - hi)) that the tensor-core
// selection scores with, and, with x.vmax_bits set, reads the chunk's values too
// and max-es max|v| (float bits; non-negative floats order like their bit
// patterns) into *x.vmax_bits: the scale of the chunk-major attention's fp16
// accumulators, which only ever sum values of complete chunks.
template <typename T>
__global__ void __launch_bounds__(128, 4) pool_kernel(const T *__restrict__ k, float *__restrict__ kbar,
                                                   int L, int d, int S, int nc, int64_t nchunks,
                                                   PoolExtras x) {
    constexpr int VEC = 16 / sizeof(T);
    constexpr int NB = 8;  // rows in flight per lane and tensor (4 blocks per SM stay resident)
    const int lane = threadIdx.x & 31;
    const int64_t bgc = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;  // this warp's chunk
    if (bgc >= nchunks) return;
    const int tpc = d / VEC;      // lanes per row (8, 16 or 32)
    const int rs = 32 / tpc;      // row parts
    const int lr = lane % tpc, part = lane / tpc;
    const int rows = S / rs;       // rows of the chunk per row part
    const int c = (int)(bgc % nc);
    const int64_t bg = bgc / nc;
    const int64_t off = ((bg * L + (int64_t)c * S + (int64_t)part * rows) * d) + lr * VEC;
    const T *src = k + off;
    double acc[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] = 0.0;
    const T *vsrc = x.vmax_bits ? static_cast<const T *>(x.v) + off : nullptr;  // bf16 values of the same chunk
    float m = 0.f;
    for (int r0 = 0; r0 < rows; r0 += NB) {
        // the round's key rows and value rows are all in flight together
        // a part shorter than NB rows (S = 16 with 4 row parts) loads zeros past its end
        uint4 raw[NB], rv[NB];
#pragma unroll
        for (int u = 0; u < NB; ++u)
            raw[u] = (r0 + u < rows) ? __ldcs(reinterpret_cast<const uint4 *>(src + (int64_t)(r0 + u) * d))
                                     : make_uint4(0, 0, 0, 0);
        if (vsrc) {
#pragma unroll
            for (int u = 0; u < NB; ++u)
                rv[u] = (r0 + u < rows) ? __ldcs(reinterpret_cast<const uint4 *>(vsrc + (int64_t)(r0 + u) * d))
                                        : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < NB; ++u) {
            const T *vals = reinterpret_cast<const T *>(&raw[u]);
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] += (double)Elem<T>::load(vals + e);
        }
        if (vsrc) {
#pragma unroll
            for (int u = 0; u < NB; ++u) {
                const T *vals = reinterpret_cast<const T *>(&rv[u]);
#pragma unroll
                for (int e = 0; e < VEC; ++e) m = fmaxf(m, fabsf(Elem<T>::load(vals + e)));
            }
        }
    }
    if (vsrc) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) atomicMax(x.vmax_bits, __float_as_int(m));
    }
    for (int o = tpc; o < 32; o <<= 1)
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
    if (part == 0) {
        float out[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) out[e] = (float)(acc[e] / S);
        float4 *dst = reinterpret_cast<float4 *>(kbar + bgc * d + lr * VEC);
#pragma unroll
        for (int e = 0; e < VEC / 4; ++e) dst[e] = make_float4(out[4 * e], out[4 * e + 1], out[4 * e + 2], out[4 * e + 3]);
        if (x.hi) {
            __align__(16) __nv_bfloat16 h[VEC], l[VEC];
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                h[e] = __float2bfloat16_rn(out[e]);
                l[e] = __float2bfloat16_rn(out[e] - __bfloat162float(h[e]));
            }
            const int64_t o2 = bgc * d + lr * VEC;
#pragma unroll
            for (int e = 0; e < VEC / 8; ++e) {
                reinterpret_cast<uint4 *>(x.hi + o2)[e] = reinterpret_cast<const uint4 *>(h)[e];
                reinterpret_cast<uint4 *>(x.lo + o2)[e] = reinterpret_cast<const uint4 *>(l)[e];
            }
        }
    }
}

cudaError_t launch_pool(const Shape &sh, const void *k, float *kbar, DevStatus *, cudaStream_t st,
                        const PoolExtras &x) {
    const int64_t chunks = (int64_t)sh.B * sh.hkv * sh.nc;
    if (chunks == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)ceil_div(chunks, 4);  // 4 warps = 4 chunks per block
    if (sh.bf16)
        pool_kernel<__nv_bfloat16><<<blocks, 128, 0, st>>>((const __nv_bfloat16 *)k, kbar, sh.L, sh.d, sh.S, sh.nc,
                                                            chunks, x);
    else
        pool_kernel<float><<<blocks, 128, 0, st>>>((const float *)k, kbar, sh.L, sh.d, sh.S, sh.nc, chunks,
                                                   PoolExtras{});  // split and max|v| serve bf16 paths only
    return cudaGetLastError();
}

// ------------------------------------------------------------------ selection
// Block = 64 tokens of one (b, g); 256 threads.  Chunk tiles of 64 pooled keys
// are scored as a 64x64 fp32 tile (4x4 per thread), then each warp merges its
// 8 tokens' rows into running top-K lists kept in shared memory.
constexpr int kSelTok = 64;
constexpr int kSelCh = 64;

template <typename T>
__global__ void __launch_bounds__(256) select_simt_kernel(
    const T *__restrict__ q_slc, const float *__restrict__ kbar, int32_t *__restrict__ idx,
    float *__restrict__ w, int L, int hkv, int d, int S, int nc, int K) {
    extern __shared__ float4 smem4[];
    float *sm = reinterpret_cast<float *>(smem4);
    float *qT = sm;                                 // [d][64]
    float *kT = qT + d * kSelTok;                   // [d][64]
    float *sc = kT + d * kSelCh;                    // [64][65]
    float *best_s = sc + kSelTok * (kSelCh + 1);    // [64][kMaxK]
    int *best_c = reinterpret_cast<int *>(best_s + kSelTok * kMaxK);

    const int bg = blockIdx.y;
    const int b = bg / hkv, g = bg % hkv;
    const int t0 = blockIdx.x * kSelTok;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float scale = 1.0f / sqrtf((float)d);

    for (int e = tid; e < kSelTok * d; e += blockDim.x) {
        const int tt = e / d, j = e % d, t = t0 + tt;
        qT[j * kSelTok + tt] = (t < L) ? Elem<T>::load(q_slc + (((int64_t)b * L + t) * hkv + g) * d + j) : 0.f;
    }
    for (int e = tid; e < kSelTok * kMaxK; e += blockDim.x) {
        best_s[e] = -CUDART_INF_F;
        best_c[e] = -1;
    }
    const int tlast = min(t0 + kSelTok, L) - 1;
    const int ne_max = min(tlast / S, nc);
    const int ty = tid / 16, tx = tid % 16;
    const float *kb = kbar + (int64_t)bg * nc * d;

    for (int c0 = 0; c0 < ne_max; c0 += kSelCh) {
        __syncthreads();
        for (int e = tid; e < kSelCh * d; e += blockDim.x) {
            const int cc = e / d, j = e % d;
            kT[j * kSelCh + cc] = (c0 + cc < nc) ? kb[(int64_t)(c0 + cc) * d + j] : 0.f;
        }
        __syncthreads();
        float acc[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) acc[a][bb] = 0.f;
        for (int j = 0; j < d; ++j) {
            const float4 qa = *reinterpret_cast<const float4 *>(qT + j * kSelTok + ty * 4);
            const float4 ka = *reinterpret_cast<const float4 *>(kT + j * kSelCh + tx * 4);
            const float qv[4] = {qa.x, qa.y, qa.z, qa.w};
            const float kv[4] = {ka.x, ka.y, ka.z, ka.w};
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int bb = 0; bb < 4; ++bb) acc[a][bb] = fmaf(qv[a], kv[bb], acc[a][bb]);
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) sc[(ty * 4 + a) * (kSelCh + 1) + tx * 4 + bb] = acc[a][bb] * scale;
        __syncthreads();
        for (int tt = warp * 8; tt < warp * 8 + 8; ++tt) {
            const int t = t0 + tt;
            if (t >= L) break;
            const int ne = min(t / S, nc);
            const int ca = c0 + lane, cb = c0 + lane + 32;
            const float sa = sc[tt * (kSelCh + 1) + lane];
            const float sb = sc[tt * (kSelCh + 1) + lane + 32];
            float ls = (lane < K) ? best_s[tt * kMaxK + lane] : CUDART_INF_F;
            int lc = (lane < K) ? best_c[tt * kMaxK + lane] : 0x7fffffff;
            topk_merge(K, sa, ca < ne ? ca : -1, sb, cb < ne ? cb : -1, ls, lc);
            if (lane < K) {
                best_s[tt * kMaxK + lane] = ls;
                best_c[tt * kMaxK + lane] = lc;
            }
        }
    }
    __syncthreads();
    for (int tt = warp * 8; tt < warp * 8 + 8; ++tt) {
        const int t = t0 + tt;
        if (t >= L) break;
        const float ls = (lane < K) ? best_s[tt * kMaxK + lane] : -CUDART_INF_F;
        const int lc = (lane < K) ? best_c[tt * kMaxK + lane] : -1;
        int sc_; float sw, ss;
        topk_finish(K, ls, lc, sc_, sw, ss);
        if (lane < K) {
            const int64_t o = (((int64_t)b * L + t) * hkv + g) * K + lane;
            idx[o] = sc_;
            w[o] = sw;
        }
    }
}

size_t select_simt_smem(int d) {
    return sizeof(float) * ((size_t)d * kSelTok + (size_t)d * kSelCh + kSelTok * (kSelCh + 1) +
                            kSelTok * kMaxK) + sizeof(int) * kSelTok * kMaxK;
}

cudaError_t launch_select_simt(const Shape &sh, const void *q_slc, const float *kbar, int32_t *idx,
                               float *w, DevStatus *, cudaStream_t st) {
    if (sh.B == 0 || sh.L == 0) return cudaSuccess;
    dim3 grid((unsigned)ceil_div(sh.L, kSelTok), (unsigned)(sh.B * sh.hkv));
    const size_t smem = select_simt_smem(sh.d);
    cudaError_t e;
    if (sh.bf16) {
        e = set_smem_once((const void *)select_simt_kernel<__nv_bfloat16>, (size_t)(smem));
        if (e != cudaSuccess) return e;
        select_simt_kernel<__nv_bfloat16><<<grid, 256, smem, st>>>(
            (const __nv_bfloat16 *)q_slc, kbar, idx, w, sh.L, sh.hkv, sh.d, sh.S, sh.nc, sh.K);
    } else {
        e = set_smem_once((const void *)select_simt_kernel<float>, (size_t)(smem));
        if (e != cudaSuccess) return e;
        select_simt_kernel<float><<<grid, 256, smem, st>>>((const float *)q_slc, kbar, idx, w, sh.L,
                                                           sh.hkv, sh.d, sh.S, sh.nc, sh.K);
    }
    return cudaGetLastError();
}

}  // namespace hsa
