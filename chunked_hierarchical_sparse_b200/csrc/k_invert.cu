// k_invert.cu -- invert the token->chunk selection into per-chunk lists.
//
// Cited page: "Hardware-aligned Hierarchical Sparse Attention for Efficient
// Long-term Memory Access" (paper notes), §kernel: the second backward phase
// walks, for each chunk, all tokens that selected it.  The lists are built as
// a stable counting sort keyed by chunk, so each chunk's entries come out in
// increasing token order and the result is deterministic:
//   1. per block of 256 tokens, a histogram over chunks;
//   2. per (b, g), a prefix over token blocks for every chunk and an exclusive
//      scan over chunks (CSR offsets);
//   3. per token block, one warp walks its tokens in order and places each
//      (token, slot) entry at its chunk's running cursor.
// Entry encoding: t * 16 + slot.
#include "hsa_internal.cuh"

namespace hsa {

__global__ void __launch_bounds__(256) inv_hist_kernel(const int32_t *__restrict__ idx,
                                                       int32_t *__restrict__ hist, int L, int hkv,
                                                       int nc, int K, int ntb, DevStatus *ds) {
    extern __shared__ int h_s[];
    const int tb = blockIdx.x, bg = blockIdx.y, b = bg / hkv, g = bg % hkv;
    for (int c = threadIdx.x; c < nc; c += blockDim.x) h_s[c] = 0;
    __syncthreads();
    const int t0 = tb * kInvTokBlock;
    for (int e = threadIdx.x; e < kInvTokBlock * K; e += blockDim.x) {
        const int t = t0 + e / K, kk = e % K;
        if (t >= L) break;
        const int c = idx[(((int64_t)b * L + t) * hkv + g) * K + kk];
        if (c < 0) continue;
        if (c >= nc || c >= t / kChunk) {
            report(ds, HSA_ERR_DEVICE_CHECK, kKInvert, t, c);
            continue;
        }
        atomicAdd(&h_s[c], 1);
    }
    __syncthreads();
    int32_t *out = hist + ((int64_t)bg * ntb + tb) * nc;
    for (int c = threadIdx.x; c < nc; c += blockDim.x) out[c] = h_s[c];
}

// In-place exclusive scan of a[0..n) by a block of 1024 threads; returns the total.
__device__ int block_exclusive_scan(int *a, int n, int *wsum) {
    const int per = (n + blockDim.x - 1) / blockDim.x;
    const int c0 = threadIdx.x * per;
    int local = 0;
    for (int c = c0; c < min(c0 + per, n); ++c) local += a[c];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    __syncthreads();
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int v = (lane < (int)(blockDim.x >> 5)) ? wsum[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, v, off);
            if (lane >= off) v += y;
        }
        wsum[lane] = v;  // inclusive over warps
    }
    __syncthreads();
    int run = incl - local + (warp > 0 ? wsum[warp - 1] : 0);
    const int total = wsum[(blockDim.x >> 5) - 1];
    for (int c = c0; c < min(c0 + per, n); ++c) {
        const int v = a[c];
        a[c] = run;
        run += v;
    }
    __syncthreads();
    return total;
}

// One block (1024 threads) per (b, g): per-chunk prefix over token blocks,
// CSR offsets over chunks, and the per-chunk segment table of phase 2.
__global__ void __launch_bounds__(1024) inv_scan_kernel(int32_t *__restrict__ hist,
                                                        int32_t *__restrict__ chunk_off,
                                                        int32_t *__restrict__ seg_off, int nc,
                                                        int ntb, int seg) {
    extern __shared__ int sm_i[];
    int *cnt_s = sm_i;        // [nc]
    int *seg_s = sm_i + nc;   // [nc]
    __shared__ int wsum[32];
    const int bg = blockIdx.x;
    int32_t *H = hist + (int64_t)bg * ntb * nc;
    for (int c = threadIdx.x; c < nc; c += blockDim.x) {
        int run = 0;
        for (int tb = 0; tb < ntb; ++tb) {
            const int v = H[(int64_t)tb * nc + c];
            H[(int64_t)tb * nc + c] = run;
            run += v;
        }
        cnt_s[c] = run;
        seg_s[c] = (run + seg - 1) / seg;
    }
    __syncthreads();
    const int total = block_exclusive_scan(cnt_s, nc, wsum);
    const int nseg = block_exclusive_scan(seg_s, nc, wsum);
    for (int c = threadIdx.x; c < nc; c += blockDim.x) {
        chunk_off[(int64_t)bg * (nc + 1) + c] = cnt_s[c];
        seg_off[(int64_t)bg * (nc + 1) + c] = seg_s[c];
        const int base = cnt_s[c];
        for (int tb = 0; tb < ntb; ++tb) H[(int64_t)tb * nc + c] += base;
    }
    if (threadIdx.x == 0) {
        chunk_off[(int64_t)bg * (nc + 1) + nc] = total;
        seg_off[(int64_t)bg * (nc + 1) + nc] = nseg;
    }
}

// One warp per (token block, b*hkv + g): tokens in order, slots in parallel.
__global__ void __launch_bounds__(32) inv_scatter_kernel(const int32_t *__restrict__ idx,
                                                         const int32_t *__restrict__ hist,
                                                         int32_t *__restrict__ entries, int L,
                                                         int hkv, int nc, int K, int ntb) {
    extern __shared__ int cur[];  // [nc]
    const int tb = blockIdx.x, bg = blockIdx.y, b = bg / hkv, g = bg % hkv;
    const int lane = threadIdx.x;
    const int32_t *H = hist + ((int64_t)bg * ntb + tb) * nc;
    for (int c = lane; c < nc; c += 32) cur[c] = H[c];
    __syncwarp();
    int32_t *E = entries + (int64_t)bg * L * K;
    const int t0 = tb * kInvTokBlock;
    const int t1 = min(t0 + kInvTokBlock, L);
    for (int t = t0; t < t1; ++t) {
        if (lane < K) {
            const int c = idx[(((int64_t)b * L + t) * hkv + g) * K + lane];
            if (c >= 0 && c < nc && c < t / kChunk) {
                const int pos = cur[c];
                cur[c] = pos + 1;
                E[pos] = t * 16 + lane;
            }
        }
        __syncwarp();
    }
}

cudaError_t launch_invert(const Shape &sh, const int32_t *idx, const BwdWs &ws, DevStatus *ds,
                          cudaStream_t st) {
    if (sh.B == 0 || sh.L == 0 || sh.nc == 0) return cudaSuccess;
    const int ntb = (int)ceil_div(sh.L, kInvTokBlock);
    const size_t smem = sizeof(int) * (size_t)sh.nc;
    cudaError_t e;
    if (2 * smem > 48 * 1024) {
        e = set_smem_once((const void *)inv_hist_kernel, (size_t)(smem));
        if (e != cudaSuccess) return e;
        e = set_smem_once((const void *)inv_scan_kernel, (size_t)(2 * smem));
        if (e != cudaSuccess) return e;
        e = set_smem_once((const void *)inv_scatter_kernel, (size_t)(smem));
        if (e != cudaSuccess) return e;
    }
    dim3 grid(ntb, sh.B * sh.hkv);
    inv_hist_kernel<<<grid, 256, smem, st>>>(idx, ws.hist, sh.L, sh.hkv, sh.nc, sh.K, ntb, ds);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    inv_scan_kernel<<<sh.B * sh.hkv, 1024, 2 * smem, st>>>(ws.hist, ws.chunk_off, ws.seg_off, sh.nc,
                                                            ntb, kBwdSeg);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    inv_scatter_kernel<<<grid, 32, smem, st>>>(idx, ws.hist, ws.entries, sh.L, sh.hkv, sh.nc, sh.K, ntb);
    return cudaGetLastError();
}

}  // namespace hsa
