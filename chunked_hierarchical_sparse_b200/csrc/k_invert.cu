// k_invert.cu -- invert the token->chunk selection into per-chunk lists.
//
// Cited page: "Hardware-aligned Hierarchical Sparse Attention for Efficient
// Long-term Memory Access" (paper notes), §kernel: the second backward phase
// walks, for each chunk, all tokens that selected it.  The lists are built as
// a stable counting sort keyed by chunk, so each chunk's entries come out in
// increasing token order and the result is deterministic:
//   1. per block of 128 tokens, a histogram over chunks;
//   2. per (b, g), a prefix over token blocks for every chunk (column scan) and
//      an exclusive scan of the chunk totals (CSR offsets); a token block's first
//      position in chunk c's list is then chunk_off[c] + its prefix;
//   3. per token block, one warp walks its tokens in order and places each
//      (token, slot) entry at its chunk's running cursor.
// Entry encoding: t * 16 + slot.
#include "hsa_internal.cuh"

namespace hsa {

__global__ void __launch_bounds__(256) inv_hist_kernel(const int32_t *__restrict__ idx,
                                                       int32_t *__restrict__ hist, int L, int hkv,
                                                       int nc, int K, int S, int ntb, DevStatus *ds) {
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
        if (c >= nc || c >= t / S) {
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

// Per-chunk exclusive prefix over token blocks, in place, and per-chunk totals.
// Block (32 x 32) per (32-chunk strip, b*hkv + g): tx = chunk in the strip
// (coalesced rows), ty = a contiguous run of token blocks.
__global__ void __launch_bounds__(1024) inv_colscan_kernel(int32_t *__restrict__ hist,
                                                           int32_t *__restrict__ chunk_cnt, int nc,
                                                           int ntb) {
    __shared__ int part[32][33];
    const int tx = threadIdx.x, ty = threadIdx.y;
    const int c = blockIdx.x * 32 + tx, bg = blockIdx.y;
    const int per = (ntb + 31) / 32;
    const int tb0 = ty * per, tb1 = min(ntb, tb0 + per);
    int32_t *H = hist + (int64_t)bg * ntb * nc;
    int local = 0;
    if (c < nc)
        for (int tb = tb0; tb < tb1; ++tb) local += H[(int64_t)tb * nc + c];
    part[ty][tx] = local;
    __syncthreads();
    int run = 0;
    for (int y = 0; y < ty; ++y) run += part[y][tx];
    if (c < nc) {
        for (int tb = tb0; tb < tb1; ++tb) {
            const int v = H[(int64_t)tb * nc + c];
            H[(int64_t)tb * nc + c] = run;
            run += v;
        }
        if (ty == 31) chunk_cnt[(int64_t)bg * (nc + 1) + c] = run;
    }
}

// One block (1024 threads) per (b, g): CSR offsets over chunks and the
// per-chunk segment table of the backward's phase 2 (from the chunk totals).
__global__ void __launch_bounds__(1024) inv_scan_kernel(int32_t *__restrict__ chunk_off,
                                                        int32_t *__restrict__ seg_off, int nc, int seg) {
    extern __shared__ int sm_i[];
    int *cnt_s = sm_i;        // [nc]
    int *seg_s = sm_i + nc;   // [nc]
    __shared__ int wsum[32];
    const int bg = blockIdx.x;
    for (int c = threadIdx.x; c < nc; c += blockDim.x) {
        const int run = chunk_off[(int64_t)bg * (nc + 1) + c];  // the chunk's total, from inv_colscan
        cnt_s[c] = run;
        seg_s[c] = (run + seg - 1) / seg;
    }
    __syncthreads();
    const int total = block_exclusive_scan(cnt_s, nc, wsum);
    const int nseg = block_exclusive_scan(seg_s, nc, wsum);
    for (int c = threadIdx.x; c < nc; c += blockDim.x) {
        chunk_off[(int64_t)bg * (nc + 1) + c] = cnt_s[c];
        seg_off[(int64_t)bg * (nc + 1) + c] = seg_s[c];
    }
    if (threadIdx.x == 0) {
        chunk_off[(int64_t)bg * (nc + 1) + nc] = total;
        seg_off[(int64_t)bg * (nc + 1) + nc] = nseg;
    }
}


// One warp per (token block, b*hkv + g): entries placed in token order.
__global__ void __launch_bounds__(32) inv_scatter_kernel(const int32_t *__restrict__ idx,
                                                         const float *__restrict__ w,
                                                         const int32_t *__restrict__ hist,
                                                         const int32_t *__restrict__ chunk_off,
                                                         int32_t *__restrict__ entries,
                                                         float *__restrict__ entw, int L,
                                                         int hkv, int nc, int K, int S, int ntb) {
    extern __shared__ int cur[];  // [nc] cursors, [kInvTokBlock * K] the block's selections and weights
    int *sel = cur + nc;
    float *selw = reinterpret_cast<float *>(sel + kInvTokBlock * K);
    const int tb = blockIdx.x, bg = blockIdx.y, b = bg / hkv, g = bg % hkv;
    const int lane = threadIdx.x;
    const int32_t *H = hist + ((int64_t)bg * ntb + tb) * nc;
    const int32_t *off = chunk_off + (int64_t)bg * (nc + 1);
    for (int c = lane; c < nc; c += 32) cur[c] = off[c] + H[c];  // the block's first position in each list
    const int t0 = tb * kInvTokBlock;
    const int t1 = min(t0 + kInvTokBlock, L);
    for (int e = lane; e < (t1 - t0) * K; e += 32) {
        const int64_t o = (((int64_t)b * L + t0 + e / K) * hkv + g) * K + e % K;
        sel[e] = idx[o];
        if (w) selw[e] = w[o];
    }
    __syncwarp();
    int32_t *E = entries + (int64_t)bg * L * K;
    float *EW = entw ? entw + (int64_t)bg * L * K : nullptr;
    // 32 / K tokens per step, lane = (token - step start) * K + slot.  Lanes that
    // hold the same chunk take consecutive positions in lane order, i.e. by token,
    // then slot (a caller-given selection may list a chunk in several slots).
    const int tpi = 32 / K;
    for (int tb = t0; tb < t1; tb += tpi) {
        const int t = tb + lane / K, kk = lane % K;
        int c = -1;
        if (lane < tpi * K && t < t1) c = sel[(t - t0) * K + kk];
        const bool ok = c >= 0 && c < nc && c < t / S;
        const unsigned peers = __match_any_sync(0xffffffffu, ok ? c : -1 - lane);
        if (ok) {
            const int pos = cur[c] + __popc(peers & ((1u << lane) - 1u));
            E[pos] = t * 16 + kk;
            if (EW) EW[pos] = selw[(t - t0) * K + kk];
        }
        __syncwarp();
        if (ok && lane == 31 - __clz(peers)) cur[c] += __popc(peers);
        __syncwarp();
    }
}

cudaError_t launch_invert(const Shape &sh, const int32_t *idx, const float *w, const BwdWs &ws, DevStatus *ds,
                          cudaStream_t st) {
    if (sh.B == 0 || sh.L == 0 || sh.nc == 0) return cudaSuccess;
    const int ntb = (int)ceil_div(sh.L, kInvTokBlock);
    const size_t smem = sizeof(int) * (size_t)sh.nc;
    cudaError_t e;
    const size_t ssmem = smem + 2 * sizeof(int) * (size_t)kInvTokBlock * sh.K;
    if (2 * smem > 48 * 1024 || ssmem > 48 * 1024) {
        e = set_smem_once((const void *)inv_hist_kernel, (size_t)(smem));
        if (e != cudaSuccess) return e;
        e = set_smem_once((const void *)inv_scan_kernel, (size_t)(2 * smem));
        if (e != cudaSuccess) return e;
        e = set_smem_once((const void *)inv_scatter_kernel, ssmem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid(ntb, sh.B * sh.hkv);
    inv_hist_kernel<<<grid, 256, smem, st>>>(idx, ws.hist, sh.L, sh.hkv, sh.nc, sh.K, sh.S, ntb, ds);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    inv_colscan_kernel<<<dim3((unsigned)ceil_div(sh.nc, 32), sh.B * sh.hkv), dim3(32, 32), 0, st>>>(
        ws.hist, ws.chunk_off, sh.nc, ntb);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    inv_scan_kernel<<<sh.B * sh.hkv, 1024, 2 * smem, st>>>(ws.chunk_off, ws.seg_off, sh.nc, kBwdSeg);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    inv_scatter_kernel<<<grid, 32, ssmem, st>>>(idx, w, ws.hist, ws.chunk_off, ws.entries, w ? ws.entw : nullptr,
                                                 sh.L, sh.hkv, sh.nc, sh.K, sh.S, ntb);
    return cudaGetLastError();
}

}  // namespace hsa
