// k_plan.cu -- work plan of the chunk-major forward attention.
//
// Input: the token->chunk lists per (b, g) from k_invert.cu (each chunk's
// (token, slot) entries in increasing token order, with per-256-token-block
// offsets).  The tokens of each (b, g) are cut into windows of W tokens; the
// window sequence j = (b*h_kv + g)*nW + w is processed in order.  Inside a
// window, the entries of chunk c form a bucket; a bucket is cut into tiles of
// TT = 128/G tokens (the tile's rows are its tokens' G query heads) and tiles
// into work units of up to plan.unit_tiles tiles (one K/V load per unit).
//
// The persistent attention kernel pulls work units window by window (the
// units of window s form queue segment s).  Combine items are not queued:
// plan_windows records each window's tile and combine-item counts, and the
// kernel's combine warps claim a window's items as soon as all its tiles are
// stored, while its partial outputs are still in L2.
#include "hsa_internal.cuh"

namespace hsa {

// One block (1024 threads) per window j.
__global__ void __launch_bounds__(1024) plan_windows_kernel(const int32_t *__restrict__ hist,
                                                            const int32_t *__restrict__ chunk_off,
                                                            AttendPlan plan) {
    extern __shared__ int s_units[];  // [nc]
    __shared__ int wsum[32];
    __shared__ int s_tiles;
    const int j = blockIdx.x;
    const int nc = plan.nc, ntb = plan.ntb;
    const int bg = j / plan.nW, w = j % plan.nW;
    const int tb0 = w * (plan.W / kInvTokBlock);
    const int tb1 = min(ntb, (w + 1) * (plan.W / kInvTokBlock));
    const int32_t *H = hist + (int64_t)bg * ntb * nc;
    const int32_t *off = chunk_off + (int64_t)bg * (nc + 1);
    if (threadIdx.x == 0) s_tiles = 0;
    __syncthreads();
    int my_tiles = 0;
    for (int c = threadIdx.x; c < nc; c += blockDim.x) {
        // hist holds each chunk's per-block offsets within the chunk's list; off[c] is the list's start
        const int e0 = off[c] + H[(int64_t)tb0 * nc + c];
        const int e1 = (tb1 < ntb) ? off[c] + H[(int64_t)tb1 * nc + c] : off[c + 1];
        const int nt = (e1 - e0 + plan.TT - 1) / plan.TT;
        my_tiles += nt;
        s_units[c] = (nt + plan.unit_tiles - 1) / plan.unit_tiles;
    }
    atomicAdd(&s_tiles, my_tiles);
    __syncthreads();
    // exclusive scan of s_units over chunks (contiguous runs per thread)
    const int per = (nc + blockDim.x - 1) / blockDim.x;
    const int c0 = threadIdx.x * per;
    int local = 0;
    for (int c = c0; c < min(c0 + per, nc); ++c) local += s_units[c];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int v = wsum[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += y;
        }
        wsum[lane] = v;
    }
    __syncthreads();
    int run = incl - local + (warp > 0 ? wsum[warp - 1] : 0);
    int32_t *up = plan.unit_prefix + (int64_t)j * (nc + 1);
    for (int c = c0; c < min(c0 + per, nc); ++c) {
        up[c] = run;
        run += s_units[c];
    }
    if (threadIdx.x == 0) {
        up[nc] = wsum[31];
        plan.win_units[j] = wsum[31];
        plan.win_tiles[j] = s_tiles;
        const int ws = w * plan.W;
        const int wt = min(plan.W, plan.L - ws);
        plan.win_ncomb[j] = (wt + kCombTokens - 1) / kCombTokens;
    }
}

// One thread: queue segment starts of the windows (J+1 entries).
__global__ void plan_segments_kernel(AttendPlan plan) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    int acc = 0;
    plan.seg_start[0] = 0;
    for (int s = 0; s < plan.J; ++s) {
        acc += plan.win_units[s];
        plan.seg_start[s + 1] = acc;
    }
}

// One block per window j: writes the descriptors of its units at their queue positions.
__global__ void __launch_bounds__(256) plan_fill_kernel(const int32_t *__restrict__ hist,
                                                        const int32_t *__restrict__ chunk_off, AttendPlan plan) {
    const int s = blockIdx.x;
    const int base = plan.seg_start[s];
    const int nc = plan.nc, ntb = plan.ntb;
    {
        const int j = s;
        const int bg = j / plan.nW, w = j % plan.nW;
        const int tb0 = w * (plan.W / kInvTokBlock);
        const int tb1 = min(ntb, (w + 1) * (plan.W / kInvTokBlock));
        const int32_t *H = hist + (int64_t)bg * ntb * nc;
        const int32_t *off = chunk_off + (int64_t)bg * (nc + 1);
        const int32_t *up = plan.unit_prefix + (int64_t)j * (nc + 1);
        for (int c = threadIdx.x; c < nc; c += blockDim.x) {
            const int u0 = up[c], u1 = up[c + 1];
            if (u0 == u1) continue;
            const int e0 = off[c] + H[(int64_t)tb0 * nc + c];
            const int e1 = (tb1 < ntb) ? off[c] + H[(int64_t)tb1 * nc + c] : off[c + 1];
            const int nt = (e1 - e0 + plan.TT - 1) / plan.TT;
            for (int u = u0; u < u1; ++u) {
                const int t0 = (u - u0) * plan.unit_tiles;
                const int q = base + u;
                if (q >= plan.max_items) continue;
                plan.items[2 * q] = make_int4(0, j, c, e0);
                plan.items[2 * q + 1] = make_int4(e1, t0, min(nt, t0 + plan.unit_tiles), 0);
            }
        }
    }
}

cudaError_t launch_plan(const Shape &sh, const BwdWs &inv, const AttendPlan &plan, cudaStream_t st) {
    if (plan.J == 0) return cudaSuccess;
    const size_t smem = sizeof(int) * (size_t)sh.nc;
    cudaError_t e = set_smem_once((const void *)plan_windows_kernel, smem);
    if (e != cudaSuccess) return e;
    plan_windows_kernel<<<plan.J, 1024, smem, st>>>(inv.hist, inv.chunk_off, plan);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    plan_segments_kernel<<<1, 32, 0, st>>>(plan);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    plan_fill_kernel<<<plan.J, 256, 0, st>>>(inv.hist, inv.chunk_off, plan);
    return cudaGetLastError();
}

}  // namespace hsa
