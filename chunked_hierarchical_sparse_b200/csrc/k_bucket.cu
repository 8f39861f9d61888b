// k_bucket.cu -- token->chunk lists and work queue of the chunk-major forward.
//
// Cited page: "Hardware-aligned Hierarchical Sparse Attention for Efficient
// Long-term Memory Access" (paper notes), §kernel: the backward's second phase
// walks, for each chunk, the tokens that selected it.  The chunk-major forward
// attention uses the same inversion: per chunk, the (token, slot) pairs that
// selected it, so that one K/V tile serves many query rows.
//
// The tokens of each (b, g) are cut into windows of W tokens; window
// j = (b*h_kv + g)*nW + w.  Inside a window, the entries of chunk c form the
// bucket (j, c).  A window's tokens are processed in blocks of kCountRows.
// Three launches:
//   1. count:   per token block, a histogram over chunks (shared memory),
//               written as one row of hist[j][block][c];
//   2. scan:    one CTA per window: per chunk, the exclusive prefix of its
//               counts over the window's blocks (in place: each block's first
//               position inside the bucket), the bucket starts (an exclusive
//               scan of the bucket sizes), each bucket cut into tiles of
//               TT = 128/G tokens and tiles into work units of up to
//               unit_tiles tiles (one K/V load), the units' descriptors written
//               into the window's slice of the queue, and the window's unit,
//               tile and convert-item counts; the last CTA to finish turns the
//               unit counts into queue positions (seg_start);
//   3. scatter: per token block, shared-memory cursors start at the block's
//               positions; each (token, slot) entry takes the next position of
//               its bucket and stores t * 16 + slot and its weight there.
// Window w of (b, g) owns the fixed slice [w*W*K, (w+1)*W*K) of that (b, g)'s
// entries and the slice [j*cap, (j+1)*cap) of the queue.  Inside a bucket the
// entries of one block come in the order its shared-memory atomics land; the
// blocks are in token order.
#include "hsa_internal.cuh"

namespace hsa {

namespace {
constexpr int kCountRows = 512;  // (token, group) rows per counting block: one window, one (b, g)
}

// Block: kCountRows consecutive tokens of one (b, g), all in one window (W is a
// multiple of kCountRows or the block is the window's tail).  A thread takes
// whole (token, group) rows: their K indices arrive in two 16-byte loads, all
// issued before any of the shared-memory counts.
__global__ void __launch_bounds__(256) bucket_count_kernel(const int32_t *__restrict__ idx, AttendPlan P,
                                                           int32_t *__restrict__ hist, DevStatus *ds) {
    extern __shared__ int h_s[];  // [nc]
    const int nc = P.nc, K = P.K;
    const int blocks_per_win = (P.W + kCountRows - 1) / kCountRows;
    const int j = blockIdx.x / blocks_per_win;            // window
    const int bg = j / P.nW, w = j % P.nW;
    const int b = bg / P.hkv, g = bg % P.hkv;
    const int t0 = w * P.W + (blockIdx.x % blocks_per_win) * kCountRows;
    const int t1 = min(min(t0 + kCountRows, (w + 1) * P.W), P.L);
    for (int c = threadIdx.x; c < nc; c += blockDim.x) h_s[c] = 0;
    __syncthreads();
    constexpr int kRowsPerThread = kCountRows / 256;
    int sel[kRowsPerThread][kMaxK];
#pragma unroll
    for (int u = 0; u < kRowsPerThread; ++u) {  // all loads first
        const int t = t0 + u * 256 + threadIdx.x;
        const int32_t *row = idx + (((int64_t)b * P.L + t) * P.hkv + g) * K;
#pragma unroll
        for (int kk = 0; kk < kMaxK; ++kk) sel[u][kk] = (t < t1 && kk < K) ? row[kk] : -1;
    }
    int bad_t = -1, bad_c = 0;  // an entry that is not a causal complete chunk: skipped and reported
#pragma unroll
    for (int u = 0; u < kRowsPerThread; ++u) {
        const int t = t0 + u * 256 + threadIdx.x;
#pragma unroll
        for (int kk = 0; kk < kMaxK; ++kk) {
            const int c = sel[u][kk];
            if (c < 0) continue;  // an empty slot (or no such token / slot)
            if (c >= nc || c >= t / kChunk) {
                bad_t = t;
                bad_c = c;
                continue;
            }
            atomicAdd(&h_s[c], 1);
        }
    }
    if (bad_t >= 0) report(ds, HSA_ERR_DEVICE_CHECK, kKInvert, bad_t, bad_c);
    __syncthreads();
    int32_t *out = hist + (int64_t)blockIdx.x * nc;  // row (j, block) = blockIdx.x
    for (int c = threadIdx.x; c < nc; c += blockDim.x) out[c] = h_s[c];
}

// In-place exclusive scan of a[0..n) by one block; returns the total.
__device__ int bucket_block_scan(int *a, int n, int *wsum) {
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

// One block (1024 threads) per window j.
__global__ void __launch_bounds__(1024) bucket_scan_kernel(AttendPlan P, int32_t *__restrict__ hist) {
    extern __shared__ int sm_b[];
    int *start = sm_b;             // [nc] bucket starts within the window's slice
    int *units = sm_b + P.nc;      // [nc] work units per bucket -> their first queue slot
    int *bcnt = sm_b + 2 * P.nc;   // [nc] bucket sizes
    __shared__ int wsum[32];
    const int j = blockIdx.x, nc = P.nc, TT = P.TT, UT = P.unit_tiles;
    const int w = j % P.nW;
    const int nblk = (P.W + kCountRows - 1) / kCountRows;
    int32_t *hj = hist + (int64_t)j * nblk * nc;
    // per chunk: the bucket size (sum over the window's blocks; the loads of a
    // column are independent and all in flight together)
    for (int c = threadIdx.x; c < nc; c += blockDim.x) {
        int run = 0;
#pragma unroll 8
        for (int k = 0; k < nblk; ++k) run += __ldcg(hj + (int64_t)k * nc + c);
        bcnt[c] = run;
    }
    __syncthreads();
    int my_tiles = 0;
    for (int c = threadIdx.x; c < nc; c += blockDim.x) {
        const int n = bcnt[c];
        const int nt = (n + TT - 1) / TT;
        start[c] = n;
        units[c] = (nt + UT - 1) / UT;
        my_tiles += nt;
    }
    __syncthreads();
    bucket_block_scan(start, nc, wsum);
    const int nunits = bucket_block_scan(units, nc, wsum);
    // tiles of the window (block reduction through the shared-memory atomics)
    __shared__ int s_tiles;
    if (threadIdx.x == 0) s_tiles = 0;
    __syncthreads();
    atomicAdd(&s_tiles, my_tiles);
    const int64_t ebase = (int64_t)w * P.W * P.K;  // the window's slice of its (b, g) entries
    int4 *items = P.items + (int64_t)2 * j * P.win_cap;
    for (int c = threadIdx.x; c < nc; c += blockDim.x) {
        const int n = bcnt[c];
        const int e0 = (int)(ebase + start[c]);
        // each block's first position in the bucket: e0 + the counts of the blocks before it
        // (loads issued in groups of 8 ahead of the dependent stores)
        int run = e0;
        for (int k0 = 0; k0 < nblk; k0 += 8) {
            int v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = k0 + u < nblk ? __ldcg(hj + (int64_t)(k0 + u) * nc + c) : 0;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (k0 + u < nblk) {
                    hj[(int64_t)(k0 + u) * nc + c] = run;
                    run += v[u];
                }
        }
        if (n == 0) continue;
        const int nt = (n + TT - 1) / TT;
        for (int u = units[c], t0 = 0; t0 < nt; ++u, t0 += UT) {
            if (u >= P.win_cap) break;  // cannot happen: win_cap bounds the units of any window
            items[2 * u] = make_int4(0, j, c, e0);
            items[2 * u + 1] = make_int4(e0 + n, t0, min(nt, t0 + UT), 0);
        }
    }
    __syncthreads();
    __shared__ int s_last;
    if (threadIdx.x == 0) {
        P.win_units[j] = min(nunits, P.win_cap);
        P.win_tiles[j] = s_tiles;
        const int wt = min(P.W, P.L - w * P.W);
        P.win_ncomb[j] = (wt + kCombTokens - 1) / kCombTokens;
        // the last window to finish turns the unit counts into queue positions
        __threadfence();
        s_last = atomicAdd(&P.counters[3 * P.J], 1) == P.J - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int carry = 0;
    if (threadIdx.x == 0) P.seg_start[0] = 0;
    for (int base = 0; base < P.J; base += blockDim.x) {
        const int i = base + threadIdx.x;
        const int v = i < P.J ? __ldcg(&P.win_units[i]) : 0;
        int incl = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int x = (lane < (int)(blockDim.x >> 5)) ? wsum[lane] : 0;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, off);
                if (lane >= off) x += y;
            }
            wsum[lane] = x;
        }
        __syncthreads();
        const int pre = carry + incl + (warp > 0 ? wsum[warp - 1] : 0);
        if (i < P.J) P.seg_start[i + 1] = pre;
        carry += wsum[(blockDim.x >> 5) - 1];
        __syncthreads();
    }
}

// Block: the same kCountRows tokens as the counting block; shared-memory cursors
// start at the block's first position in each bucket.  A thread takes whole
// (token, group) rows; all loads are issued before any cursor update.
__global__ void __launch_bounds__(256) bucket_scatter_kernel(const int32_t *__restrict__ idx, const float *__restrict__ w,
                                                             AttendPlan P, const int32_t *__restrict__ hist,
                                                             int32_t *__restrict__ entries, float *__restrict__ entw) {
    extern __shared__ int cur[];  // [nc]
    const int nc = P.nc, K = P.K;
    const int blocks_per_win = (P.W + kCountRows - 1) / kCountRows;
    const int j = blockIdx.x / blocks_per_win;
    const int bg = j / P.nW, wi = j % P.nW;
    const int b = bg / P.hkv, g = bg % P.hkv;
    const int t0 = wi * P.W + (blockIdx.x % blocks_per_win) * kCountRows;
    const int t1 = min(min(t0 + kCountRows, (wi + 1) * P.W), P.L);
    const int32_t *hrow = hist + (int64_t)blockIdx.x * nc;
    for (int c = threadIdx.x; c < nc; c += blockDim.x) cur[c] = hrow[c];
    constexpr int kRowsPerThread = kCountRows / 256;
    int sel[kRowsPerThread][kMaxK];
    float wt[kRowsPerThread][kMaxK];
#pragma unroll
    for (int u = 0; u < kRowsPerThread; ++u) {
        const int t = t0 + u * 256 + threadIdx.x;
        const int64_t row = (((int64_t)b * P.L + t) * P.hkv + g) * K;
#pragma unroll
        for (int kk = 0; kk < kMaxK; ++kk) {
            const bool in = t < t1 && kk < K;
            sel[u][kk] = in ? idx[row + kk] : -1;
            wt[u][kk] = in ? w[row + kk] : 0.f;
        }
    }
    __syncthreads();
    const int64_t ebase = (int64_t)bg * P.ent_stride;  // the (b, g) entries
#pragma unroll
    for (int u = 0; u < kRowsPerThread; ++u) {
        const int t = t0 + u * 256 + threadIdx.x;
#pragma unroll
        for (int kk = 0; kk < kMaxK; ++kk) {
            const int c = sel[u][kk];
            if (c < 0 || c >= nc || c >= t / kChunk) continue;  // empty, or reported by the count
            const int pos = atomicAdd(&cur[c], 1);
            entries[ebase + pos] = t * 16 + kk;
            entw[ebase + pos] = wt[u][kk];
        }
    }
}

cudaError_t launch_bucket_plan(const Shape &sh, const int32_t *idx, const float *w, const AttendPlan &P,
                               int32_t *hist, int32_t *entries, float *entw, DevStatus *ds, cudaStream_t st) {
    if (P.J == 0) return cudaSuccess;
    cudaError_t e;
    const size_t hsmem = sizeof(int) * (size_t)sh.nc;
    if ((e = set_smem_once((const void *)bucket_count_kernel, hsmem)) != cudaSuccess) return e;
    if ((e = set_smem_once((const void *)bucket_scan_kernel, 3 * hsmem)) != cudaSuccess) return e;
    if ((e = set_smem_once((const void *)bucket_scatter_kernel, hsmem)) != cudaSuccess) return e;
    const int blocks = P.J * ((P.W + kCountRows - 1) / kCountRows);
    if (sh.nc > 0) {
        bucket_count_kernel<<<blocks, 256, hsmem, st>>>(idx, P, hist, ds);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    bucket_scan_kernel<<<P.J, 1024, 3 * hsmem, st>>>(P, hist);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (sh.nc > 0) {
        bucket_scatter_kernel<<<blocks, 256, hsmem, st>>>(idx, w, P, hist, entries, entw);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

size_t bucket_hist_elems(const AttendPlan &P) {
    return (size_t)P.J * ((P.W + kCountRows - 1) / kCountRows) * P.nc;
}

}  // namespace hsa
