// topk_warp.cuh -- one warp keeps a running top-K over streamed chunk scores.
//
// Order (the pages leave ties open; this library breaks them toward the more
// recent chunk): (s1, c1) beats (s2, c2) iff s1 > s2, or s1 == s2 and c1 > c2.
// The running list lives in lanes 0..K-1 (one entry per lane); empty entries
// are (-inf, -1) and lose to any real candidate.
#pragma once

#include <cuda_runtime.h>
#include <math_constants.h>

namespace hsa {

__device__ __forceinline__ bool beats(float s1, int c1, float s2, int c2) {
    return s1 > s2 || (s1 == s2 && c1 > c2);
}

// Warp argmax (better = beats) of (s, c, lane); every lane receives the winner.
__device__ __forceinline__ void warp_best(float &s, int &c, int &lane_of) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float so = __shfl_xor_sync(0xffffffffu, s, off);
        const int co = __shfl_xor_sync(0xffffffffu, c, off);
        const int lo = __shfl_xor_sync(0xffffffffu, lane_of, off);
        if (beats(so, co, s, c) || (so == s && co == c && lo < lane_of)) {
            s = so; c = co; lane_of = lo;
        }
    }
}

// Warp argmin (worse = beaten by the other).
__device__ __forceinline__ void warp_worst(float &s, int &c, int &lane_of) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float so = __shfl_xor_sync(0xffffffffu, s, off);
        const int co = __shfl_xor_sync(0xffffffffu, c, off);
        const int lo = __shfl_xor_sync(0xffffffffu, lane_of, off);
        if (beats(s, c, so, co) || (so == s && co == c && lo < lane_of)) {
            s = so; c = co; lane_of = lo;
        }
    }
}

// Merge up to 64 candidates (two per lane: (sa, ca) and (sb, cb); a candidate
// with c < 0 is absent) into the list held in lanes < K as (ls, lc).
__device__ __forceinline__ void topk_merge(int K, float sa, int ca, float sb, int cb, float &ls,
                                           int &lc) {
    const int lane = threadIdx.x & 31;
    bool va = ca >= 0, vb = cb >= 0;
    for (int iter = 0; iter < 64; ++iter) {
        // worst entry of the list (lanes >= K never count)
        float ws = (lane < K) ? ls : CUDART_INF_F;
        int wc = (lane < K) ? lc : 0x7fffffff;
        int wl = lane;
        warp_worst(ws, wc, wl);
        const bool pa = va && beats(sa, ca, ws, wc);
        const bool pb = vb && beats(sb, cb, ws, wc);
        if (!__any_sync(0xffffffffu, pa || pb)) break;
        // best surviving candidate
        float bs = -CUDART_INF_F;
        int bc = -1, which = 0;
        if (pa) { bs = sa; bc = ca; which = 1; }
        if (pb && (!pa || beats(sb, cb, sa, ca))) { bs = sb; bc = cb; which = 2; }
        int bl = (which ? lane : 64);
        if (!which) { bs = -CUDART_INF_F; bc = -2; }
        warp_best(bs, bc, bl);
        if (lane == wl) { ls = bs; lc = bc; }
        if (lane == bl) {
            if (bc == ca) va = false;
            else vb = false;
        }
    }
}

// Final step for one row: the list (lanes < K) is reordered most-recent-first
// (descending chunk index) and the stick-breaking weights are formed:
//   w_r = sig(s_r) * prod_{j<r} (1 - sig(s_j)).
// Lane r < K receives slot r's (chunk, weight, score); empty slots get
// (-1, 0, 0).
__device__ __forceinline__ void topk_finish(int K, float ls, int lc, int &slot_c, float &slot_w,
                                            float &slot_s) {
    const int lane = threadIdx.x & 31;
    const bool valid = lane < K && lc >= 0;
    const unsigned vmask = __ballot_sync(0xffffffffu, valid);
    const int n_sel = __popc(vmask);
    // rank among valid entries by descending chunk index
    int rank = 0;
    for (int j = 0; j < K; ++j) {
        const int cj = __shfl_sync(0xffffffffu, lc, j);
        const bool vj = (vmask >> j) & 1u;
        if (valid && vj && cj > lc) ++rank;
    }
    const float sg = valid ? 1.0f / (1.0f + expf(-ls)) : 0.0f;
    // gather (chunk, sig, score) into slot order: slot r pulls the entry of rank r
    slot_c = -1; slot_w = 0.0f; slot_s = 0.0f;
    float keep = 1.0f;  // prod_{j<r} (1 - sig_j)
    for (int r = 0; r < n_sel; ++r) {
        const unsigned who = __ballot_sync(0xffffffffu, valid && rank == r);
        const int src = __ffs(who) - 1;
        const float sr = __shfl_sync(0xffffffffu, sg, src);
        const int cr = __shfl_sync(0xffffffffu, lc, src);
        const float scr = __shfl_sync(0xffffffffu, ls, src);
        if (lane == r) { slot_c = cr; slot_w = sr * keep; slot_s = scr; }
        keep *= (1.0f - sr);
    }
}

}  // namespace hsa
