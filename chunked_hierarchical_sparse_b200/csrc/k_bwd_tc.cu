// k_bwd_tc.cu -- the backward pass, chunk-major, on the 5th-generation tensor
// cores (tcgen05 + TMEM + TMA), persistent and warp-specialised.
//
// Cited page: "Hardware-aligned Hierarchical Sparse Attention for Efficient
// Long-term Memory Access" (paper notes), §kernel: the backward is split into
// a per-token phase (the gradients of the queries and of the chunk weights)
// and a per-chunk phase (the gradients of the keys and values, over the
// inverted token lists).  Both phases need the same recomputed probabilities,
// so here they run as one chunk-major pass over the forward's work plan: a
// tile holds TT = 128/G tokens that selected chunk c, with the G query heads
// of each token as rows.  Per tile (x = S/sqrt(d), p = exp(x - lse)):
//   S  = Q K_c^T,  dP = dO V_c^T                 (tcgen05, fp32 in TMEM)
//   Delta = rowsum(p * dP)   (= dO . O_k, since O_k = sum_i p_i v_i)
//   dS = w p (dP - Delta),  wP = w p            (bf16 into SMEM)
//   dQ  = dS K_c              -> fp32 reduce-add into the window's dq slot
//   dK^T += Q^T dS,  dV^T += dO^T wP            (accumulated in TMEM over a
//                                               work unit, then reduce-added)
//   dw[t, slot] = sum over the token's G rows of Delta
// The window slots are converted to dq (times 1/sqrt(d)) and re-zeroed by a
// convert step, as in the forward.  The stick-breaking backward (dw -> dq_slc,
// dkbar) and the mean-pool path run afterwards on CUDA cores.
//
// Roles (12 warps): warps 0-3 gradient core, warps 4-7 dQ epilogue and the
// dK/dV flush, warps 8-9 convert step, warp 10 producer (TMA), warp 11 MMA
// issuer.  Every wait is bounded; on expiry the kernel records HSA_ERR_TIMEOUT
// and returns.
//
// Head dims 128 and 64.  For d = 64 every MMA keeps M = 128: a tile's Q and dO
// rows share one buffer, each 8-row group holding its Q rows then its dO rows,
// which is the d = 128 layout of Q with dO in place of the second 64-column
// half.  Read as an MN-major operand of 128 rows that buffer is [Q^T; dO^T], so
//   [Q^T; dO^T] dS = [dK^T; dO^T dS]   (TMEM lanes 0-63 hold dK^T)
//   [Q^T; dO^T] wP = [Q^T wP; dV^T]    (TMEM lanes 64-127 hold dV^T)
// and the flush reads the lanes that hold the gradients.
#include <algorithm>

#include "hsa_internal.cuh"
#include "sm100.cuh"

namespace hsa {

using namespace sm100;


namespace {


// unrolling of the epilogue's column loops: rolled, the roles' hot code fits the instruction cache
constexpr int kBEpiUnroll = 1;

constexpr int kBThreads = 384;
constexpr int kBWarpEpi = 4, kBWarpConv = 8, kBWarpProd = 10, kBWarpMma = 11;
constexpr int kBConvThreads = 64;
constexpr int kBInfo = 8;  // tile-info ring entries
constexpr int kBItemTile = 0, kBItemEnd = 2;

struct BTileInfo {
    int type;
    int j;        // window
    int b, g, c;  // sequence, group, chunk
    int ntok;     // valid tokens in the tile
    int kvph, useq, unit_first, unit_last;
    int qs, qph;
    int tok[16];
    int slot[16];
    float w[16];  // stick-breaking weight of each token's slot
};

template <int D> struct BSmem {
    // d = 128: a 128-row Q (or dO) tile is 16 groups of 8 rows, each group's two 64-column
    // halves one after the other (1 KB each), so one TMA box loads a group.
    // d = 64: one 32 KB buffer per stage holds the Q and the dO rows of a tile, each
    // group's Q rows (1 KB) then its dO rows (1 KB).
    static constexpr bool kStack = D == 64;
    static constexpr int QHALF = 128 * 128;  // bytes of one 64-column half of a 128-row tile
    static constexpr int QBYTES = 2 * QHALF;
    static constexpr int NQBUF = kStack ? 2 : 4;  // 32 KB buffers: [2] Q and [2] dO, or [2] Q|dO
    static constexpr int KVHALF = 64 * 128;
    static constexpr int KVBYTES = (D / 64) * KVHALF;
    static constexpr int PB = 128 * 128;     // 128 rows x 64 keys bf16
    static constexpr int OFF_Q = 0;                      // [2] query tiles
    static constexpr int OFF_DO = kStack ? OFF_Q + 1024 : OFF_Q + 2 * QBYTES;  // [2] output-gradient tiles
    static constexpr int OFF_K = OFF_Q + NQBUF * QBYTES;
    static constexpr int OFF_V = OFF_K + KVBYTES;
    static constexpr int OFF_DS = OFF_V + KVBYTES;       // dS (bf16, swizzled rows)
    static constexpr int OFF_WP = OFF_DS + PB;           // w p (bf16, swizzled rows)
    static constexpr int OFF_X = OFF_WP + PB;            // epilogue transpose scratch, 4 KB per warp
    static constexpr int OFF_INFO = OFF_X + 4 * 4096;
    static constexpr int OFF_BAR = OFF_INFO + kBInfo * (int)sizeof(BTileInfo);
    static constexpr int NBAR = 2 * kBInfo + 2 * 2 + 2 + 2 * 2 + 2 + 2 + 2 + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_MISC + 64;
    static constexpr int ALLOC = BYTES + 1024;  // slack for 1 KB alignment
};
static_assert(BSmem<128>::ALLOC <= 227 * 1024, "backward tile buffers exceed the shared memory of a CTA");

// TMEM columns: S 0..63, dP 64..127, dQ[2] 128..383, dK^T 384..447, dV^T 448..511 (the gradient
// warps copy S and dP out at once, so one buffer each; the dQ drain overlaps the next dQ)
constexpr uint32_t kColS = 0, kColDP = 64, kColDQ = 128, kColDK = 384, kColDV = 448;

__device__ __forceinline__ float bex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ int bld_acquire(const int32_t *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// bounded spin until *p >= target; false on timeout or once *abort is set
__device__ bool bspin_geq(const int32_t *p, int target, volatile int *abort, uint64_t wait_ns) {
    if (bld_acquire(p) >= target) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
        __nanosleep(256);
        if (bld_acquire(p) >= target) return true;
        if (*abort) return false;
        if (globaltimer() - t0 > wait_ns) return false;
    }
}

// 8 floats -> 8 bf16 packed in 16 bytes
__device__ __forceinline__ uint4 pack8(const float *f) {
    __nv_bfloat162 a0 = __floats2bfloat162_rn(f[0], f[1]);
    __nv_bfloat162 a1 = __floats2bfloat162_rn(f[2], f[3]);
    __nv_bfloat162 a2 = __floats2bfloat162_rn(f[4], f[5]);
    __nv_bfloat162 a3 = __floats2bfloat162_rn(f[6], f[7]);
    uint4 pk;
    pk.x = *reinterpret_cast<uint32_t *>(&a0); pk.y = *reinterpret_cast<uint32_t *>(&a1);
    pk.z = *reinterpret_cast<uint32_t *>(&a2); pk.w = *reinterpret_cast<uint32_t *>(&a3);
    return pk;
}

}  // namespace

template <int G, int D>
__global__ void __launch_bounds__(kBThreads, 1) bwd_tc_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    const __grid_constant__ AttendPlan P, const int32_t *__restrict__ entries, const float *__restrict__ entw,
    const float *__restrict__ lse, float *__restrict__ dw, __half *__restrict__ acc, __nv_bfloat16 *__restrict__ dq,
    float *__restrict__ dk_acc, float *__restrict__ dv_acc, DevStatus *ds, uint64_t wait_ns) {
    using L = BSmem<D>;
    constexpr int TT = 128 / G;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    BTileInfo *info = reinterpret_cast<BTileInfo *>(sm + L::OFF_INFO);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L::OFF_BAR);
    uint64_t *info_full = bar, *info_empty = bar + kBInfo;
    uint64_t *qd_full = bar + 2 * kBInfo, *qd_empty = qd_full + 2;  // [2] Q + dO tiles
    uint64_t *kv_full = qd_empty + 2, *kv_empty = kv_full + 1;      // the unit's K/V
    uint64_t *sd_full = kv_empty + 1, *sd_empty = sd_full + 1;      // S and dP in TMEM
    uint64_t *ds_full = sd_empty + 1, *ds_empty = ds_full + 1;      // dS / wP in SMEM
    uint64_t *dq_full = ds_empty + 1, *dq_empty = dq_full + 2;      // [2] dQ in TMEM
    uint64_t *dkv_full = dq_empty + 2, *dkv_empty = dkv_full + 1;   // dK^T / dV^T in TMEM
    uint64_t *mma_done = dkv_empty + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::OFF_MISC + 16);
    volatile int *eg_flag = reinterpret_cast<volatile int *>(sm + L::OFF_MISC + 40);  // [2] epilogue group
    volatile int *cg_flag = reinterpret_cast<volatile int *>(sm + L::OFF_MISC + 48);  // [2] convert group

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kBInfo; ++i) { mbar_init(&info_full[i], 1); mbar_init(&info_empty[i], 2); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&qd_full[i], 1); mbar_init(&qd_empty[i], 1);
            mbar_init(&dq_full[i], 1); mbar_init(&dq_empty[i], 4);
        }
        mbar_init(kv_full, 1); mbar_init(kv_empty, 1);
        mbar_init(ds_full, 4); mbar_init(ds_empty, 1);
        mbar_init(sd_full, 1); mbar_init(sd_empty, 4);
        mbar_init(dkv_full, 1); mbar_init(dkv_empty, 4);
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    // Q / dO rows of a ragged tile's missing tokens are never loaded; dK^T and dV^T
    // contract over all 128 rows, so the buffers start at zero and only ever hold
    // finite input rows afterwards (their dS / wP rows are zero).
    for (int e = threadIdx.x; e < L::NQBUF * L::QBYTES / 16; e += kBThreads)
        reinterpret_cast<uint4 *>(sm + L::OFF_Q)[e] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
    if (warp == kBWarpMma) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    if (warp == kBWarpProd && lane == 0) {
        prefetch_tmap(&tm_q); prefetch_tmap(&tm_do); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    int32_t *tiles_done = P.counters;
    int32_t *comb_done = P.counters + P.J;
    int32_t *comb_head = P.counters + 2 * P.J;
    const float scale = 1.0f / sqrtf((float)D);
    // power-of-two scale of the fp16 dq accumulators: 2^e >= 2 max||v_row|| max||dO_row|| max|k| / sqrt(d),
    // a bound of every partial dq sum (|dS_i| <= 2 w p_i ||dO|| max||v||, sum_i p_i < 1, sum_k w_k <= 1)
    float acc_scale, acc_inv;
    {
        const float nv = __int_as_float(P.counters[3 * P.J + 1]);
        const float ndo = __int_as_float(P.counters[3 * P.J + 2]);
        const float mk = __int_as_float(P.counters[3 * P.J + 3]);
        const float bound = 2.f * nv * ndo * mk * scale;
        int ev = 0;
        if (bound > 0.f) {
            const uint32_t vb = __float_as_uint(bound);
            ev = (int)((vb >> 23) & 0xff) - 127;
            if (vb & 0x7fffffu) ev += 1;
        }
        ev = max(-100, min(ev, 120));
        acc_scale = __int_as_float((ev + 127) << 23);
        acc_inv = __int_as_float((127 - ev) << 23);
    }

    auto warp_wait = [&](uint64_t *b, uint32_t par) -> bool {  // every lane waits; the warp decides by a vote
        return __all_sync(0xffffffffu, mbar_wait(b, par, wait_ns));
    };

    if (warp == kBWarpProd) {
        // ============================================================ producer
        // Units (whole (window, chunk) buckets) are dealt to the CTAs in queue
        // order; descriptors are loaded one unit ahead and each tile's entries
        // and weights one tile ahead.
        int it = 0, qc = 0, useq = 0;
        bool ok = true;
        const int total = min(P.seg_start[P.J], P.max_items);
        const int qstep = gridDim.x;
        int guard_ok_j = -1;
        struct Desc { int4 a, b; };
        auto load_desc = [&](int q) -> Desc {
            Desc d;
            if (q < total) { d.a = P.items[2 * q]; d.b = P.items[2 * q + 1]; }
            else { d.a = make_int4(kBItemEnd, 0, 0, 0); d.b = make_int4(0, 0, 0, 0); }
            return d;
        };
        struct Pay { int e; float w; };  // entry and weight of token `lane` of a tile
        auto tile_pay = [&](const Desc &d, int tt) -> Pay {
            Pay p{0, 0.f};
            if (d.a.x == kBItemTile) {
                const int64_t base = (int64_t)(d.a.y / P.nW) * P.L * P.K;
                const int ub = d.a.w + tt * TT;
                if (lane < min(TT, d.b.x - ub)) { p.e = entries[base + ub + lane]; p.w = entw[base + ub + lane]; }
            }
            return p;
        };
        int qn = blockIdx.x;
        Desc dc = load_desc(qn), dn = load_desc(qn + qstep);
        Pay pc = tile_pay(dc, dc.b.y);
        while (ok) {
            if (*abort_flag) { ok = false; break; }
            const int type = dc.a.x, j = dc.a.y, c = dc.a.z, e0 = dc.a.w;
            const int e1 = dc.b.x, t0 = dc.b.y, t1 = dc.b.z;
            if (type == kBItemEnd) {
                const int ii = it % kBInfo;
                if (it >= kBInfo && !warp_wait(&info_empty[ii], ((it / kBInfo) - 1) & 1)) { ok = false; break; }
                if (lane == 0) {
                    info[ii].type = kBItemEnd;
                    mbar_arrive(&info_full[ii]);
                }
                break;
            }
            const int bg = j / P.nW;
            const int b = bg / P.hkv, g = bg % P.hkv;
            // ring guard: window j's dq slot was last used by window j - kRing
            if (j >= kRing && j > guard_ok_j) {
                int g_ok = 1;
                if (lane == 0) g_ok = bspin_geq(&comb_done[j - kRing], P.win_ncomb[j - kRing], abort_flag, wait_ns) ? 1 : 0;
                if (!__shfl_sync(0xffffffffu, g_ok, 0)) {
                    if (lane == 0 && !*abort_flag) report(ds, HSA_ERR_TIMEOUT, kKBwdTc, 1, j);
                    ok = false;
                    break;
                }
                guard_ok_j = j;
            }
            // K/V of chunk c (single buffer: free once the previous unit's last dQ is done)
            if (useq >= 1 && !warp_wait(kv_empty, (useq - 1) & 1)) { ok = false; break; }
            if (lane == 0) {
                mbar_arrive_expect_tx(kv_full, 2 * L::KVBYTES);
                const int row = bg * P.L + c * kChunk;
#pragma unroll
                for (int h = 0; h < D / 64; ++h) {
                    tma_load_2d(sm + L::OFF_K + h * L::KVHALF, &tm_k, h * 64, row, kv_full);
                    tma_load_2d(sm + L::OFF_V + h * L::KVHALF, &tm_v, h * 64, row, kv_full);
                }
            }
            for (int tt = t0; tt < t1 && ok; ++tt) {
                const Pay pn = (tt + 1 < t1) ? tile_pay(dc, tt + 1) : tile_pay(dn, dn.b.y);
                const int ii = it % kBInfo;
                if (it >= kBInfo && !warp_wait(&info_empty[ii], ((it / kBInfo) - 1) & 1)) { ok = false; break; }
                const int qs = qc & 1, qph = (qc >> 1) & 1;
                if (qc >= 2 && !warp_wait(&qd_empty[qs], ((qc >> 1) - 1) & 1)) { ok = false; break; }
                BTileInfo &ti_ = info[ii];
                const int ntok = min(TT, e1 - (e0 + tt * TT));
                int t = pc.e >> 4, slot = pc.e & 15;
                {  // an entry outside its window (inconsistent lists) is reported and made harmless
                    const int wsv = (j % P.nW) * P.W;
                    const bool bad = lane < ntok && (t < wsv || t >= min(P.L, wsv + P.W) || slot >= P.K);
                    if (bad) { report(ds, HSA_ERR_DEVICE_CHECK, kKBwdTc, t, c); t = wsv; slot = 0; }
                    if (lane < 16) {
                        ti_.tok[lane] = (lane < ntok) ? t : -1;
                        ti_.slot[lane] = (lane < ntok) ? slot : 0;
                        ti_.w[lane] = (lane < ntok && !bad) ? pc.w : 0.f;
                    }
                }
                if (lane == 0) {
                    ti_.type = kBItemTile; ti_.j = j; ti_.b = b; ti_.g = g; ti_.c = c; ti_.ntok = ntok;
                    ti_.kvph = useq & 1; ti_.useq = useq;
                    ti_.unit_first = (tt == t0); ti_.unit_last = (tt == t1 - 1);
                    ti_.qs = qs; ti_.qph = qph;
                    mbar_arrive_expect_tx(&qd_full[qs], 2 * ntok * G * D * 2);  // Q and dO rows, bf16
                }
                __syncwarp();
                {  // per 8-row group: d = 128, one 3D box (both 64-column halves, 2 KB) for Q and
                   // for dO; d = 64, one 2D box (1 KB) each, side by side in the group's 2 KB
                    constexpr int GPT = G / 8;  // 8-row groups per token
                    const int tq = __shfl_sync(0xffffffffu, t, lane / GPT);
                    if (lane < ntok * GPT) {
                        const int row = (b * P.L + tq) * P.hq + g * G + (lane % GPT) * 8;
                        if constexpr (D == 128) {
                            tma_load_3d(sm + L::OFF_Q + qs * L::QBYTES + lane * 2048, &tm_q, 0, row, 0, &qd_full[qs]);
                            tma_load_3d(sm + L::OFF_DO + qs * L::QBYTES + lane * 2048, &tm_do, 0, row, 0, &qd_full[qs]);
                        } else {
                            tma_load_2d(sm + L::OFF_Q + qs * L::QBYTES + lane * 2048, &tm_q, 0, row, &qd_full[qs]);
                            tma_load_2d(sm + L::OFF_DO + qs * L::QBYTES + lane * 2048, &tm_do, 0, row, &qd_full[qs]);
                        }
                    }
                }
                __syncwarp();
                mbar_arrive_lane0(&info_full[ii], lane);
                pc = pn;
                ++qc;
                ++it;
            }
            if (!ok) break;
            dc = dn;
            dn = load_desc(qn + 2 * qstep);
            qn += qstep;
            ++useq;
        }
        if (!ok) {
            *abort_flag = 1;
            if (lane == 0) {
                report(ds, HSA_ERR_TIMEOUT, kKBwdTc, 2, it);
                // let the loads already issued land before the CTA goes away (bounded)
                for (int s2 = 0; s2 < 2; ++s2)
                    if (qc > s2) mbar_wait(&qd_full[(qc - 1 - s2) & 1], ((qc - 1 - s2) >> 1) & 1, kDrainWaitNs);
                if (useq > 0) mbar_wait(kv_full, (useq - 1) & 1, kDrainWaitNs);
            }
            __syncwarp();
        }
    } else if (warp == kBWarpMma) {
        // ============================================================ MMA issuer
        // Two in-order streams polled by one lane:
        //   scores:    S = Q K^T and dP = dO V^T of tile ts (needs Q, dO, K, V and a free S/dP buffer)
        //   gradients: dQ = dS K, dK^T += Q^T dS, dV^T += dO^T wP of tile tg (needs dS / wP, a free
        //              dQ buffer and, at a unit's first tile, the previous unit's dK/dV flushed)
        // dK^T / dV^T have M = 128: the d = 128 rows of Q^T / dO^T, or for d = 64 the stacked
        // [Q^T; dO^T] of the shared buffer (both MMAs read it; see the file comment)
        constexpr uint32_t id_s = idesc_bf16_f32(128, 64, false, false);
        constexpr uint32_t id_dq = idesc_bf16_f32(128, D, false, true);
        constexpr uint32_t id_dkv = idesc_bf16_f32(128, 64, true, true);
        bool ok = true;
        int ts = 0, tg = 0;
        if (lane == 0) {
            bool s_done = false;
            uint64_t t_last = globaltimer();
            while (true) {
                bool prog = false;
                if (!s_done) {
                    const int ii = ts % kBInfo;
                    if (mbar_test(&info_full[ii], (ts / kBInfo) & 1)) {
                        const BTileInfo &inf = info[ii];
                        if (inf.type == kBItemEnd) {
                            s_done = true;
                            prog = true;
                        } else if ((!inf.unit_first || mbar_test(kv_full, inf.kvph)) &&
                                   mbar_test(&qd_full[inf.qs], inf.qph) &&
                                   (ts < 1 || mbar_test(sd_empty, (ts - 1) & 1))) {
                            tc_fence_after();
                            const uint32_t qa = smem_u32(sm + L::OFF_Q + inf.qs * L::QBYTES);
                            const uint32_t oa = smem_u32(sm + L::OFF_DO + inf.qs * L::QBYTES);
                            const uint32_t kb = smem_u32(sm + L::OFF_K);
                            const uint32_t vb = smem_u32(sm + L::OFF_V);
#pragma unroll
                            for (int ks = 0; ks < D / 16; ++ks) {
                                const int h = ks >> 2, kk = ks & 3;
                                mma_bf16_ss(tmem + kColS, smem_desc_sw128(qa + h * 1024 + kk * 32, 16, 2048),
                                            smem_desc_sw128(kb + h * L::KVHALF + kk * 32, 16, 1024), id_s, ks > 0);
                            }
#pragma unroll
                            for (int ks = 0; ks < D / 16; ++ks) {
                                const int h = ks >> 2, kk = ks & 3;
                                mma_bf16_ss(tmem + kColDP, smem_desc_sw128(oa + h * 1024 + kk * 32, 16, 2048),
                                            smem_desc_sw128(vb + h * L::KVHALF + kk * 32, 16, 1024), id_s, ks > 0);
                            }
                            mma_commit(sd_full);
                            ++ts;
                            prog = true;
                        }
                    }
                }
                if (tg < ts) {
                    const int ii = tg % kBInfo;
                    const BTileInfo &inf = info[ii];
                    const int qb = tg & 1;  // dQ buffer
                    if (mbar_test(ds_full, tg & 1) && (tg < 2 || mbar_test(&dq_empty[qb], ((tg >> 1) - 1) & 1)) &&
                        (!inf.unit_first || inf.useq < 1 || mbar_test(dkv_empty, (inf.useq - 1) & 1))) {
                        tc_fence_after();
                        const uint32_t qa = smem_u32(sm + L::OFF_Q + inf.qs * L::QBYTES);
                        const uint32_t oa = L::kStack ? qa : smem_u32(sm + L::OFF_DO + inf.qs * L::QBYTES);
                        const uint32_t kb = smem_u32(sm + L::OFF_K);
                        const uint32_t dsa = smem_u32(sm + L::OFF_DS);
                        const uint32_t wpa = smem_u32(sm + L::OFF_WP);
                        // dQ = dS K  (K = the chunk's 64 keys)
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            mma_bf16_ss(tmem + kColDQ + qb * 128, smem_desc_sw128(dsa + ks * 32, 16, 1024),
                                        smem_desc_sw128(kb + ks * 2048, L::KVHALF, 1024), id_dq, ks > 0);
                        mma_commit(&dq_full[qb]);
                        // dK^T += Q^T dS,  dV^T += dO^T wP  (K = the tile's 128 rows)
                        const bool first = inf.unit_first != 0;
#pragma unroll
                        for (int ks = 0; ks < 8; ++ks)
                            mma_bf16_ss(tmem + kColDK, smem_desc_sw128(qa + ks * 4096, 1024, 2048),
                                        smem_desc_sw128(dsa + ks * 2048, L::PB, 1024), id_dkv, ks > 0 || !first);
#pragma unroll
                        for (int ks = 0; ks < 8; ++ks)
                            mma_bf16_ss(tmem + kColDV, smem_desc_sw128(oa + ks * 4096, 1024, 2048),
                                        smem_desc_sw128(wpa + ks * 2048, L::PB, 1024), id_dkv, ks > 0 || !first);
                        mma_commit(ds_empty);
                        mma_commit(&qd_empty[inf.qs]);
                        if (inf.unit_last) {
                            mma_commit(kv_empty);
                            mma_commit(dkv_full);
                        }
                        mbar_arrive(&info_empty[ii]);
                        ++tg;
                        prog = true;
                    }
                } else if (s_done) {
                    break;
                }
                if (prog) {
                    t_last = globaltimer();
                } else {
                    if (*abort_flag || globaltimer() - t_last > wait_ns) { ok = false; break; }
                    __nanosleep(32);  // leave the issue slots to the working warps meanwhile
                }
            }
            if (!ok) {
                *abort_flag = 1;
                report(ds, HSA_ERR_TIMEOUT, kKBwdTc, 3, ts);
            }
            // drain: every MMA issued by this warp has finished before TMEM is released
            mma_commit(mma_done);
            mbar_wait(mma_done, 0, kDrainWaitNs);
        }
        __syncwarp();
    } else if (warp < kBWarpEpi) {
        // ============================================================ gradient core
        const int wq = warp & 3;                 // TMEM lane quadrant of this warp
        const int r = wq * 32 + lane;            // tile row = token * G + head
        const int tid = threadIdx.x;             // 0..127
        const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
        const float L2E = 1.4426950408889634f;
        const float sl2 = scale * L2E;
        int it = 0;
        bool ok = true;
        // every warp of the group waits for itself (converged, sleeping in try_wait);
        // the warps only meet at the mbarriers they arrive on
        auto wg_wait = [&](uint64_t *b, uint32_t par) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(b, par, wait_ns));
        };
        while (ok) {
            const int ii = it % kBInfo;
            if (!wg_wait(&info_full[ii], (it / kBInfo) & 1)) { ok = false; break; }
            const BTileInfo &inf = info[ii];
            if (inf.type == kBItemEnd) break;
            const int ti = r / G, hh = r % G;
            const bool valid = ti < inf.ntok;
            const int t = valid ? inf.tok[ti] : 0, slot = valid ? inf.slot[ti] : 0;
            const float wk = valid ? inf.w[ti] : 0.f;
            // the row's log-normaliser from the forward, loaded before the scores are waited for
            const float lrow =
                valid ? lse[(((int64_t)inf.b * P.L + t) * P.hq + inf.g * G + hh) * P.K + slot] : 0.f;
            if (!wg_wait(sd_full, it & 1)) { ok = false; break; }
            tc_fence_after();
            float x0[32], x1[32], d0[32], d1[32];
            tmem_ld32(lane_base + kColS, x0);
            tmem_ld32(lane_base + kColS + 32, x1);
            tmem_ld32(lane_base + kColDP, d0);
            tmem_ld32(lane_base + kColDP + 32, d1);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            mbar_arrive_lane0(sd_empty, lane);
            float delta = 0.f;
            if (valid) {
                // p = exp(x - lse), x = S / sqrt(d);  Delta = sum_i p_i dP_i
                const float lb = lrow * L2E;
                float dl[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    x0[i] = bex2(fmaf(x0[i], sl2, -lb));
                    x0[i + 1] = bex2(fmaf(x0[i + 1], sl2, -lb));
                    x1[i] = bex2(fmaf(x1[i], sl2, -lb));
                    x1[i + 1] = bex2(fmaf(x1[i + 1], sl2, -lb));
                    dl[0] = fmaf(x0[i], d0[i], dl[0]);
                    dl[1] = fmaf(x0[i + 1], d0[i + 1], dl[1]);
                    dl[2] = fmaf(x1[i], d1[i], dl[2]);
                    dl[3] = fmaf(x1[i + 1], d1[i + 1], dl[3]);
                }
                delta = (dl[0] + dl[1]) + (dl[2] + dl[3]);
                // dS = w p (dP - Delta) into d, wP = w p into x
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    d0[i] = wk * x0[i] * (d0[i] - delta);
                    d1[i] = wk * x1[i] * (d1[i] - delta);
                    x0[i] *= wk;
                    x1[i] *= wk;
                }
            }
            // dw[t, slot] = sum of Delta over the token's G rows (G consecutive lanes)
            float dsum = delta;
#pragma unroll
            for (int off = 1; off < G; off <<= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
            if (valid && hh == 0) dw[(((int64_t)inf.b * P.L + t) * P.hkv + inf.g) * P.K + slot] = dsum;
            // the dS / wP buffer is free once the previous tile's gradient MMAs have read it
            if (it >= 1 && !wg_wait(ds_empty, (it - 1) & 1)) { ok = false; break; }
            uint8_t *dsrow = sm + L::OFF_DS + r * 128;
            uint8_t *wprow = sm + L::OFF_WP + r * 128;
            if (valid) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const int sw = (ch ^ (r & 7)) << 4;
                    *reinterpret_cast<uint4 *>(dsrow + sw) = pack8((ch < 4) ? (d0 + ch * 8) : (d1 + (ch - 4) * 8));
                    *reinterpret_cast<uint4 *>(wprow + sw) = pack8((ch < 4) ? (x0 + ch * 8) : (x1 + (ch - 4) * 8));
                }
            } else {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    *reinterpret_cast<uint4 *>(dsrow + (ch << 4)) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4 *>(wprow + (ch << 4)) = make_uint4(0, 0, 0, 0);
                }
            }
            fence_proxy_async_smem();  // each writer orders its dS / wP rows before the MMA's reads
            __syncwarp();
            mbar_arrive_lane0(ds_full, lane);  // one arrival per warp
            ++it;
        }
        if (!ok) { *abort_flag = 1; if (tid == 0) report(ds, HSA_ERR_TIMEOUT, kKBwdTc, 5, it); }
    } else if (warp < kBWarpConv) {
        // ============================================================ dQ epilogue + dK/dV flush
        // dQ rows (times 1/sqrt(d)) are transposed through a 4 KB per-warp
        // scratch so each warp-wide vector reduction covers four whole 128-byte
        // lines of the window's dq slot.  At a unit's last tile, dK^T and dV^T
        // (TMEM lane = column of d, TMEM column = key of the chunk) are reduce-
        // added into the fp32 dk / dv accumulators, one 128-byte line per warp
        // instruction.  Reduced tiles are published per window as in the forward.
        const int wq = warp & 3;
        const int r = wq * 32 + lane;
        const int tid = threadIdx.x - kBWarpEpi * 32;  // 0..127
        const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
        float4 *xs = reinterpret_cast<float4 *>(sm + L::OFF_X + wq * 4096);  // [32 rows][8 chunks]
        int it = 0, ecnt = 0, ecnt_j = -1, vcnt = 0;
        bool ok = true;
        auto eg_sync = [&]() { asm volatile("bar.sync 2, 128;" ::: "memory"); };
        auto eg_vote = [&](int v) -> bool {
            const int slot = (vcnt++) & 1;
            if (tid == 0) eg_flag[slot] = v;
            eg_sync();
            return eg_flag[slot] != 0;
        };
        auto eg_wait = [&](uint64_t *b, uint32_t par) -> bool {
            int v = 1;
            if (tid == 0) v = mbar_wait(b, par, wait_ns) ? 1 : 0;
            return eg_vote(v);
        };
        auto flush = [&]() {  // publish the reductions of the tiles counted so far
            __threadfence();
            eg_sync();
            if (tid == 0) {
                __threadfence();
                atomicAdd(&tiles_done[ecnt_j], ecnt);
            }
            ecnt = 0;
        };
        while (ok) {
            const int ii = it % kBInfo;
            const uint32_t ipar = (it / kBInfo) & 1;
            if (ecnt > 0) {  // never sit on unpublished tiles while the next one is not there yet
                int ready = 1;
                if (tid == 0) ready = mbar_test(&info_full[ii], ipar) ? 1 : 0;
                if (!eg_vote(ready)) flush();
            }
            if (!eg_wait(&info_full[ii], ipar)) { ok = false; break; }
            const BTileInfo &inf = info[ii];
            if (inf.type == kBItemEnd) break;
            if (inf.j != ecnt_j) {
                if (ecnt > 0) flush();
                ecnt_j = inf.j;
            }
            const int qb = it & 1;  // dQ buffer of this tile
            if (!eg_wait(&dq_full[qb], (it >> 1) & 1)) { ok = false; break; }
            tc_fence_after();
            const int s = inf.j % kRing;
            const int ws = (inf.j % P.nW) * P.W;
            // this lane reduces, for m = 0..7, the 16-byte chunk lane % 8 (8 halves) of warp row 4m + lane / 8
            const float cf = scale * acc_inv;
            __half *dst[8];
            bool dok[8];
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int tr = wq * 32 + 4 * m + (lane >> 3);
                const int i = tr / G;
                dok[m] = i < inf.ntok;
                dst[m] = acc + ((int64_t)(s * P.W + inf.tok[i] - ws) * G + tr % G) * D + (lane & 7) * 8;
            }
            uint4 *xs4 = reinterpret_cast<uint4 *>(xs);
#pragma unroll kBEpiUnroll
            for (int q = 0; q < D / 64; ++q) {  // 64 columns = one 128-byte fp16 line per row
                float v[2][32];                   // both 32-column loads in flight, one wait
                tmem_ld32(lane_base + kColDQ + qb * 128 + q * 64, v[0]);
                tmem_ld32(lane_base + kColDQ + qb * 128 + q * 64 + 32, v[1]);
                tmem_wait_ld();
#pragma unroll
                for (int hv = 0; hv < 2; ++hv) {  // 4 chunks of 8 halves each
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        const int ch = hv * 4 + c4;
                        __half2 h[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            h[e] = __floats2half2_rn(v[hv][c4 * 8 + 2 * e] * cf, v[hv][c4 * 8 + 2 * e + 1] * cf);
                        xs4[lane * 8 + (ch ^ (lane & 7))] = *reinterpret_cast<uint4 *>(h);
                    }
                }
                if (q == D / 64 - 1) {  // dQ read completely: hand the buffer back before the last reductions
                    tc_fence_before();
                    __syncwarp();
                    mbar_arrive_lane0(&dq_empty[qb], lane);
                }
                __syncwarp();
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const int row = 4 * m + (lane >> 3);
                    const uint4 f = xs4[row * 8 + ((lane & 7) ^ (row & 7))];
                    if (dok[m]) red_add_v4_f16x2(dst[m] + q * 64, f);
                }
                __syncwarp();
            }
            if (inf.unit_last) {
                if (!eg_wait(dkv_full, inf.useq & 1)) { ok = false; break; }
                tc_fence_after();
                const int64_t kbase = ((int64_t)(inf.b * P.hkv + inf.g) * P.L + (int64_t)inf.c * kChunk) * D;
                if constexpr (D == 128) {
                    const int64_t krow = kbase + r;
#pragma unroll kBEpiUnroll
                    for (int hk = 0; hk < 2; ++hk) {
                        float v[32];
                        tmem_ld32(lane_base + kColDK + hk * 32, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) atomicAdd(dk_acc + krow + (int64_t)(hk * 32 + i) * D, v[i] * scale);
                        tmem_ld32(lane_base + kColDV + hk * 32, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) atomicAdd(dv_acc + krow + (int64_t)(hk * 32 + i) * D, v[i]);
                    }
                } else {
                    // d = 64: warps 0-1 hold dK^T (lanes 0-63 of its columns), warps 2-3 dV^T
                    // (lanes 64-127 of its columns); lane r is column r mod 64 of d
                    const bool isk = wq < 2;
                    float *dst = (isk ? dk_acc : dv_acc) + kbase + (r & 63);
                    const float sc = isk ? scale : 1.f;
                    const uint32_t col = isk ? kColDK : kColDV;
#pragma unroll kBEpiUnroll
                    for (int hk = 0; hk < 2; ++hk) {
                        float v[32];
                        tmem_ld32(lane_base + col + hk * 32, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) atomicAdd(dst + (int64_t)(hk * 32 + i) * D, v[i] * sc);
                    }
                }
                tc_fence_before();
                __syncwarp();
                mbar_arrive_lane0(dkv_empty, lane);
            }
            eg_sync();  // the whole group is done with this tile's info entry
            if (tid == 0) mbar_arrive(&info_empty[ii]);
            ++ecnt;
            ++it;
        }
        if (ok && ecnt > 0) flush();
        if (!ok) { *abort_flag = 1; if (tid == 0) report(ds, HSA_ERR_TIMEOUT, kKBwdTc, 6, it); }
    } else if (warp < kBWarpProd) {
        // ============================================================ convert group
        // Converts each window's fp32 dq slot into dq (bf16) and re-zeroes it,
        // claiming kCombTokens-token items of a window once all its tiles are reduced.
        const int tid = threadIdx.x - kBWarpConv * 32;  // 0..kBConvThreads-1
        int vcnt = 0;
        bool ok = true;
        auto cg_sync = [&]() { asm volatile("bar.sync 3, %0;" ::"n"(kBConvThreads) : "memory"); };
        auto cg_bcast = [&](int v) -> int {
            const int slot = (vcnt++) & 1;
            if (tid == 0) cg_flag[slot] = v;
            cg_sync();
            return cg_flag[slot];
        };
        for (int jc = 0; jc < P.J && ok; ++jc) {
            int gok = 1;
            if (tid == 0) gok = bspin_geq(&tiles_done[jc], P.win_tiles[jc], abort_flag, wait_ns) ? 1 : 0;
            if (!cg_bcast(gok)) {
                if (tid == 0 && !*abort_flag) report(ds, HSA_ERR_TIMEOUT, kKBwdTc, 4, jc);
                ok = false;
                break;
            }
            const int ncomb = P.win_ncomb[jc];
            const int b = (jc / P.nW) / P.hkv, g = (jc / P.nW) % P.hkv;
            const int s = jc % kRing;
            const int ws = (jc % P.nW) * P.W;
            const int we = min(P.L, ws + P.W);
            while (true) {
                const int item = cg_bcast(tid == 0 ? atomicAdd(&comb_head[jc], 1) : 0);
                if (item >= ncomb) break;
                const int ta = ws + item * kCombTokens, tb = min(we, ta + kCombTokens);
                constexpr int UPT = G * D / 8;  // 8-value units per token
                constexpr int kBatch = 8;
                uint4 *A = reinterpret_cast<uint4 *>(acc + (int64_t)(s * P.W + (ta - ws)) * G * D);
                const int nunits = (tb - ta) * UPT;
                for (int u0 = 0; u0 < nunits; u0 += kBConvThreads * kBatch) {
                    uint4 raw[kBatch];
#pragma unroll
                    for (int k = 0; k < kBatch; ++k) {
                        const int u = u0 + k * kBConvThreads + tid;
                        if (u < nunits) raw[k] = __ldcg(A + u);
                    }
#pragma unroll
                    for (int k = 0; k < kBatch; ++k) {
                        const int u = u0 + k * kBConvThreads + tid;
                        if (u < nunits) {
                            const int t = ta + u / UPT, e = u % UPT;
                            const __half2 *h2 = reinterpret_cast<const __half2 *>(&raw[k]);
                            float f[8];
#pragma unroll
                            for (int x = 0; x < 4; ++x) {
                                const float2 g2 = __half22float2(h2[x]);
                                f[2 * x] = g2.x * acc_scale;
                                f[2 * x + 1] = g2.y * acc_scale;
                            }
                            __stcs(reinterpret_cast<uint4 *>(dq + (((int64_t)b * P.L + t) * P.hq + g * G) * D + e * 8),
                                   pack8(f));
                            A[u] = make_uint4(0, 0, 0, 0);
                        }
                    }
                }
                cg_sync();
                if (tid == 0) {
                    __threadfence();
                    atomicAdd(&comb_done[jc], 1);
                }
            }
        }
        if (!ok) { *abort_flag = 1; if (tid == 0) report(ds, HSA_ERR_TIMEOUT, kKBwdTc, 7, 0); }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kBWarpMma) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ stick-breaking backward
// The D / 32 consecutive fp32 values of lane `lane` of a d = D row (one vector load).
template <int D>
__device__ __forceinline__ void lane_cols_f32(const float *row, int lane, float (&f)[D / 32]) {
    if constexpr (D == 128) {
        const float4 v = *reinterpret_cast<const float4 *>(row + lane * 4);
        f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
    } else {
        const float2 v = *reinterpret_cast<const float2 *>(row + lane * 2);
        f[0] = v.x; f[1] = v.y;
    }
}

// The D / 32 consecutive bf16 values of lane `lane` of a d = D row, as floats.
template <int D>
__device__ __forceinline__ void lane_cols(const __nv_bfloat16 *row, int lane, float (&f)[D / 32]) {
    if constexpr (D == 128) {
        const uint2 raw = *reinterpret_cast<const uint2 *>(row + lane * 4);
        const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
        const float2 f0 = __bfloat1622float2(h2[0]), f1 = __bfloat1622float2(h2[1]);
        f[0] = f0.x; f[1] = f0.y; f[2] = f1.x; f[3] = f1.y;
    } else {
        const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(row + lane * 2));
        f[0] = f0.x; f[1] = f0.y;
    }
}

// One warp per (b, t, g), d = D (D / 32 columns per lane).  With the chunk
// weights' gradients dw from the attention pass, recompute the selected
// chunks' scores s_j = q_slc . kbar_{c_j} / sqrt(d) and sig_j = sigmoid(s_j):
//   ds_j   = dw_j w_j (1 - sig_j) - sig_j sum_{k>j} dw_k w_k
//   dq_slc = sum_j ds_j kbar_{c_j} / sqrt(d),   dkbar_{c_j} += ds_j q_slc / sqrt(d)
// Cited page: "Hardware-aligned Hierarchical Sparse Attention ..." §HSA
// "end-to-end learning" (the chunk weight's gradient reaches the scores).
template <int D>
__global__ void __launch_bounds__(256) bwd_select_kernel(const __nv_bfloat16 *__restrict__ q_slc,
                                                         const int32_t *__restrict__ idx, const float *__restrict__ w,
                                                         float *dw_ds, const float *__restrict__ kbar,
                                                         __nv_bfloat16 *__restrict__ dq_slc,
                                                         int64_t rows, int L, int hkv, int nc, int K) {
    const int lane = threadIdx.x & 31;
    const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (gw >= rows) return;
    const int g = (int)(gw % hkv);
    const int64_t bt = gw / hkv;  // b * L + t
    const int b = (int)(bt / L);
    const int64_t bg = (int64_t)b * hkv + g;
    constexpr int NC = D / 32;  // columns per lane
    const float scale = 1.0f / sqrtf((float)D);
    float qv[NC];
    lane_cols<D>(q_slc + gw * D, lane, qv);
    // lane k < K: the slot's chunk, weight, weight gradient and score; an index
    // that is not causally eligible is skipped (the inversion reports it)
    const int t = (int)(bt % L);
    int ck = (lane < K) ? idx[gw * K + lane] : -1;
    if (ck >= min(nc, t / kChunk)) ck = -1;
    const float wk = (ck >= 0) ? w[gw * K + lane] : 0.f;
    const float dwk = (ck >= 0) ? dw_ds[gw * K + lane] : 0.f;
    float sk = 0.f;
    for (int k = 0; k < K; ++k) {
        const int c = __shfl_sync(0xffffffffu, ck, k);
        if (c < 0) continue;  // an empty or ineligible slot: score and gradient stay 0
        float kr[NC];
        lane_cols_f32<D>(kbar + (bg * nc + c) * D, lane, kr);
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < NC; ++e) a = fmaf(qv[e], kr[e], a);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
        if (lane == k) sk = a * scale;
    }
    const float sg = (ck >= 0) ? 1.0f / (1.0f + expf(-sk)) : 0.f;
    // tail_j = sum_{k>j} dw_k w_k: suffix sum over the lanes
    const float prod = dwk * wk;
    float incl = prod;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_down_sync(0xffffffffu, incl, off);
        if (lane + off < 32) incl += y;
    }
    const float dsk = (ck >= 0) ? prod * (1.f - sg) - sg * (incl - prod) : 0.f;
    float dqv[NC];
#pragma unroll
    for (int e = 0; e < NC; ++e) dqv[e] = 0.f;
    for (int k = 0; k < K; ++k) {
        const int c = __shfl_sync(0xffffffffu, ck, k);
        if (c < 0) continue;
        const float dsj = __shfl_sync(0xffffffffu, dsk, k) * scale;
        float kr[NC];
        lane_cols_f32<D>(kbar + (bg * nc + c) * D, lane, kr);
#pragma unroll
        for (int e = 0; e < NC; ++e) dqv[e] = fmaf(dsj, kr[e], dqv[e]);
    }
    // the slot's score gradient (times 1/sqrt(d)) replaces its weight gradient in place (each
    // lane read its own entry above); bwd_dkbar_kernel sums it into the pooled-key gradient
    if (lane < K) dw_ds[gw * K + lane] = dsk * scale;
    if constexpr (NC == 4) {
        __nv_bfloat162 o0 = __floats2bfloat162_rn(dqv[0], dqv[1]), o1 = __floats2bfloat162_rn(dqv[2], dqv[3]);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t *>(&o0);
        pk.y = *reinterpret_cast<uint32_t *>(&o1);
        *reinterpret_cast<uint2 *>(dq_slc + gw * D + lane * 4) = pk;
    } else {
        *reinterpret_cast<__nv_bfloat162 *>(dq_slc + gw * D + lane * 2) = __floats2bfloat162_rn(dqv[0], dqv[1]);
    }
}

// Gradient of the pooled keys, chunk-major: dkbar[c] = sum over the (token, slot) entries
// of chunk c's list of ds(token, slot) * q_slc[token].  One warp per list segment of
// kBwdSeg entries (segment z of (b, g) belongs to the chunk c with seg_off[c] <= z <
// seg_off[c+1]); a lane owns D / 32 of the D columns; one reduction per segment.
template <int D>
__global__ void __launch_bounds__(256) bwd_dkbar_kernel(const __nv_bfloat16 *__restrict__ q_slc,
                                                        const float *__restrict__ ds, const int32_t *__restrict__ chunk_off,
                                                        const int32_t *__restrict__ seg_off,
                                                        const int32_t *__restrict__ entries, float *__restrict__ dkbar,
                                                        int L, int hkv, int nc, int K) {
    constexpr int NC = D / 32;
    const int lane = threadIdx.x & 31;
    const int z = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int bg = blockIdx.y, b = bg / hkv, g = bg % hkv;
    const int32_t *so = seg_off + (int64_t)bg * (nc + 1);
    if (z >= so[nc]) return;
    int lo = 0, hi = nc - 1;  // last c with so[c] <= z
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (so[mid] <= z) lo = mid; else hi = mid - 1;
    }
    const int c = lo;
    const int32_t *off = chunk_off + (int64_t)bg * (nc + 1);
    const int beg = off[c] + (z - so[c]) * kBwdSeg;
    const int n = min(off[c + 1], beg + kBwdSeg) - beg;
    if (n <= 0) return;
    const int32_t *E = entries + (int64_t)bg * L * K;
    int64_t qrow = 0;  // this lane's entry: its selection-query row and score gradient
    float dsv = 0.f;
    if (lane < n) {
        const int ent = E[beg + lane];
        const int64_t row = ((int64_t)b * L + (ent >> 4)) * hkv + g;
        qrow = row * D;
        dsv = ds[row * K + (ent & 15)];
    }
    float acc[NC];
#pragma unroll
    for (int e = 0; e < NC; ++e) acc[e] = 0.f;
    for (int i = 0; i < n; ++i) {
        const int64_t qr = __shfl_sync(0xffffffffu, qrow, i);
        const float d = __shfl_sync(0xffffffffu, dsv, i);
        float f[NC];
        lane_cols<D>(q_slc + qr, lane, f);
#pragma unroll
        for (int e = 0; e < NC; ++e) acc[e] = fmaf(d, f[e], acc[e]);
    }
    float *dst = dkbar + ((int64_t)bg * nc + c) * D + lane * NC;
    if constexpr (NC == 4) {
        red_add_v4_f32(dst, make_float4(acc[0], acc[1], acc[2], acc[3]));
    } else {
        atomicAdd(dst, acc[0]);
        atomicAdd(dst + 1, acc[1]);
    }
}

// ------------------------------------------------------------------ magnitude bound
// max over rows of the L2 norm of a row of d = D bf16 values, as float bits max-ed into
// *bits.  A row is D / 8 lanes x 16 bytes; every thread keeps 4 rows' loads in flight.
template <int D>
__global__ void __launch_bounds__(256) rownorm_max_kernel(const __nv_bfloat16 *__restrict__ x, int64_t rows,
                                                          int32_t *__restrict__ bits) {
    constexpr int kU = 4;
    constexpr int LPR = D / 8;  // lanes per row
    const int64_t nvec = rows * LPR;  // 16-byte vectors
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    float m = 0.f;
    for (int64_t v0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v0 - (int64_t)(threadIdx.x & 31) < nvec;
         v0 += kU * stride) {
        uint4 raw[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t vi = v0 + u * stride;
            raw[u] = vi < nvec ? __ldcs(reinterpret_cast<const uint4 *>(x) + vi) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&raw[u]);
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h[e]);
                ss += f.x * f.x + f.y * f.y;
            }
#pragma unroll
            for (int off = LPR / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);  // one row
            m = fmaxf(m, sqrtf(ss));
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0) atomicMax(bits, __float_as_int(m));
}

cudaError_t launch_rownorm_max(const void *x, int64_t rows, int d, int32_t *bits, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    if (d != 64 && d != 128) return cudaErrorInvalidValue;
    const int blocks = (int)std::min<int64_t>(ceil_div(rows * (d / 8), 256 * 4), 148 * 8);
    if (d == 128)
        rownorm_max_kernel<128><<<blocks, 256, 0, st>>>((const __nv_bfloat16 *)x, rows, bits);
    else
        rownorm_max_kernel<64><<<blocks, 256, 0, st>>>((const __nv_bfloat16 *)x, rows, bits);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ host side
namespace {
typedef CUresult (*BEncodeFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                              const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
BEncodeFn b_encode() {
    static BEncodeFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<BEncodeFn>(p);
    }
    return fn;
}
// 2D bf16 map: inner dim `cols` (contiguous), outer `rows`; box 64 x box_rows, 128B swizzle
bool b_map(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
    BEncodeFn enc = b_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// token rows of d = 128 as a 3D view (64 columns, rows, 2 halves of 128 bytes); box =
// 8 rows x both halves, stored half after half (2 KB per 8-row group, 128B swizzle)
bool b_map_q3(CUtensorMap *m, const void *base, uint64_t rows) {
    BEncodeFn enc = b_encode();
    if (!enc) return false;
    cuuint64_t dims[3] = {64, rows, 2};
    cuuint64_t strides[2] = {256, 128};
    cuuint32_t box[3] = {64, 8, 2};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int G, int D>
cudaError_t launch_btc(const Shape &sh, const AttendPlan &plan, const BwdWs &inv, const void *q, const void *k,
                       const void *v, const void *dO, const float *lse, float *dw, __half *acc, void *dq,
                       float *dk_acc, float *dv_acc, DevStatus *ds, cudaStream_t st) {
    CUtensorMap mq, mo, mk, mv;
    const uint64_t qrows = (uint64_t)sh.B * sh.L * sh.hq, krows = (uint64_t)sh.B * sh.hkv * sh.L;
    // query / output-gradient rows: d = 128, the 3D view (8 rows x both halves per box);
    // d = 64, 2D boxes of 8 rows x 64 columns
    const bool qok = (D == 128) ? (b_map_q3(&mq, q, qrows) && b_map_q3(&mo, dO, qrows))
                                : (b_map(&mq, q, 64, qrows, 8) && b_map(&mo, dO, 64, qrows, 8));
    if (!qok || !b_map(&mk, k, D, krows, 64) || !b_map(&mv, v, D, krows, 64)) return cudaErrorInvalidValue;
    const size_t smem = BSmem<D>::ALLOC;
    cudaError_t e = set_smem_once((const void *)bwd_tc_kernel<G, D>, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    bwd_tc_kernel<G, D><<<sms, kBThreads, smem, st>>>(mq, mo, mk, mv, plan, inv.entries, inv.entw, lse, dw, acc,
                                                   (__nv_bfloat16 *)dq, dk_acc, dv_acc, ds, wait_limit_ns());
    return cudaGetLastError();
}
}  // namespace

bool bwd_tc_supported(const Shape &sh) {
    return sh.bf16 && sh.S == kChunk && (sh.d == 64 || sh.d == 128) && (sh.G == 8 || sh.G == 16) &&
           sh.K <= 16 && b_encode() != nullptr;
}

cudaError_t launch_bwd_tc(const Shape &sh, const AttendPlan &plan, const BwdWs &inv, const void *q, const void *k,
                          const void *v, const void *dO, const float *lse, float *dw, __half *acc, void *dq,
                          float *dk_acc, float *dv_acc, DevStatus *ds, cudaStream_t st) {
    if (sh.d == 128) {
        if (sh.G == 8) return launch_btc<8, 128>(sh, plan, inv, q, k, v, dO, lse, dw, acc, dq, dk_acc, dv_acc, ds, st);
        if (sh.G == 16) return launch_btc<16, 128>(sh, plan, inv, q, k, v, dO, lse, dw, acc, dq, dk_acc, dv_acc, ds, st);
    } else if (sh.d == 64) {
        if (sh.G == 8) return launch_btc<8, 64>(sh, plan, inv, q, k, v, dO, lse, dw, acc, dq, dk_acc, dv_acc, ds, st);
        if (sh.G == 16) return launch_btc<16, 64>(sh, plan, inv, q, k, v, dO, lse, dw, acc, dq, dk_acc, dv_acc, ds, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_bwd_select(const Shape &sh, const void *q_slc, const int32_t *idx, const float *w, float *dw,
                              const float *kbar, void *dq_slc, float *dkbar, const BwdWs &inv, cudaStream_t st) {
    const int64_t rows = (int64_t)sh.B * sh.L * sh.hkv;
    if (rows == 0) return cudaSuccess;
    if (sh.d == 128)
        bwd_select_kernel<128><<<(unsigned)ceil_div(rows, 8), 256, 0, st>>>(
            (const __nv_bfloat16 *)q_slc, idx, w, dw, kbar, (__nv_bfloat16 *)dq_slc, rows, sh.L, sh.hkv,
            std::max(sh.nc, 1), sh.K);
    else
        bwd_select_kernel<64><<<(unsigned)ceil_div(rows, 8), 256, 0, st>>>(
            (const __nv_bfloat16 *)q_slc, idx, w, dw, kbar, (__nv_bfloat16 *)dq_slc, rows, sh.L, sh.hkv,
            std::max(sh.nc, 1), sh.K);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || sh.nc == 0) return e;
    // segments of kBwdSeg list entries: at most L*K/kBwdSeg + nc per (b, g); 8 per block
    const int64_t maxseg = ceil_div((int64_t)sh.L * sh.K, kBwdSeg) + sh.nc;
    const dim3 grid((unsigned)ceil_div(maxseg, 8), (unsigned)(sh.B * sh.hkv));
    if (sh.d == 128)
        bwd_dkbar_kernel<128><<<grid, 256, 0, st>>>((const __nv_bfloat16 *)q_slc, dw, inv.chunk_off, inv.seg_off,
                                                    inv.entries, dkbar, sh.L, sh.hkv, sh.nc, sh.K);
    else
        bwd_dkbar_kernel<64><<<grid, 256, 0, st>>>((const __nv_bfloat16 *)q_slc, dw, inv.chunk_off, inv.seg_off,
                                                   inv.entries, dkbar, sh.L, sh.hkv, sh.nc, sh.K);
    return cudaGetLastError();
}

}  // namespace hsa
