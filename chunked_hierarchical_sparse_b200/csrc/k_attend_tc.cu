// k_attend_tc.cu -- chunk-major softmax-off-by-one attention with
// stick-breaking fusion on the 5th-generation tensor cores (tcgen05 + TMEM +
// TMA), persistent, warp-specialised.
//
// Cited page: "Hardware-aligned Hierarchical Sparse Attention for Efficient
// Long-term Memory Access" (paper notes), §HSA first and second stages (token-
// level attention inside each selected chunk, stick-breaking fusion of the
// chunk outputs) and §kernel (softmax-off-by-one; the backward's second phase
// walks, per chunk, the tokens that selected it).  The pages' forward kernel
// is token-major; this one is chunk-major: a tile holds TT = 128/G tokens
// that selected the same chunk, with the G query heads of each token as rows
// (the GQA-group idea of the NSA blog), so one 64-key K/V tile loaded by TMA
// serves 128 query rows on the tensor cores:
//   S[128 x 64]  = Q_tile[128 x d] . K_c^T          (tcgen05, fp32 in TMEM)
//   p = exp(x - m) / (e^{-m} + sum exp(x - m)),  x = S / sqrt(d), m = max(0, max x)
//   O[128 x d]   = P[128 x 64] . V_c                (tcgen05, fp32 in TMEM)
//   acc[t, h] += (w_{t,g,slot} / Z) * O * 2^-e   (fp16 reduce-add in L2 into the
//                                             window's accumulator slot; 2^e >= max|v|)
// Once every tile of a window has been reduced, the convert step of the same
// persistent kernel writes o[t, h] = bf16(acc[t, h]) and zeroes the slot for
// the window that reuses it kRing windows later.  The slot sums each token's
// chunk outputs in fp32, so no per-chunk partial is ever rounded or spilled.
//
// Roles (12 warps): warp 8 pulls work units and issues the TMA loads, warp 9
// allocates TMEM and issues the MMAs (one elected lane), warps 0-3 do the
// softmax and the epilogue (TMEM -> fp32 x coefficient -> swizzled SMEM),
// warp 10 issues the reductions, warps 4-7 run the convert step.  Every wait
// is bounded (a wall-clock limit); on expiry the kernel records
// HSA_ERR_TIMEOUT, unwinds, frees its TMEM and returns.
#include <algorithm>

#include "hsa_internal.cuh"
#include "sm100.cuh"

namespace hsa {

using namespace sm100;


namespace {

constexpr int kConvBatch = 8;  // 16-byte accumulator loads in flight per convert thread

// 16 warps:
//   warps 0-3 softmax, warps 4-7 and 8-11 two epilogue groups (weighted O ->
//   fp32 reductions into the window accumulators; group e takes the tiles whose
//   O buffer is e), warps 12-13 convert step, warp 14 producer, warp 15 MMA issuer
constexpr int kThreads = 512;
constexpr int kWarpEpi = 4, kWarpConv = 12, kWarpProd = 14, kWarpMma = 15;
constexpr int kConvThreads = 64;
constexpr int kInfo = 8;                 // tile-info ring entries
constexpr int kQStages = 3;              // query-tile buffers (P lives in TMEM, not SMEM)
// TMEM columns: S[2] 0..127 (fp32), O[2] 128..383 (fp32), P[2] 384..447 (bf16 pairs)
constexpr uint32_t kColO = 128, kColP = 384;

enum ItemType : int { kItemTile = 0, kItemEnd = 2 };

struct TileInfo {
    int type;
    int j;        // window
    int b, g, c;  // sequence, group, chunk
    int ntok;     // valid tokens in the tile
    int kvs, kvph, unit_first, unit_last;
    int qs, qph;
    int tok[16];
    int slot[16];
    float w[16];  // stick-breaking weight of each token's slot
};

template <int D> struct Smem {
    // A query tile is 16 groups of 8 rows; a group holds its rows' 64-column halves
    // one after the other (1 KB each), so one TMA box loads a whole group.
    static constexpr int QHALF = 128 * 128;  // bytes per 64-column half of a 128-row tile
    static constexpr int NH = D / 64;        // halves along d
    static constexpr int QBYTES = NH * QHALF;
    static constexpr int KVHALF = 64 * 128;
    static constexpr int KVBYTES = NH * KVHALF;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + kQStages * QBYTES;
    static constexpr int OFF_V = OFF_K + 2 * KVBYTES;
    static constexpr int OFF_X = OFF_V + 2 * KVBYTES;           // epilogue transpose scratch, 2 KB per warp
    static constexpr int OFF_COEF = OFF_X + 8 * 2048;           // [kInfo][128] fp32 row coefficients w / Z
    static constexpr int OFF_INFO = OFF_COEF + kInfo * 128 * 4;
    static constexpr int OFF_BAR = OFF_INFO + kInfo * (int)sizeof(TileInfo);
    static constexpr int NBAR = 3 * kInfo + 2 * kQStages + 2 * 2 + 2 * 2 + 2 + 2 * 2 + 1 + 2;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_MISC + 64;
    static constexpr int ALLOC = BYTES + 1024;  // slack for 1 KB alignment
};

static_assert(Smem<128>::ALLOC <= 227 * 1024, "attention tile buffers exceed the shared memory of a CTA");

struct Bars {
    uint64_t *info_full, *info_empty;  // [kInfo]
    uint64_t *q_full, *q_empty;        // [kQStages]
    uint64_t *kv_full, *kv_empty;      // [2]
    uint64_t *s_full, *s_empty;        // [2]
    uint64_t *p_full;                  // [2]
    uint64_t *o_full, *o_empty;        // [2]
};

__device__ __forceinline__ int ld_acquire(const int32_t *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// 2^x with the hardware approximation (relative error about 2^-22, subnormal
// results flushed to zero); its inputs here are <= 0 logits in base 2.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// bounded spin until *p >= target; false on timeout or once *abort is set
__device__ bool spin_geq_live(const int32_t *p, int target, volatile int *abort, uint64_t wait_ns) {
    if (ld_acquire(p) >= target) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
        __nanosleep(256);
        if (ld_acquire(p) >= target) return true;
        if (*abort) return false;
        if (globaltimer() - t0 > wait_ns) return false;
    }
}


}  // namespace

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 1) attend_tc_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v,
    const __grid_constant__ AttendPlan P, const int32_t *__restrict__ entries,
    const float *__restrict__ entw, __half *__restrict__ acc,
    __nv_bfloat16 *__restrict__ out, float *__restrict__ lse, DevStatus *ds, uint64_t wait_ns) {
    using L = Smem<D>;
    constexpr int TT = 128 / G;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    TileInfo *info = reinterpret_cast<TileInfo *>(sm + L::OFF_INFO);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L::OFF_BAR);
    Bars B;
    B.info_full = bar; B.info_empty = bar + kInfo;
    B.q_full = bar + 2 * kInfo; B.q_empty = B.q_full + kQStages;
    B.kv_full = B.q_empty + kQStages; B.kv_empty = B.kv_full + 2;
    B.s_full = B.kv_empty + 2; B.s_empty = B.s_full + 2;
    B.p_full = B.s_empty + 2;
    B.o_full = B.p_full + 2; B.o_empty = B.o_full + 2;
    uint64_t *mma_done = B.o_empty + 2;
    uint64_t *coef_full = mma_done + 1;  // [kInfo] row coefficients written (softmax -> epilogue)
    uint64_t *p_empty = coef_full + kInfo;  // [2] P buffer read by its O = P.V (MMA -> softmax)
    float *ecoef = reinterpret_cast<float *>(sm + L::OFF_COEF);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::OFF_MISC + 16);
    volatile int *cg_flag = reinterpret_cast<volatile int *>(sm + L::OFF_MISC + 56);  // [2] convert group

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kInfo; ++i) { mbar_init(&B.info_full[i], 1); mbar_init(&B.info_empty[i], 1 + 8); }
        for (int i = 0; i < kQStages; ++i) { mbar_init(&B.q_full[i], 1); mbar_init(&B.q_empty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&B.kv_full[i], 1); mbar_init(&B.kv_empty[i], 1);
            mbar_init(&B.s_full[i], 1); mbar_init(&B.s_empty[i], 4);
            mbar_init(&B.p_full[i], 4);
            mbar_init(&B.o_full[i], 1); mbar_init(&B.o_empty[i], 4);
        }
        mbar_init(mma_done, 1);
        for (int i = 0; i < kInfo; ++i) mbar_init(&coef_full[i], 4);
        for (int i = 0; i < 2; ++i) mbar_init(&p_empty[i], 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    if (warp == kWarpProd && lane == 0) {
        prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    int32_t *tiles_done = P.counters;
    int32_t *comb_done = P.counters + P.J;
    int32_t *comb_head = P.counters + 2 * P.J;
    const float scale = 1.0f / sqrtf((float)D);
    // power-of-two scale of the fp16 accumulators: 2^e >= max|v| * max(1, max_row sum|w|)
    // (bits written by vmax_kernel and, for a caller-given selection, wsum_kernel)
    float acc_scale, acc_inv;
    {
        const float wsum = __int_as_float(P.counters[3 * P.J + 2]);
        const uint32_t vb = (uint32_t)__float_as_int(__int_as_float(P.counters[3 * P.J + 1]) * fmaxf(1.f, wsum));
        int ev = (int)((vb >> 23) & 0xff) - 127;
        if (vb & 0x7fffffu) ev += 1;
        if (vb == 0) ev = 0;
        ev = max(-100, min(ev, 120));
        acc_scale = __int_as_float((ev + 127) << 23);
        acc_inv = __int_as_float((127 - ev) << 23);
    }

    // every lane waits (converged, sleeping in try_wait); the warp decides by a vote
    auto warp_wait = [&](uint64_t *b, uint32_t par) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(b, par, wait_ns));
    };

    if (warp == kWarpProd) {
        // ============================================================ producer
        // Work units are dealt to the CTAs in queue order (unit q to CTA
        // q mod gridDim.x), which keeps every CTA in window order.  Descriptors
        // are loaded two units ahead and a unit's entries and weights one unit
        // ahead, so no global-memory latency sits on the tile path.
        int it = 0, qc = 0, kvc = 0;
        bool ok = true;
        const int total = min(P.seg_start[P.J], P.max_items);
        const int qstep = gridDim.x;
        int guard_ok_j = -1;  // highest window whose ring guard already passed
        struct Desc { int4 a, b; };
        // queue position q of window jw is unit q - seg_start[jw] of jw's slice of the
        // queue; the positions looked up only grow, so the window only moves forward and
        // its bounds stay in registers (a load only when a window boundary is crossed)
        int jw = 0, seg_lo = 0, seg_hi = P.J > 1 ? P.seg_start[1] : total;
        auto load_desc = [&](int q) -> Desc {  // every lane loads the same 32 bytes
            Desc d;
            if (q < total) {
                while (q >= seg_hi && jw + 1 < P.J) {
                    ++jw;
                    seg_lo = seg_hi;
                    seg_hi = jw + 1 < P.J ? P.seg_start[jw + 1] : total;
                }
                const int64_t u = (int64_t)jw * P.win_cap + (q - seg_lo);
                d.a = P.items[2 * u];
                d.b = P.items[2 * u + 1];
            } else {
                d.a = make_int4(kItemEnd, 0, 0, 0);
                d.b = make_int4(0, 0, 0, 0);
            }
            return d;
        };
        struct Pay { int ea, eb; float wa, wb; };  // a unit's (token, slot) entries and weights, two per lane
        auto load_pay = [&](const Desc &d) -> Pay {
            Pay p{0, 0, 0.f, 0.f};
            if (d.a.x == kItemTile) {
                const int64_t base = (int64_t)(d.a.y / P.nW) * P.ent_stride;
                const int ub = d.a.w + d.b.y * TT;
                const int un = min(d.b.x, d.a.w + d.b.z * TT) - ub;
                if (lane < un) { p.ea = entries[base + ub + lane]; p.wa = entw[base + ub + lane]; }
                if (lane + 32 < un) { p.eb = entries[base + ub + lane + 32]; p.wb = entw[base + ub + lane + 32]; }
            }
            return p;
        };
        int qn = blockIdx.x;  // queue index of the unit in dc
        Desc dc = load_desc(qn), dn = load_desc(qn + qstep);
        Pay pc = load_pay(dc);
        while (ok) {
            const int ii = it % kInfo;
            if (it >= kInfo && !warp_wait(&B.info_empty[ii], ((it / kInfo) - 1) & 1)) { ok = false; break; }
            if (*abort_flag) { ok = false; break; }
            const int type = dc.a.x, j = dc.a.y, c = dc.a.z, e0 = dc.a.w;
            const int e1 = dc.b.x, t0 = dc.b.y, t1 = dc.b.z;
            const int ent_a = pc.ea, ent_b = pc.eb;
            const float w_a = pc.wa, w_b = pc.wb;
            TileInfo &inf = info[ii];
            if (type == kItemEnd) {
                if (lane == 0) {
                    inf.type = kItemEnd;
                    mbar_arrive(&B.info_full[ii]);
                }
                break;
            }
            {  // the next units' data in flight while this one is issued
                const Pay pn = load_pay(dn);
                dc = dn;
                dn = load_desc(qn + 2 * qstep);
                pc = pn;
                qn += qstep;
            }
            const int bg = j / P.nW;
            const int b = bg / P.hkv, g = bg % P.hkv;
            // ---- work unit: chunk c, tiles [t0, t1) of the bucket entries [e0, e1) of window j
            // the unit's (token, slot) entries: up to kUnitTiles * TT <= 64, two per lane
            const int ub = e0 + t0 * TT;
            const int un = min(e1, e0 + t1 * TT) - ub;
            // ring guard: window j's partial slot was last used by window j - kRing
            if (j >= kRing && j > guard_ok_j) {
                int g_ok = 1;
                if (lane == 0) g_ok = spin_geq_live(&comb_done[j - kRing], P.win_ncomb[j - kRing], abort_flag, wait_ns) ? 1 : 0;
                if (!__shfl_sync(0xffffffffu, g_ok, 0)) {
                    if (lane == 0 && !*abort_flag) report(ds, HSA_ERR_TIMEOUT, kKAttendTc, 1, j);
                    ok = false;
                    break;
                }
                guard_ok_j = j;
            }
            // K/V tiles of chunk c
            const int kvs = kvc & 1, kvph = (kvc >> 1) & 1;
            if (kvc >= 2 && !warp_wait(&B.kv_empty[kvs], ((kvc >> 1) - 1) & 1)) { ok = false; break; }
            if (lane == 0) {
                mbar_arrive_expect_tx(&B.kv_full[kvs], 2 * L::KVBYTES);
                const int row = bg * P.L + c * kChunk;
#pragma unroll
                for (int h = 0; h < L::NH; ++h) {
                    tma_load_2d(sm + L::OFF_K + kvs * L::KVBYTES + h * L::KVHALF, &tm_k, h * 64, row, &B.kv_full[kvs]);
                    tma_load_2d(sm + L::OFF_V + kvs * L::KVBYTES + h * L::KVHALF, &tm_v, h * 64, row, &B.kv_full[kvs]);
                }
            }
            ++kvc;
            for (int tt = t0; tt < t1; ++tt) {
                const int ti = it % kInfo;
                if (it >= kInfo && !warp_wait(&B.info_empty[ti], ((it / kInfo) - 1) & 1)) { ok = false; break; }
                const int qs = qc % kQStages, qph = (qc / kQStages) & 1;
                if (qc >= kQStages && !warp_wait(&B.q_empty[qs], ((qc / kQStages) - 1) & 1)) { ok = false; break; }
                TileInfo &ti_ = info[ti];
                const int lo = (tt - t0) * TT;          // first entry of this tile within the unit
                const int ntok = min(TT, un - lo);
                // entry of token `lane` of this tile lives in lane (lo + lane) % 32 of ent_a/ent_b
                const int src = (lo + lane) & 31;
                const int va = __shfl_sync(0xffffffffu, ent_a, src);
                const int vb = __shfl_sync(0xffffffffu, ent_b, src);
                const int ent = (lo + lane < 32) ? va : vb;
                const float wva = __shfl_sync(0xffffffffu, w_a, src);
                const float wvb = __shfl_sync(0xffffffffu, w_b, src);
                const float wgt = (lo + lane < 32) ? wva : wvb;
                int t = ent >> 4, slot = ent & 15;
                {  // an entry outside its window (inconsistent lists) is reported and made harmless
                    const int wsv = (j % P.nW) * P.W;
                    const bool bad = lane < ntok && (t < wsv || t >= min(P.L, wsv + P.W) || slot >= P.K);
                    if (bad) { report(ds, HSA_ERR_DEVICE_CHECK, kKAttendTc, t, c); t = wsv; slot = 0; }
                    if (lane < 16) {
                        ti_.tok[lane] = (lane < ntok) ? t : -1;
                        ti_.slot[lane] = (lane < ntok) ? slot : 0;
                        ti_.w[lane] = (lane < ntok && !bad) ? wgt : 0.f;
                    }
                }
                // the query rows first (their gathers fly while the tile info is written)
                if (lane == 0) mbar_arrive_expect_tx(&B.q_full[qs], ntok * L::NH * G * 128);
                __syncwarp();
                if constexpr (L::NH == 2) {
                    // one 3D box per 8-row group (both 64-column halves): 128 rows = 16 loads
                    constexpr int GPT = G / 8;  // 8-row groups per token
                    const int tq = __shfl_sync(0xffffffffu, t, lane / GPT);
                    if (lane < ntok * GPT) {
                        const int row = (b * P.L + tq) * P.hq + g * G + (lane % GPT) * 8;
                        tma_load_3d(sm + L::OFF_Q + qs * L::QBYTES + lane * 2048, &tm_q, 0, row, 0, &B.q_full[qs]);
                    }
                } else if (lane < ntok) {
                    const int row = (b * P.L + t) * P.hq + g * G;
                    tma_load_2d(sm + L::OFF_Q + qs * L::QBYTES + lane * G * 128, &tm_q, 0, row, &B.q_full[qs]);
                }
                if (lane == 0) {
                    ti_.type = kItemTile; ti_.j = j; ti_.b = b; ti_.g = g; ti_.c = c; ti_.ntok = ntok;
                    ti_.kvs = kvs; ti_.kvph = kvph; ti_.unit_first = (tt == t0); ti_.unit_last = (tt == t1 - 1);
                    ti_.qs = qs; ti_.qph = qph;
                }
                __syncwarp();
                __syncwarp();
                mbar_arrive_lane0(&B.info_full[ti], lane);
                ++qc;
                ++it;
            }
        }
        if (!ok) {
            *abort_flag = 1;
            if (lane == 0) {
                report(ds, HSA_ERR_TIMEOUT, kKAttendTc, 2, it);
                // let the loads already issued land before the CTA goes away (bounded)
                for (int s2 = 0; s2 < kQStages; ++s2) {
                    if (qc > s2) mbar_wait(&B.q_full[(qc - 1 - s2) % kQStages], ((qc - 1 - s2) / kQStages) & 1, kDrainWaitNs);
                    if (s2 < 2 && kvc > s2) mbar_wait(&B.kv_full[(kvc - 1 - s2) & 1], ((kvc - 1 - s2) >> 1) & 1, kDrainWaitNs);
                }
            }
            __syncwarp();
        }
    } else if (warp == kWarpMma) {
        // ============================================================ MMA issuer
        // Two in-order streams polled by one lane: S(t) = Q_t K^T is issued as
        // soon as the tile's Q and K are in SMEM and an S buffer is free, and
        // O(t) = P_t V as soon as P_t is written and an O buffer is free, so a
        // slow epilogue never holds back the scores of the following tiles.
        constexpr uint32_t idesc1 = idesc_bf16_f32(128, 64, false, false);
        constexpr uint32_t idesc2 = idesc_bf16_f32(128, D, false, true);
        bool ok = true;
        int ts = 0, tp = 0;
        if (lane == 0) {
            bool s_done = false;  // the S stream has met the end item
            uint64_t t_last = globaltimer();
            while (true) {
                bool prog = false;
                if (!s_done) {
                    const int ii = ts % kInfo;
                    if (mbar_test(&B.info_full[ii], (ts / kInfo) & 1)) {
                        const TileInfo &inf = info[ii];
                        const int sb = ts & 1;
                        if (inf.type == kItemEnd) {
                            s_done = true;
                            prog = true;
                        } else if ((!inf.unit_first || mbar_test(&B.kv_full[inf.kvs], inf.kvph)) &&
                                   mbar_test(&B.q_full[inf.qs], inf.qph) &&
                                   (ts < 2 || mbar_test(&B.s_empty[sb], ((ts >> 1) - 1) & 1))) {
                            tc_fence_after();
                            const uint32_t qa = smem_u32(sm + L::OFF_Q + inf.qs * L::QBYTES);
                            const uint32_t kb = smem_u32(sm + L::OFF_K + inf.kvs * L::KVBYTES);
                            const uint32_t dcol = tmem + sb * 64;
#pragma unroll
                            for (int ks = 0; ks < D / 16; ++ks) {
                                const int h = ks >> 2, kk = ks & 3;
                                // Q: d = 128 in 2 KB groups of 8 rows x both halves; d = 64 in 1 KB groups
                                mma_bf16_ss(dcol, smem_desc_sw128(qa + h * 1024 + kk * 32, 16, L::NH * 1024),
                                            smem_desc_sw128(kb + h * L::KVHALF + kk * 32, 16, 1024), idesc1, ks > 0);
                            }
                            mma_commit(&B.s_full[sb]);
                            mma_commit(&B.q_empty[inf.qs]);
                            ++ts;
                            prog = true;
                        }
                    }
                }
                if (tp < ts) {
                    const int ii = tp % kInfo;
                    const TileInfo &inf = info[ii];
                    const int pb = tp & 1;
                    if (mbar_test(&B.p_full[pb], (tp >> 1) & 1) &&
                        (tp < 2 || mbar_test(&B.o_empty[pb], ((tp >> 1) - 1) & 1))) {
                        tc_fence_after();
                        const uint32_t pa = tmem + kColP + pb * 32;  // P: 64 keys as 32 bf16 pairs per row
                        const uint32_t vb = smem_u32(sm + L::OFF_V + inf.kvs * L::KVBYTES);
                        const uint32_t dcol = tmem + kColO + pb * 128;
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)  // 16 keys = 8 TMEM columns per step
                            mma_bf16_ts(dcol, pa + ks * 8, smem_desc_sw128(vb + ks * 2048, L::KVHALF, 1024), idesc2,
                                        ks > 0);
                        mma_commit(&B.o_full[pb]);
                        mma_commit(&p_empty[pb]);
                        if (inf.unit_last) mma_commit(&B.kv_empty[inf.kvs]);
                        mbar_arrive(&B.info_empty[ii]);
                        ++tp;
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
                report(ds, HSA_ERR_TIMEOUT, kKAttendTc, 3, ts);
            }
            // drain: every MMA issued by this warp has finished before TMEM is released
            mma_commit(mma_done);
            mbar_wait(mma_done, 0, kDrainWaitNs);
        }
        __syncwarp();
    } else if (warp < kWarpEpi) {
        // ============================================================ softmax
        const int wq = warp & 3;                 // TMEM lane quadrant of this warp
        const int r = wq * 32 + lane;            // tile row = token * G + head
        const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
        int it = 0, tseq = 0;
        bool ok = true;

        // every warp waits for itself (all lanes, sleeping in try_wait): the four warps
        // only meet at the mbarriers they arrive on
        while (ok) {
            const int ii = it % kInfo;
            const uint32_t ipar = (it / kInfo) & 1;
            if (!warp_wait(&B.info_full[ii], ipar)) { ok = false; break; }
            const TileInfo &inf = info[ii];
            const int type = inf.type;
            if (type == kItemEnd) break;
            // ---------------- softmax of this tile
            const int sb = tseq & 1;
            if (!warp_wait(&B.s_full[sb], (tseq >> 1) & 1)) { ok = false; break; }
            tc_fence_after();
            float x0[32], x1[32];
            tmem_ld32(lane_base + sb * 64, x0);
            tmem_ld32(lane_base + sb * 64 + 32, x1);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            mbar_arrive_lane0(&B.s_empty[sb], lane);
            // P buffer sb is free once the O = P.V of tile tseq - 2 has read it
            if (tseq >= 2 && !warp_wait(&p_empty[sb], ((tseq >> 1) - 1) & 1)) { ok = false; break; }
            const int ti = r / G, hh = r % G;
            const bool valid = ti < inf.ntok;
            uint32_t pr[32];  // this row's P: key pairs (2j, 2j+1) as bf16x2, the lower key in the low half
            float coef = 0.f;
            if (valid) {
                const int t = inf.tok[ti], slot = inf.slot[ti];
                const float L2E = 1.4426950408889634f;
                // running maxima start at 0: the off-by-one term is a logit of 0.
                // scale > 0, so max(scale * x) = scale * max(x) exactly.
                float mq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    mq[0] = fmaxf(mq[0], x0[i]);
                    mq[1] = fmaxf(mq[1], x0[i + 1]);
                    mq[2] = fmaxf(mq[2], x1[i]);
                    mq[3] = fmaxf(mq[3], x1[i + 1]);
                }
                const float m = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])) * scale;
                const float mb = m * L2E, sl2 = scale * L2E;
                float zq[4] = {ex2_approx(-mb), 0.f, 0.f, 0.f};
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    x0[i] = ex2_approx(fmaf(x0[i], sl2, -mb));
                    x0[i + 1] = ex2_approx(fmaf(x0[i + 1], sl2, -mb));
                    x1[i] = ex2_approx(fmaf(x1[i], sl2, -mb));
                    x1[i + 1] = ex2_approx(fmaf(x1[i + 1], sl2, -mb));
                    zq[0] += x0[i];
                    zq[1] += x0[i + 1];
                    zq[2] += x1[i];
                    zq[3] += x1[i + 1];
                }
                const float z = (zq[0] + zq[1]) + (zq[2] + zq[3]);
                coef = inf.w[ti] / z;
                if (lse) lse[(((int64_t)inf.b * P.L + t) * P.hq + inf.g * G + hh) * P.K + slot] = m + logf(z);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const __nv_bfloat162 a = __floats2bfloat162_rn(x0[2 * j], x0[2 * j + 1]);
                    const __nv_bfloat162 c = __floats2bfloat162_rn(x1[2 * j], x1[2 * j + 1]);
                    pr[j] = *reinterpret_cast<const uint32_t *>(&a);
                    pr[16 + j] = *reinterpret_cast<const uint32_t *>(&c);
                }
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) pr[j] = 0u;
            }
            // P into its TMEM buffer (the A operand of O = P.V), then handed to the MMA issuer
            tmem_st32(lane_base + kColP + sb * 32, pr);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            mbar_arrive_lane0(&B.p_full[sb], lane);  // one arrival per warp
            // the row's output coefficient w / Z for the epilogue group
            ecoef[ii * 128 + r] = coef;
            __syncwarp();
            mbar_arrive_lane0(&coef_full[ii], lane);
            ++tseq;
            ++it;
        }
        if (!ok) { *abort_flag = 1; if (lane == 0) report(ds, HSA_ERR_TIMEOUT, kKAttendTc, 5, it); }
    } else if (warp < kWarpConv) {
        // ============================================================ epilogue
        // Per tile: O (fp32, TMEM) times the row coefficient w / Z, transposed
        // through a 4 KB per-warp scratch so that each warp-wide vector reduction
        // covers four whole 128-byte lines, then reduce-added into the window's
        // accumulator slot in L2.  The tiles reduced per window are published in
        // tiles_done[window] (after a fence) when the window changes, when the
        // next tile is not there yet, and at the end.
        const int eg = (warp - kWarpEpi) >> 2;                    // epilogue group = its O buffer
        const int wq = warp & 3;
        const int r = wq * 32 + lane;                             // tile row of this lane's TMEM loads
        const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
        float4 *xs = reinterpret_cast<float4 *>(sm + L::OFF_X + (warp - kWarpEpi) * 2048);  // [32 rows][4 chunks]
        int it = 0, tseq = 0, ecnt = 0, ecnt_j = -1;
        bool ok = true;
        // Each warp runs on its own: it waits for itself, acknowledges each info slot
        // itself and publishes its own reduced rows per window (a window is complete
        // when its tiles are counted by all four warps of their group).
        auto flush = [&]() {  // publish this warp's reductions of the tiles counted so far
            __threadfence();
            __syncwarp();
            if (lane == 0) {
                __threadfence();
                atomicAdd(&tiles_done[ecnt_j], ecnt);
            }
            ecnt = 0;
        };
        while (ok) {
            const int ii = it % kInfo;
            const uint32_t ipar = (it / kInfo) & 1;
            if (ecnt > 0 && !__all_sync(0xffffffffu, mbar_test(&B.info_full[ii], ipar)))
                flush();  // never sit on unpublished tiles while the next one is not there yet
            if (!warp_wait(&B.info_full[ii], ipar)) { ok = false; break; }
            const TileInfo &inf = info[ii];
            if (inf.type == kItemEnd) break;
            if ((tseq & 1) != eg) {  // the other group's tile: acknowledge the slot and move on
                __syncwarp();
                mbar_arrive_lane0(&B.info_empty[ii], lane);
                ++tseq;
                ++it;
                continue;
            }
            if (inf.j != ecnt_j) {
                if (ecnt > 0) flush();
                ecnt_j = inf.j;
            }
            const int sb = tseq & 1;
            if (!warp_wait(&B.o_full[sb], (tseq >> 1) & 1)) { ok = false; break; }
            if (!warp_wait(&coef_full[ii], ipar)) { ok = false; break; }
            tc_fence_after();
            const float coef = ecoef[ii * 128 + r];
            const int s = inf.j % kRing;
            const int ws = (inf.j % P.nW) * P.W;
            // this lane reduces, for m = 0..3, the 16-byte chunk lane % 4 (8 halves) of warp row 8m + lane / 4
            // of each 32-column slice: one warp-wide reduction covers 8 rows x 64 contiguous bytes
            const float cf = coef * acc_inv;
            __half *dst[4];
            bool dok[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int tr = wq * 32 + 8 * m + (lane >> 2);
                const int i = tr / G;
                dok[m] = i < inf.ntok;
                dst[m] = acc + ((int64_t)(s * P.W + inf.tok[i] - ws) * G + tr % G) * D + (lane & 3) * 8;
            }
            uint4 *xs4 = reinterpret_cast<uint4 *>(xs);
#pragma unroll 1
            for (int q = 0; q < D / 32; ++q) {  // 32 columns = 64 fp16 bytes per row
                float v[32];
                tmem_ld32(lane_base + kColO + sb * 128 + q * 32, v);
                tmem_wait_ld();
                if (q == D / 32 - 1) {  // O read completely: hand the buffer back before the last reductions
                    tc_fence_before();
                    __syncwarp();
                    mbar_arrive_lane0(&B.o_empty[sb], lane);
                }
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    __half2 h[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        h[e] = __floats2half2_rn(v[c4 * 8 + 2 * e] * cf, v[c4 * 8 + 2 * e + 1] * cf);
                    xs4[lane * 4 + (c4 ^ ((lane >> 1) & 3))] = *reinterpret_cast<uint4 *>(h);
                }
                __syncwarp();
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int row = 8 * m + (lane >> 2);
                    const uint4 f = xs4[row * 4 + ((lane & 3) ^ ((row >> 1) & 3))];
                    if (dok[m]) red_add_v4_f16x2(dst[m] + q * 32, f);
                }
                __syncwarp();
            }
            mbar_arrive_lane0(&B.info_empty[ii], lane);  // this warp is done with the tile's info entry
            ++ecnt;
            ++tseq;
            ++it;
        }
        if (ok && ecnt > 0) flush();
        if (!ok) { *abort_flag = 1; if (lane == 0) report(ds, HSA_ERR_TIMEOUT, kKAttendTc, 6, it); }
    } else if (warp < kWarpProd) {
        // ============================================================ convert group
        // Converts each window's fp32 accumulators into o.  Every CTA's convert
        // group walks the windows in order: it waits until all tiles of window
        // jc are reduced, then claims jc's convert items (kCombTokens tokens
        // each) from comb_head[jc] until none are left, so a finished window is
        // converted by all CTAs at once while the tile pipeline moves on.
        const int tid = threadIdx.x - kWarpConv * 32;  // 0..kConvThreads-1
        int ci_n = 0, vcnt = 0;
        bool ok = true;
        auto cg_sync = [&]() { asm volatile("bar.sync 2, %0;" ::"n"(kConvThreads) : "memory"); };
        auto cg_bcast = [&](int v) -> int {  // thread 0's value to the whole group
            const int slot = (vcnt++) & 1;
            if (tid == 0) cg_flag[slot] = v;
            cg_sync();
            return cg_flag[slot];
        };
        for (int jc = 0; jc < P.J && ok; ++jc) {
            int gok = 1;
            // every tile is counted by the four warps of its epilogue group
            if (tid == 0) gok = spin_geq_live(&tiles_done[jc], 4 * P.win_tiles[jc], abort_flag, wait_ns) ? 1 : 0;
            if (!cg_bcast(gok)) { if (tid == 0 && !*abort_flag) report(ds, HSA_ERR_TIMEOUT, kKAttendTc, 4, jc); ok = false; break; }
            const int ncomb = P.win_ncomb[jc];
            while (true) {
                const int item = cg_bcast(tid == 0 ? atomicAdd(&comb_head[jc], 1) : 0);
                if (item >= ncomb) break;
                const int j = jc, b = (jc / P.nW) / P.hkv, g = (jc / P.nW) % P.hkv;
                const int s = j % kRing;
                const int ws = (j % P.nW) * P.W;
                const int we = min(P.L, ws + P.W);
                const int ta = ws + item * kCombTokens, tb = min(we, ta + kCombTokens);
                // fp16 accumulators of tokens [ta, tb): G*D contiguous values per token, and
                // o of (token, group g): G*D contiguous bf16.  A unit is 8 values -> 16 bytes of o.
                constexpr int UPT = G * D / 8;  // units per token
                constexpr int kBatch = kConvBatch;  // units in flight per thread
                uint4 *A = reinterpret_cast<uint4 *>(acc + (int64_t)(s * P.W + (ta - ws)) * G * D);
                const int nunits = (tb - ta) * UPT;
                for (int u0 = 0; u0 < nunits; u0 += kConvThreads * kBatch) {
                    uint4 raw[kBatch];
#pragma unroll
                    for (int k = 0; k < kBatch; ++k) {
                        const int u = u0 + k * kConvThreads + tid;
                        if (u < nunits) raw[k] = __ldcg(A + u);
                    }
#pragma unroll
                    for (int k = 0; k < kBatch; ++k) {
                        const int u = u0 + k * kConvThreads + tid;
                        if (u < nunits) {
                            const int t = ta + u / UPT, e = u % UPT;
                            const __half2 *h2 = reinterpret_cast<const __half2 *>(&raw[k]);
                            __nv_bfloat162 o2[4];
#pragma unroll
                            for (int x = 0; x < 4; ++x) {
                                const float2 f = __half22float2(h2[x]);
                                o2[x] = __floats2bfloat162_rn(f.x * acc_scale, f.y * acc_scale);
                            }
                            // o is not read again here: streaming store
                            __stcs(reinterpret_cast<uint4 *>(out + (((int64_t)b * P.L + t) * P.hq + g * G) * D + e * 8),
                                   *reinterpret_cast<uint4 *>(o2));
                            // the slot starts the window kRing later at zero
                            A[u] = make_uint4(0, 0, 0, 0);
                        }
                    }
                }
                cg_sync();
                if (tid == 0) {
                    __threadfence();
                    atomicAdd(&comb_done[j], 1);
                }
                ++ci_n;
            }
        }
        if (!ok) { *abort_flag = 1; if (tid == 0) report(ds, HSA_ERR_TIMEOUT, kKAttendTc, 7, ci_n); }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMma) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ host side
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2D bf16 map: inner dim `cols` (contiguous), outer `rows`; box 64 x box_rows, 128B swizzle
bool make_map(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// query rows of d = 128 as a 3D view (64 columns, rows, 2 halves of 128 bytes);
// box = 8 rows x both halves, stored half after half (2 KB, 128B swizzle)
bool make_map_q3(CUtensorMap *m, const void *base, uint64_t rows) {
    EncodeTiledFn enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[3] = {64, rows, 2};
    cuuint64_t strides[2] = {256, 128};
    cuuint32_t box[3] = {64, 8, 2};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int G>
cudaError_t launch_tc(const Shape &sh, const AttendPlan &plan, const int32_t *entries, const float *entw,
                      const void *q, const void *k, const void *v, __half *acc, void *o, float *lse, DevStatus *ds,
                      cudaStream_t st) {
    CUtensorMap mq, mk, mv;
    const bool qok = D == 128 ? make_map_q3(&mq, q, (uint64_t)sh.B * sh.L * sh.hq)
                              : make_map(&mq, q, D, (uint64_t)sh.B * sh.L * sh.hq, G);
    if (!qok ||
        !make_map(&mk, k, D, (uint64_t)sh.B * sh.hkv * sh.L, 64) ||
        !make_map(&mv, v, D, (uint64_t)sh.B * sh.hkv * sh.L, 64))
        return cudaErrorInvalidValue;
    const size_t smem = Smem<D>::ALLOC;
    cudaError_t e = set_smem_once((const void *)attend_tc_kernel<D, G>, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    attend_tc_kernel<D, G><<<sms, kThreads, smem, st>>>(mq, mk, mv, plan, entries, entw, acc,
                                                        (__nv_bfloat16 *)o, lse, ds, wait_limit_ns());
    return cudaGetLastError();
}

}  // namespace


// max|v| over the value tensor (bf16, length a multiple of 8), as float bits
// max-ed into *bits: non-negative floats order like their bit patterns.
__global__ void __launch_bounds__(256) vmax_kernel(const __nv_bfloat16 *__restrict__ v, int64_t n8,
                                                   int32_t *__restrict__ bits) {
    float m = 0.f;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        const uint4 raw = __ldcs(reinterpret_cast<const uint4 *>(v) + i);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(h[e]);
            m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0) atomicMax(bits, __float_as_int(m));
}

cudaError_t launch_vmax(const Shape &sh, const void *v, int32_t *bits, cudaStream_t st) {
    const int64_t n8 = (int64_t)sh.B * sh.hkv * sh.L * sh.d / 8;
    if (n8 == 0) return cudaSuccess;
    const int blocks = (int)std::min<int64_t>(ceil_div(n8, 256), 148 * 4);
    vmax_kernel<<<blocks, 256, 0, st>>>((const __nv_bfloat16 *)v, n8, bits);
    return cudaGetLastError();
}

// max over (token, group) rows of sum_k |w_k| over the row's non-empty slots,
// as float bits max-ed into *bits.  Stick-breaking weights sum to at most 1;
// a caller-given selection may not, and the accumulators' scale takes it in.
__global__ void __launch_bounds__(256) wsum_kernel(const int32_t *__restrict__ idx, const float *__restrict__ w,
                                                   int64_t rows, int K, int32_t *__restrict__ bits) {
    float m = 0.f;
    for (int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; r < rows; r += (int64_t)gridDim.x * blockDim.x) {
        float s = 0.f;
        for (int kk = 0; kk < K; ++kk)
            if (idx[r * K + kk] >= 0) s += fabsf(w[r * K + kk]);
        m = fmaxf(m, s);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0) atomicMax(bits, __float_as_int(m));
}

cudaError_t launch_wsum(const Shape &sh, const int32_t *idx, const float *w, int32_t *bits, cudaStream_t st) {
    const int64_t rows = (int64_t)sh.B * sh.L * sh.hkv;
    if (rows == 0) return cudaSuccess;
    const int blocks = (int)std::min<int64_t>(ceil_div(rows, 256), 148 * 4);
    wsum_kernel<<<blocks, 256, 0, st>>>(idx, w, rows, sh.K, bits);
    return cudaGetLastError();
}

bool attend_tc_supported(const Shape &sh) {
    return sh.bf16 && sh.S == kChunk && (sh.d == 64 || sh.d == 128) && (sh.G == 8 || sh.G == 16) &&
           sh.K <= 16 && get_encode() != nullptr;
}

cudaError_t launch_attend_tc(const Shape &sh, const AttendPlan &plan, const int32_t *entries, const float *entw,
                             const void *q, const void *k, const void *v, __half *acc, void *o, float *lse,
                             DevStatus *ds, cudaStream_t st) {
    if (sh.d == 128 && sh.G == 8) return launch_tc<128, 8>(sh, plan, entries, entw, q, k, v, acc, o, lse, ds, st);
    if (sh.d == 128 && sh.G == 16) return launch_tc<128, 16>(sh, plan, entries, entw, q, k, v, acc, o, lse, ds, st);
    if (sh.d == 64 && sh.G == 8) return launch_tc<64, 8>(sh, plan, entries, entw, q, k, v, acc, o, lse, ds, st);
    if (sh.d == 64 && sh.G == 16) return launch_tc<64, 16>(sh, plan, entries, entw, q, k, v, acc, o, lse, ds, st);
    return cudaErrorInvalidValue;
}

}  // namespace hsa
