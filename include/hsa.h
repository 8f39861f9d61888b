/*
 * hsa.h -- C ABI of the B200 (sm_100a) Hierarchical Sparse Attention library.
 *
 * Cited pages:
 *   [P1] "Hardware-aligned Hierarchical Sparse Attention for Efficient
 *        Long-term Memory Access" -- paper notes (papernotes.org); sections
 *        "层次化稀疏注意力（HSA）" (HSA), "硬件对齐 Kernel" (kernel),
 *        "训练与推理优化" (training / inference), "局限与展望" (limitations).
 *   [P3] "Hardware-aligned Hierarchical Sparse Attention for Efficient
 *        Long-term Memory Access" -- AI summary (atlas.scime.ai), "Approach"
 *        and "Measured effects".
 *
 * What is computed (conventions the pages leave open are marked "conv."):
 *   pool    kbar[b,g,c,:] = mean of the S keys of chunk c      [P1 §HSA]
 *   select  s[t,g,c] = q_slc[t,g,:] . kbar[g,c,:] / sqrt(d) over the chunks
 *           c < floor(t/S) (conv.: a chunk is eligible when it ends at or
 *           before the start of t's own chunk); top-K per (token, KV group)
 *           [P1 §HSA "Chunk Selection"], ties toward the higher index (conv.);
 *           the chosen chunks listed most-recent-first (conv.) with
 *           stick-breaking weights w_k = sig(s_k) prod_{j<k} (1 - sig(s_j))
 *           [P1 §HSA second stage].  Empty slots: idx = -1, w = 0.
 *   fwd     for each query head h of group g = floor(h / (h_q/h_kv)) and slot
 *           k (chunk c): x_i = q[t,h] . k[g,cS+i] / sqrt(d), softmax-off-by-one
 *           p_i = e^{x_i} / (1 + sum_j e^{x_j}) [P1 §kernel],
 *           O_k = sum_i p_i v[g,cS+i]; o[t,h] = sum_k w_k O_k  [P1 §HSA, §kernel].
 *           Tokens of chunk 0 select nothing and output 0.
 *           lse[t,h,k] = log(1 + sum_i e^{x_i}) (0 for empty slots).
 *   decode  one new token at position P against a cache of P tokens and its
 *           chunk index [P1 §training/inference "KV Cache Offloading"]: the
 *           forward row t = P.
 *   bwd     gradients of sum(dO * o) w.r.t. q, k, v, q_slc; two phases as in
 *           [P1 §kernel]: per token (dq, dw -> dq_slc and dkbar through the
 *           stick-breaking weights [P1 §HSA "end-to-end"]), then per chunk over
 *           the inverted token->chunk lists (dk, dv); dk includes dkbar / S
 *           from the pooling.  The top-K choice itself carries no gradient.
 *
 * Layouts (row-major, contiguous; n_c = floor(L/S)):
 *   q, o, dO, dq        [B, L, h_q, d]
 *   q_slc, dq_slc       [B, L, h_kv, d]
 *   k, v, dk, dv        [B, h_kv, L, d]       (a chunk is S*d contiguous values)
 *   kbar                [B, h_kv, n_c, d]     always fp32
 *   idx (int32), w      [B, L, h_kv, K]       w always fp32
 *   lse                 [B, L, h_q, K]        always fp32
 *   decode: q [B,h_q,d], q_slc [B,h_kv,d], o [B,h_q,d], k/v caches
 *           [B,h_kv,P,d], kbar [B,h_kv,floor(P/S),d], idx/w [B,h_kv,K]
 *
 * Element types: shape.dtype selects fp32 (HSA_F32) or bf16 (HSA_BF16) for q,
 * k, v, q_slc, o, dO, dq, dk, dv, dq_slc.  Arithmetic is fp32 (bf16 tensor-core
 * products accumulate in fp32); outputs are rounded once, to nearest even.
 *
 * Supported shapes: S in {16, 32, 64, 128}; d in {64, 128}; 1 <= K <= 16;
 * h_q % h_kv == 0 and h_q/h_kv <= 16; B >= 1, L >= 0; every pointer 16-byte
 * aligned.  The tensor-core kernels take S = 64 (the pages' chunk size); the
 * other chunk sizes run on the CUDA-core kernels.
 *
 * Ownership: the caller owns every buffer (inputs, outputs, workspace); the
 * library never allocates, frees or synchronises -- each call only enqueues
 * kernels on `stream` (a cudaStream_t; NULL = legacy default stream) and
 * returns.  Device pointers everywhere except where a name says "host"; they
 * and `stream` belong to the calling thread's current CUDA device, which is
 * where the kernels are launched.
 *
 * Errors: arguments are checked on the host before any launch (INVALID_ARG,
 * UNSUPPORTED, WORKSPACE); a failed launch returns HSA_ERR_CUDA.  Kernels never
 * trap: a device-side problem (a bounded wait that ran out, a bad index in the
 * inputs) is written into the status word at the start of the workspace,
 * which hsa_device_status reads.  Every call clears that word first.
 */
#ifndef HSA_H
#define HSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HSA_API __attribute__((visibility("default")))
#else
#define HSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HSA_OK = 0,
    HSA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, inconsistent shape      */
    HSA_ERR_UNSUPPORTED = 2,  /* valid but not built: S or d outside the above    */
    HSA_ERR_WORKSPACE = 3,    /* ws_bytes < hsa_workspace_size(shape, op)         */
    HSA_ERR_CUDA = 4,         /* a CUDA launch or API call failed                 */
    HSA_ERR_TIMEOUT = 5,      /* device status: a bounded wait ran out            */
    HSA_ERR_DEVICE_CHECK = 6  /* device status: an input index was out of range   */
} hsa_status_t;

typedef enum { HSA_F32 = 0, HSA_BF16 = 1 } hsa_dtype_t;

typedef struct {
    int32_t B;     /* batch                                                  */
    int32_t L;     /* tokens per sequence (decode: cached prompt length P)   */
    int32_t h_q;   /* query heads                                            */
    int32_t h_kv;  /* KV heads = query groups                                */
    int32_t d;     /* head dimension                                         */
    int32_t S;     /* chunk size: 16, 32, 64 or 128 ([P1 §limitations] fixes 64) */
    int32_t K;     /* chunks selected per (token, group)                     */
    int32_t dtype; /* hsa_dtype_t of the token tensors                       */
} hsa_shape_t;

typedef enum {
    HSA_OP_POOL = 0,
    HSA_OP_SELECT = 1,
    HSA_OP_FWD = 2,
    HSA_OP_DECODE = 3,
    HSA_OP_BWD = 4
} hsa_op_t;

/* Bytes of workspace `op` needs for `shape` (0 for an invalid shape).  The
 * workspace must be 256-byte aligned; its first 256 bytes hold the status
 * word.  Contents need no initialisation and are scratch between calls. */
HSA_API size_t hsa_workspace_size(const hsa_shape_t *shape, int op);

/* Step a1: mean-pooled chunk keys [P1 §HSA "Chunk Selection"].
 * k [B,h_kv,L,d] -> kbar [B,h_kv,n_c,d] fp32; the mean is summed in fp64 and
 * rounded once to fp32.  A trailing partial chunk is not pooled. */
HSA_API hsa_status_t hsa_pool(const hsa_shape_t *shape, const void *k, float *kbar, void *ws,
                      size_t ws_bytes, void *stream);

/* Steps a1-a4: pooling, causal chunk scores, top-K, most-recent-first order,
 * stick-breaking weights [P1 §HSA].  Outputs kbar, idx, w (all required). */
HSA_API hsa_status_t hsa_select(const hsa_shape_t *shape, const void *q_slc, const void *k, float *kbar,
                        int32_t *idx, float *w, void *ws, size_t ws_bytes, void *stream);

/* Steps a1-a6: the fused forward pass [P1 §HSA, §kernel].
 * o is required.  lse (needed by hsa_bwd), idx, w and kbar are optional
 * outputs: pass NULL to keep them in the workspace. */
HSA_API hsa_status_t hsa_fwd(const hsa_shape_t *shape, const void *q, const void *k, const void *v,
                     const void *q_slc, void *o, float *lse, int32_t *idx, float *w, float *kbar,
                     void *ws, size_t ws_bytes, void *stream);

/* Steps a5-a6 for a given selection: one chunk selection shared by several
 * HSA layers [P1 §training/inference: one retrieval per step serves all HSA
 * layers].  Run hsa_select (or hsa_fwd) once, then hsa_attend per layer with
 * that layer's q, k, v.  idx [B,L,h_kv,K] int32 and w [B,L,h_kv,K] fp32 are
 * inputs in hsa_select's layout.  A negative entry is an empty slot (its
 * weight is ignored); an entry c >= 0 must satisfy c < n_c and c < t/S for
 * token t (a causal, complete chunk) -- one that does not is skipped and
 * reported as HSA_ERR_DEVICE_CHECK in the status word.  A chunk listed twice
 * for one token contributes twice.  Weights are any finite values (the fp16
 * cross-chunk sums are scaled by max|v| times the largest per-row sum of |w|).
 * o is required, lse optional (as in hsa_fwd).
 * Workspace: hsa_workspace_size(shape, HSA_OP_FWD). */
HSA_API hsa_status_t hsa_attend(const hsa_shape_t *shape, const void *q, const void *k, const void *v,
                        const int32_t *idx, const float *w, void *o, float *lse, void *ws,
                        size_t ws_bytes, void *stream);

/* Step a7: one decode step per sequence against the chunk-level index
 * [P1 §training/inference]: shape.L = P (cached tokens); the new token sits at
 * position P, so all floor(P/S) cached chunks are eligible.  kbar is an input
 * (e.g. from hsa_pool over the cache) and stays in device memory.  idx and w
 * are optional outputs.
 * KV cache offloading [P1 §training/inference "KV Cache Offloading"]:
 * k_cache and v_cache may be device memory or page-locked host memory
 * (cudaHostAlloc / cudaHostRegister, mapped).  In host memory only the K
 * selected chunks per (sequence, group) cross the host link, each read once,
 * straight into the attending thread block's shared memory.  Pageable host
 * memory is refused with HSA_ERR_INVALID_ARG before any launch. */
HSA_API hsa_status_t hsa_decode(const hsa_shape_t *shape, const void *q, const void *q_slc,
                        const void *k_cache, const void *v_cache, const float *kbar, void *o,
                        int32_t *idx, float *w, void *ws, size_t ws_bytes, void *stream);

/* Most layers one hsa_decode_multi call serves. */
#define HSA_MAX_LAYERS 8

/* hsa_decode for n_layers HSA layers that share one chunk selection and one
 * KV cache [P1 §training/inference: all HSA layers share the retrieval and the
 * single host-device exchange of a step; P3 "Measured effects" reports the
 * cost of not sharing].  q and o are [n_layers, B, h_q, d] (layer-major); the
 * selection comes from q_slc, k_cache, v_cache and kbar as in hsa_decode and
 * each selected chunk is read once for all layers.  1 <= n_layers <=
 * HSA_MAX_LAYERS, else HSA_ERR_INVALID_ARG.  hsa_decode is n_layers = 1.
 * Workspace: hsa_workspace_size(shape, HSA_OP_DECODE). */
HSA_API hsa_status_t hsa_decode_multi(const hsa_shape_t *shape, int32_t n_layers, const void *q,
                              const void *q_slc, const void *k_cache, const void *v_cache,
                              const float *kbar, void *o, int32_t *idx, float *w, void *ws,
                              size_t ws_bytes, void *stream);

/* Steps a8-a10: backward of hsa_fwd [P1 §kernel, §HSA "end-to-end"].
 * Inputs: the forward's inputs, its lse, idx, w and kbar outputs, and dO.
 * Outputs (all required, the token dtype): dq, dk, dv, dq_slc. */
HSA_API hsa_status_t hsa_bwd(const hsa_shape_t *shape, const void *q, const void *k, const void *v,
                     const void *q_slc, const void *dO, const float *lse, const int32_t *idx,
                     const float *w, const float *kbar, void *dq, void *dk, void *dv,
                     void *dq_slc, void *ws, size_t ws_bytes, void *stream);

/* hsa_fwd without a caller-provided workspace.  The source pages have no
 * counterpart to this call; it exists for callers that cannot allocate device
 * memory where they run the forward pass -- e.g. a plug-in inside an inference
 * runtime that owns all device allocations and forbids cudaMalloc to its
 * plug-ins, or a latency-critical loop where cudaMalloc/cudaFree (which may
 * synchronise the device) is not allowed.  Inputs and outputs are passed as in
 * hsa_fwd (o required; lse, idx, w, kbar optional).  Scratch comes from one
 * fixed 32 MiB device array owned by the library (held by each GPU that loads
 * it until process exit); a problem whose scratch would exceed it -- status
 * word plus kbar, idx, w for those not supplied -- returns HSA_ERR_WORKSPACE
 * without launching.  The first call on a device looks the array's address up
 * (make it before any stream capture).  All calls on a device share the array:
 * calls that may overlap on the GPU race and must not be issued.  It runs the
 * token-major CUDA-core kernel sequence and allocates nothing.  Its status
 * word lives in the library's array, which hsa_device_status cannot read; no
 * device-side check of this sequence can fire (the indices it checks are the
 * ones its own selection wrote, and its kernels have no bounded waits). */
HSA_API hsa_status_t hsa_fwd_noalloc(const hsa_shape_t *shape, const void *q, const void *k,
                                     const void *v, const void *q_slc, void *o, float *lse,
                                     int32_t *idx, float *w, float *kbar, void *stream);

/* Synchronises `stream`, then reads the device status word of workspace `ws`
 * into *code_out (an hsa_status_t value; HSA_OK when nothing went wrong). */
HSA_API hsa_status_t hsa_device_status(const void *ws, int32_t *code_out, void *stream);

/* Testing aid for the failure path.  Every wait inside the library's persistent
 * kernels (the chunk-major attention, the tensor-core selection and the
 * tensor-core backward) is bounded by `ns` nanoseconds of wall-clock time; 0
 * restores the default bound of 2 s.  A wait that runs out makes the kernel
 * record HSA_ERR_TIMEOUT in the status word, stop its work, let the copies and
 * MMAs it has issued finish (these waits keep the 2 s bound), free its tensor
 * memory and return: nothing traps and the device stays usable.  The outputs
 * of that call are undefined; the next call starts clean.  The value is
 * process-wide (all threads and devices) and read when a kernel is launched;
 * it returns HSA_OK. */
HSA_API hsa_status_t hsa_set_wait_limit_ns(uint64_t ns);

/* Kernel timing, a profiling aid.  While enabled, each kernel (or fixed group
 * of kernels) this library launches is bracketed by a pair of CUDA events
 * recorded on the launching stream; hsa_timing_read waits for the recorded
 * events and returns the summed elapsed time and the number of kernel
 * launches per kind.  Timing is process-wide host state; enabling it clears
 * the previous records.  Off by default. */
typedef enum {
    HSA_K_POOL = 1,        /* mean pooling                                   */
    HSA_K_SELECT = 2,      /* scores + top-K + stick-breaking                */
    HSA_K_ATTEND_SIMT = 3, /* token-major attention (CUDA cores)             */
    HSA_K_DECODE = 4,      /* decode step                                    */
    HSA_K_BWD1 = 5,        /* backward phase 1 (per token)                   */
    HSA_K_INVERT = 6,      /* token->chunk list inversion (4 launches)       */
    HSA_K_BWD2 = 7,        /* backward phase 2 (per chunk) + finishing pass  */
    HSA_K_ATTEND_TC = 8,   /* chunk-major attention (tcgen05)                */
    HSA_K_PLAN = 9,        /* chunk-major work planning                      */
    HSA_K_BWD_TC = 10,     /* chunk-major backward (tcgen05): dq, dw, dk, dv */
    HSA_K_BWD_SEL = 11,    /* stick-breaking backward + finishing pass       */
    HSA_K_COUNT = 16
} hsa_kernel_t;

HSA_API hsa_status_t hsa_timing_enable(int on);
HSA_API hsa_status_t hsa_timing_read(int kind, double *total_ms, int64_t *launches);

/* Static description of a status code. */
HSA_API const char *hsa_status_string(int32_t code);

#ifdef __cplusplus
}
#endif

#endif /* HSA_H */
