// hsa_noalloc.cu -- a forward entry point that needs no caller-provided workspace.
//
// Who needs it: callers that cannot allocate device memory where they run the
// forward pass.  Examples are plug-ins hosted inside an inference runtime that
// owns every device allocation and does not let its plug-ins call cudaMalloc,
// and latency-critical loops where an allocation (cudaMalloc/cudaFree may
// synchronise the whole device) is not acceptable.  They still pass their
// inputs and outputs; everything else the forward pass needs lives in one
// fixed array of device memory that belongs to this library.
//
// The scratch array: a file-scope __device__ variable of kNoAllocScratchBytes
// (32 MiB), 256-byte aligned.  Each GPU that loads this code keeps those bytes
// until the process exits.  Host code must not use the variable's name as a
// pointer (on the host it only names a stand-in): the device address is looked
// up once per device with cudaGetSymbolAddress, with that device current, the
// first time hsa_fwd_noalloc runs on it.  Make that first call on a device
// before any stream capture.
//
// Sharing: every call on a device uses the same array and leaves its contents
// behind.  Calls that overlap on the GPU (different streams, or different host
// threads, without ordering between them) race on it and must not be issued.
// Each call clears the status word at the start of the array; the other
// scratch regions are written in full before they are read.  No caller can
// read that status word (hsa_device_status takes a caller's workspace), and
// none of this sequence's device-side checks can fire: the chunk indices the
// attention checks are the ones the same call's selection just wrote, and
// these kernels contain no bounded waits.
//
// Kernel sequence: the same launchers as the forward pass -- pooling, chunk
// selection, token-major chunk attention with stick-breaking fusion -- with
// the workspace regions (status word, pooled keys, chunk indices and weights)
// carved from the array.  It makes no cudaMalloc, cudaFree or other allocating
// call.
#include <mutex>

#include "hsa_internal.cuh"

namespace hsa {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 256;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices];

// Device address of the scratch array on the current device (looked up once).
cudaError_t noalloc_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return cudaSuccess;
}

size_t r256(size_t n) { return (n + 255) / 256 * 256; }

bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
}  // namespace

}  // namespace hsa

extern "C" HSA_API hsa_status_t hsa_fwd_noalloc(const hsa_shape_t *shape, const void *q,
                                                const void *k, const void *v, const void *q_slc,
                                                void *o, float *lse, int32_t *idx, float *w,
                                                float *kbar, void *stream) {
    using namespace hsa;
    const hsa_status_t chk = check_shape(shape, false);  // the same validation as hsa_fwd
    if (chk != HSA_OK) return chk;
    const hsa_shape_t &s = *shape;
    const Shape sh = make_shape(s);
    // scratch needed: status word, plus each intermediate the caller did not ask for
    const size_t kbar_b = r256(sizeof(float) * (size_t)sh.B * sh.hkv * sh.nc * sh.d);
    const size_t sel_b = r256(sizeof(float) * (size_t)sh.B * sh.L * sh.hkv * sh.K);
    const size_t need = kWsHeader + (kbar ? 0 : kbar_b) + (idx ? 0 : sel_b) + (w ? 0 : sel_b);
    if (need > kNoAllocScratchBytes) return HSA_ERR_WORKSPACE;  // beyond the fixed 32 MiB array
    const bool empty = (int64_t)sh.B * sh.L == 0;
    if (!empty && (!q || !k || !v || !q_slc || !o || !al16(q) || !al16(k) || !al16(v) ||
                   !al16(q_slc) || !al16(o)))
        return HSA_ERR_INVALID_ARG;
    if (!al16(lse) || !al16(idx) || !al16(w) || !al16(kbar)) return HSA_ERR_INVALID_ARG;

    void *base = nullptr;
    if (noalloc_scratch(&base) != cudaSuccess) return HSA_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    DevStatus *ds = static_cast<DevStatus *>(base);
    cudaError_t e = cudaMemsetAsync(ds, 0, sizeof(DevStatus), st);
    if (e != cudaSuccess || empty) return e == cudaSuccess ? HSA_OK : HSA_ERR_CUDA;
    char *p = static_cast<char *>(base) + kWsHeader;
    float *kb = kbar;
    if (!kb) { kb = reinterpret_cast<float *>(p); p += kbar_b; }
    int32_t *ix = idx;
    if (!ix) { ix = reinterpret_cast<int32_t *>(p); p += sel_b; }
    float *wt = w;
    if (!wt) { wt = reinterpret_cast<float *>(p); p += sel_b; }
    {
        TimedLaunch tl(HSA_K_POOL, 1, st);
        e = launch_pool(sh, k, kb, ds, st);
    }
    if (e == cudaSuccess) {
        TimedLaunch tl(HSA_K_SELECT, 1, st);
        e = launch_select_simt(sh, q_slc, kb, ix, wt, ds, st);
    }
    if (e == cudaSuccess) {
        TimedLaunch tl(HSA_K_ATTEND_SIMT, 1, st);
        e = launch_attend_simt(sh, q, k, v, ix, wt, o, lse, ds, st);
    }
    return e == cudaSuccess ? HSA_OK : HSA_ERR_CUDA;
}
