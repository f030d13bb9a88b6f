// swa_decode_noalloc: the split-K decode step with its scratch in a static
// device array instead of a caller-provided workspace.
//
// Who needs it: callers that cannot call cudaMalloc (or any allocator) when
// they decode -- a plain C host program with no allocator of its own, a
// plugin running inside a runtime that owns all device memory and does not
// let its extensions allocate, or a latency-critical serving loop where an
// allocation could block on the device.  They pass inputs and outputs only.
//
// The scratch is one fixed array, kScratchBytes long, that exists on every GPU
// which loads this library, for the life of the process.  All calls share it:
// two calls whose kernels overlap on the GPU (different streams, or different
// host threads on one device) race on it and give wrong results.  Each call
// writes every partial record it later reads, so nothing needs clearing
// between calls; the array simply keeps the last call's contents.
#include <cuda_runtime.h>
#include <math.h>

#include <mutex>

#include "swa.h"
#include "swa_internal.h"

namespace {

// 16 MiB: the 64-sequence, 32-head, d=128, W=4096 decode needs 8.5 MB.
constexpr size_t kScratchBytes = 16u << 20;
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// The device address of g_decode_scratch on the current device.  Host code
// only sees a host-side stand-in for the array, so the address has to be
// queried once per device, with that device current.
swa_status scratch_for_current_device(float **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SWA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return SWA_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = static_cast<float *>(g_scratch_ptr[dev]);
    return SWA_OK;
}

}  // namespace

extern "C" swa_status swa_decode_noalloc(const void *q, const void *k_cache, const void *v_cache, void *o, float *lse,
                                         const int32_t *pos, int B, int Hq, int Hkv, int d, int W, float scale,
                                         swa_dtype dt, void *stream)
{
    SWA_NVTX_RANGE("swa_decode_noalloc");
    if (dt != SWA_DTYPE_BF16 && dt != SWA_DTYPE_F32) return SWA_ERR_INVALID_ARG;
    if (B < 0 || Hq < 1 || Hkv < 1 || W < 1 || d < 1 || Hq % Hkv != 0) return SWA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !isfinite(scale)) return SWA_ERR_INVALID_ARG;
    const int G = Hq / Hkv;
    if (d != 32 && d != 64 && d != 128) return SWA_ERR_UNSUPPORTED;
    if (G != 1 && G != 2 && G != 4 && G != 8) return SWA_ERR_UNSUPPORTED;
    // the one size limit: the split partials must fit the static array
    if (swa::decode_workspace_bytes(B, Hq, Hkv, d, W) > kScratchBytes) return SWA_ERR_UNSUPPORTED;
    if (B == 0) return SWA_OK;
    const uintptr_t a16 = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k_cache) |
                          reinterpret_cast<uintptr_t>(v_cache) | reinterpret_cast<uintptr_t>(o);
    if (!q || !k_cache || !v_cache || !o || !pos || (a16 & 15) || (reinterpret_cast<uintptr_t>(pos) & 3) ||
        (lse && (reinterpret_cast<uintptr_t>(lse) & 3)))
        return SWA_ERR_INVALID_ARG;

    swa::DecodeArgs a{};
    a.q = q; a.kc = k_cache; a.vc = v_cache; a.o = o; a.lse = lse; a.pos = pos;
    a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.d = d; a.W = W;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.splits = swa::decode_splits(B, Hq, Hkv, d, W);
    swa_status st = scratch_for_current_device(&a.partial);
    if (st != SWA_OK) return st;
    if (swa::device_ctl(&a.ctl) != 0) return SWA_ERR_CUDA;
    const cudaError_t e = swa::launch_decode(dt == SWA_DTYPE_BF16, a, static_cast<cudaStream_t>(stream));
    if (e == cudaSuccess) return SWA_OK;
    return e == cudaErrorInvalidValue ? SWA_ERR_INVALID_ARG : SWA_ERR_CUDA;
}
