// The C ABI declared in include/swa.h: argument checks (host only, before any
// CUDA call), kernel selection and launch on the caller's stream, and the
// per-device status word that device-side failures are recorded in.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "swa.h"
#include "swa_internal.h"

// Written by kernels (atomicMax of SWA_STATUS_*), read and cleared by
// swa_get_device_status.  One instance per device context.
__device__ int g_swa_status;

namespace {

constexpr int kMaxDevices = 64;
unsigned long long g_wait_limit_ns = 2000000000ull;

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

swa_status status_ptr(int **out)
{
    static int *addr[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SWA_ERR_CUDA;
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_swa_status) != cudaSuccess) return SWA_ERR_CUDA;
        addr[dev] = static_cast<int *>(p);
    }
    *out = addr[dev];
    return SWA_OK;
}

swa_status ctl(swa::DeviceCtl *c)
{
    c->limit_ns = g_wait_limit_ns;
    return status_ptr(&c->status);
}

swa_status from_cuda(cudaError_t e)
{
    if (e == cudaSuccess) return SWA_OK;
    if (e == cudaErrorInvalidValue) return SWA_ERR_INVALID_ARG;
    return SWA_ERR_CUDA;
}

size_t elt_size(swa_dtype dt) { return dt == SWA_DTYPE_BF16 ? 2 : 4; }

// log2(page_size) for a paged ring of W slots: page_size a power of two that
// divides W; -1 otherwise.
int page_shift_of(int page_size, int W)
{
    if (page_size < 1 || (page_size & (page_size - 1)) != 0 || W % page_size != 0) return -1;
    int sh = 0;
    while ((1 << sh) < page_size) ++sh;
    return sh;
}

bool valid_dtype(swa_dtype dt) { return dt == SWA_DTYPE_BF16 || dt == SWA_DTYPE_F32; }

// Shared checks of the prefill calls.
swa_status check_prefill(const void *q, const void *k, const void *v, const void *o, const float *lse, int B, int T,
                         int Hq, int Hkv, int d, int W, float scale, swa_dtype dt)
{
    if (!valid_dtype(dt)) return SWA_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || Hq < 1 || Hkv < 1 || W < 1 || d < 1) return SWA_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return SWA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !isfinite(scale)) return SWA_ERR_INVALID_ARG;
    if (T > (1 << 28)) return SWA_ERR_UNSUPPORTED;
    if (B == 0 || T == 0) return SWA_OK;
    if (!q || !k || !v || !o) return SWA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16)) return SWA_ERR_INVALID_ARG;
    if (lse && !aligned(lse, 4)) return SWA_ERR_INVALID_ARG;
    if (dt == SWA_DTYPE_BF16) {
        if (d != 32 && d != 64 && d != 128) return SWA_ERR_UNSUPPORTED;
    } else {
        if (d > 128 || d % 4 != 0) return SWA_ERR_UNSUPPORTED;
    }
    return SWA_OK;
}

// Workspace layout of a dilated prefill: per residue group, the permuted q,
// k, v, o and (when asked for) lse, each at a 256-byte boundary.
struct DilatedPlan {
    int ng = 0;
    swa::DilateGroup g[2];
    size_t q[2], k[2], v[2], o[2], l[2];
    size_t total = 0;
};

DilatedPlan dilated_plan(int B, int T, int Hq, int Hkv, int d, int dil, swa_dtype dt, bool with_lse)
{
    DilatedPlan p;
    const int a = T % dil, lo = T / dil;
    const int row16 = (int)(d * elt_size(dt) / 16);
    auto add = [&](int r0, int n, int L) {
        if (n <= 0 || L <= 0) return;
        swa::DilateGroup g{B, T, 0, row16, dil, r0, n, L};
        const size_t rows = (size_t)B * n * L;
        auto take = [&](size_t bytes) {
            const size_t off = p.total;
            p.total += (bytes + 255) / 256 * 256;
            return off;
        };
        const size_t rb = (size_t)d * elt_size(dt);
        p.q[p.ng] = take(rows * Hq * rb);
        p.k[p.ng] = take(rows * Hkv * rb);
        p.v[p.ng] = take(rows * Hkv * rb);
        p.o[p.ng] = take(rows * Hq * rb);
        p.l[p.ng] = with_lse ? take(rows * Hq * sizeof(float)) : 0;
        p.g[p.ng++] = g;
    };
    add(0, a, lo + 1);      // residues with one row more
    add(a, dil - a, lo);
    return p;
}

}  // namespace

int swa::device_ctl(swa::DeviceCtl *c) { return ctl(c) == SWA_OK ? 0 : 1; }

extern "C" {

const char *swa_status_string(swa_status s)
{
    switch (s) {
    case SWA_OK: return "ok";
    case SWA_ERR_INVALID_ARG: return "invalid argument";
    case SWA_ERR_UNSUPPORTED: return "unsupported configuration";
    case SWA_ERR_CUDA: return "CUDA error";
    case SWA_ERR_TIMEOUT: return "device wait timed out";
    case SWA_ERR_INTERNAL: return "device consistency check failed (debug build)";
    }
    return "unknown status";
}

void swa_set_wait_limit_ns(unsigned long long ns) { g_wait_limit_ns = ns > 0 ? ns : 1; }

swa_status swa_prefill(const void *q, const void *k, const void *v, void *o, float *lse, int B, int T, int Hq,
                       int Hkv, int d, int W, float scale, swa_dtype dt, void *stream)
{
    SWA_NVTX_RANGE("swa_prefill");
    swa_status st = check_prefill(q, k, v, o, lse, B, T, Hq, Hkv, d, W, scale, dt);
    if (st != SWA_OK || B == 0 || T == 0) return st;
    const int left = W - 1 < T ? W - 1 : T;  // a window wider than T is T
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dt == SWA_DTYPE_F32) {
        swa::F32PrefillArgs a{static_cast<const float *>(q), static_cast<const float *>(k),
                              static_cast<const float *>(v), static_cast<float *>(o), lse, B, T, Hq, Hkv, d, left, 0,
                              nullptr, 0, scale};
        return from_cuda(swa::launch_prefill_f32(a, s));
    }
    swa::TcPrefillArgs a{};
    a.B = B; a.T = T; a.Hq = Hq; a.Hkv = Hkv;
    a.left = left; a.right = 0;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.lse = lse; a.gidx = nullptr; a.g = 0;
    a.q = q; a.k = k; a.v = v; a.o = o;
    if ((st = ctl(&a.ctl)) != SWA_OK) return st;
    return from_cuda(swa::launch_prefill_tc(d, 0, a, swa::RingArgs{}, s));
}

swa_status swa_prefill_global(const void *q, const void *k, const void *v, void *o, float *lse,
                              const int32_t *global_idx, int g, int B, int T, int Hq, int Hkv, int d, int W,
                              float scale, swa_dtype dt, void *stream)
{
    SWA_NVTX_RANGE("swa_prefill_global");
    swa_status st = check_prefill(q, k, v, o, lse, B, T, Hq, Hkv, d, W, scale, dt);
    if (st != SWA_OK) return st;
    if (g < 0 || g > T) return SWA_ERR_INVALID_ARG;
    if (g > 0 && (!global_idx || !aligned(global_idx, 4))) return SWA_ERR_INVALID_ARG;
    if (B == 0 || T == 0) return SWA_OK;
    const int half = W / 2 < T ? W / 2 : T;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dt == SWA_DTYPE_F32) {
        swa::F32PrefillArgs a{static_cast<const float *>(q), static_cast<const float *>(k),
                              static_cast<const float *>(v), static_cast<float *>(o), lse, B, T, Hq, Hkv, d, half,
                              half, g > 0 ? global_idx : nullptr, g, scale};
        return from_cuda(swa::launch_prefill_f32(a, s));
    }
    swa::TcPrefillArgs a{};
    a.B = B; a.T = T; a.Hq = Hq; a.Hkv = Hkv;
    a.left = half; a.right = half;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.lse = lse; a.gidx = g > 0 ? global_idx : nullptr; a.g = g;
    a.q = q; a.k = k; a.v = v; a.o = o;
    if ((st = ctl(&a.ctl)) != SWA_OK) return st;
    return from_cuda(swa::launch_prefill_tc(d, 0, a, swa::RingArgs{}, s));
}

size_t swa_prefill_backward_workspace_bytes(int B, int T, int Hq)
{
    if (B <= 0 || T <= 0 || Hq < 1) return 0;
    return ((size_t)B * T * Hq * sizeof(float) + 255) & ~(size_t)255;
}

swa_status swa_prefill_backward(const void *q, const void *k, const void *v, const void *o, const float *lse,
                                const void *dout, void *dq, void *dk, void *dv, int symmetric, int B, int T, int Hq,
                                int Hkv, int d, int W, float scale, swa_dtype dt, void *workspace,
                                size_t workspace_bytes, void *stream)
{
    SWA_NVTX_RANGE("swa_prefill_backward");
    if (!valid_dtype(dt)) return SWA_ERR_INVALID_ARG;
    if (symmetric != 0 && symmetric != 1) return SWA_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || Hq < 1 || Hkv < 1 || d < 1 || W < 1 || Hq % Hkv != 0) return SWA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !isfinite(scale)) return SWA_ERR_INVALID_ARG;
    if (dt != SWA_DTYPE_BF16 || (d != 64 && d != 128)) return SWA_ERR_UNSUPPORTED;
    if ((long long)B * T * Hq > (1LL << 31) || Hq > 65535 || B > 65535) return SWA_ERR_UNSUPPORTED;
    if (B == 0 || T == 0) return SWA_OK;
    const void *p16[] = {q, k, v, o, dout, dq, dk, dv, workspace};
    for (const void *p : p16)
        if (!p || !aligned(p, 16)) return SWA_ERR_INVALID_ARG;
    if (!lse || !aligned(lse, 4)) return SWA_ERR_INVALID_ARG;
    if (workspace_bytes < swa_prefill_backward_workspace_bytes(B, T, Hq)) return SWA_ERR_INVALID_ARG;
    swa::BwdArgs a{};
    a.q = q; a.k = k; a.v = v; a.o = o; a.dout = dout; a.lse = lse;
    a.delta = static_cast<float *>(workspace);
    a.dq = dq; a.dk = dk; a.dv = dv;
    a.B = B; a.T = T; a.Hq = Hq; a.Hkv = Hkv;
    if (symmetric) {
        a.left = a.right = W / 2 < T ? W / 2 : T;
    } else {
        a.left = W - 1 < T ? W - 1 : T;
        a.right = 0;
    }
    a.scale = scale;
    a.scale_log2 = scale * 1.4426950408889634f;
    swa_status st = ctl(&a.ctl);
    if (st != SWA_OK) return st;
    return from_cuda(swa::launch_prefill_backward(d, a, static_cast<cudaStream_t>(stream)));
}

size_t swa_prefill_dilated_workspace_bytes(int B, int T, int Hq, int Hkv, int d, int dil, swa_dtype dt, int with_lse)
{
    if (!valid_dtype(dt) || B <= 0 || T <= 0 || Hq < 1 || Hkv < 1 || d < 1 || dil <= 1) return 0;
    return dilated_plan(B, T, Hq, Hkv, d, dil, dt, with_lse != 0).total;
}

swa_status swa_prefill_dilated(const void *q, const void *k, const void *v, void *o, float *lse, int dil,
                               int symmetric, int B, int T, int Hq, int Hkv, int d, int W, float scale, swa_dtype dt,
                               void *workspace, size_t workspace_bytes, void *stream)
{
    SWA_NVTX_RANGE("swa_prefill_dilated");
    swa_status st = check_prefill(q, k, v, o, lse, B, T, Hq, Hkv, d, W, scale, dt);
    if (st != SWA_OK) return st;
    if (dil < 1 || (symmetric != 0 && symmetric != 1)) return SWA_ERR_INVALID_ARG;
    if (B == 0 || T == 0) return SWA_OK;
    if (dil == 1)
        return symmetric ? swa_prefill_global(q, k, v, o, lse, nullptr, 0, B, T, Hq, Hkv, d, W, scale, dt, stream)
                         : swa_prefill(q, k, v, o, lse, B, T, Hq, Hkv, d, W, scale, dt, stream);
    const DilatedPlan p = dilated_plan(B, T, Hq, Hkv, d, dil, dt, lse != nullptr);
    if (!workspace || workspace_bytes < p.total || !aligned(workspace, 256)) return SWA_ERR_INVALID_ARG;
    if ((long long)B * dil > (1 << 30)) return SWA_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    swa::DeviceCtl c;
    if ((st = ctl(&c)) != SWA_OK) return st;
    for (int i = 0; i < p.ng; ++i) {
        swa::DilateGroup gq = p.g[i], gk = p.g[i];
        gq.H = Hq;
        gk.H = Hkv;
        cudaError_t e;
        if ((e = swa::launch_dilate_rows(q, ws + p.q[i], gq, 1, s)) != cudaSuccess) return from_cuda(e);
        if ((e = swa::launch_dilate_rows(k, ws + p.k[i], gk, 1, s)) != cudaSuccess) return from_cuda(e);
        if ((e = swa::launch_dilate_rows(v, ws + p.v[i], gk, 1, s)) != cudaSuccess) return from_cuda(e);
        // the sub-sequences as a batch of B*n sequences of L rows
        const int Bg = B * gq.n, L = gq.L;
        const int left = symmetric ? (W / 2 < L ? W / 2 : L) : (W - 1 < L ? W - 1 : L);
        const int right = symmetric ? left : 0;
        float *lse_g = lse ? reinterpret_cast<float *>(ws + p.l[i]) : nullptr;
        if (dt == SWA_DTYPE_F32) {
            swa::F32PrefillArgs a{reinterpret_cast<const float *>(ws + p.q[i]), reinterpret_cast<const float *>(ws + p.k[i]),
                                  reinterpret_cast<const float *>(ws + p.v[i]), reinterpret_cast<float *>(ws + p.o[i]),
                                  lse_g, Bg, L, Hq, Hkv, d, left, right, nullptr, 0, scale};
            e = swa::launch_prefill_f32(a, s);
        } else {
            swa::TcPrefillArgs a{};
            a.B = Bg; a.T = L; a.Hq = Hq; a.Hkv = Hkv;
            a.left = left; a.right = right;
            a.scale_log2 = scale * 1.4426950408889634f;
            a.lse = lse_g; a.gidx = nullptr; a.g = 0;
            a.q = ws + p.q[i]; a.k = ws + p.k[i]; a.v = ws + p.v[i]; a.o = ws + p.o[i];
            a.ctl = c;
            e = swa::launch_prefill_tc(d, 0, a, swa::RingArgs{}, s);
        }
        if (e != cudaSuccess) return from_cuda(e);
        if ((e = swa::launch_dilate_rows(ws + p.o[i], o, gq, 0, s)) != cudaSuccess) return from_cuda(e);
        if (lse) {
            gq.H = Hq;
            if ((e = swa::launch_dilate_lse(lse_g, lse, gq, s)) != cudaSuccess) return from_cuda(e);
        }
    }
    return SWA_OK;
}

swa_status swa_prefill_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                              const int32_t *cu_seqlens, const int32_t *windows, int nseq, int total, int max_seqlen,
                              int Hq, int Hkv, int d, int W, float scale, swa_dtype dt, void *stream)
{
    SWA_NVTX_RANGE("swa_prefill_varlen");
    swa_status st = check_prefill(q, k, v, o, lse, 1, total, Hq, Hkv, d, W, scale, dt);
    if (st != SWA_OK) return st;
    if (nseq < 0 || max_seqlen < 0 || max_seqlen > total) return SWA_ERR_INVALID_ARG;
    if (nseq == 0 || total == 0 || max_seqlen == 0) return SWA_OK;
    if (!cu_seqlens || !aligned(cu_seqlens, 4)) return SWA_ERR_INVALID_ARG;
    if (windows && !aligned(windows, 4)) return SWA_ERR_INVALID_ARG;
    // with one window per sequence, `left` is the bound every window is
    // clipped to (a window wider than the longest sequence is the whole
    // sequence)
    const int left = windows ? max_seqlen : (W - 1 < max_seqlen ? W - 1 : max_seqlen);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dt == SWA_DTYPE_F32) {
        swa::F32PrefillArgs a{static_cast<const float *>(q), static_cast<const float *>(k),
                              static_cast<const float *>(v), static_cast<float *>(o), lse, 1, total, Hq, Hkv, d, left, 0,
                              nullptr, 0, scale};
        a.cu = cu_seqlens;
        a.nseq = nseq;
        a.wseq = windows;
        if (windows && (st = ctl(&a.ctl)) != SWA_OK) return st;
        return from_cuda(swa::launch_prefill_f32(a, s));
    }
    swa::TcPrefillArgs a{};
    a.B = nseq; a.T = total; a.Hq = Hq; a.Hkv = Hkv;
    a.left = left; a.right = 0;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.lse = lse; a.gidx = nullptr; a.g = 0;
    a.q = q; a.k = k; a.v = v; a.o = o;
    if ((st = ctl(&a.ctl)) != SWA_OK) return st;
    return from_cuda(swa::launch_prefill_varlen(d, a, swa::VarlenArgs{cu_seqlens, max_seqlen, windows}, s));
}

swa_status swa_prefill_sinks(const void *q, const void *k, const void *v, void *o, float *lse, int n_sink, int B,
                             int T, int Hq, int Hkv, int d, int W, float scale, swa_dtype dt, void *stream)
{
    SWA_NVTX_RANGE("swa_prefill_sinks");
    swa_status st = check_prefill(q, k, v, o, lse, B, T, Hq, Hkv, d, W, scale, dt);
    if (st != SWA_OK) return st;
    if (n_sink < 0) return SWA_ERR_INVALID_ARG;
    if (B == 0 || T == 0) return SWA_OK;
    if (n_sink > T) n_sink = T;
    const int left = W - 1 < T ? W - 1 : T;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dt == SWA_DTYPE_F32) {
        // null global positions with g > 0: the first g positions are sinks
        swa::F32PrefillArgs a{static_cast<const float *>(q), static_cast<const float *>(k),
                              static_cast<const float *>(v), static_cast<float *>(o), lse, B, T, Hq, Hkv, d, left, 0,
                              nullptr, n_sink, scale};
        return from_cuda(swa::launch_prefill_f32(a, s));
    }
    swa::TcPrefillArgs a{};
    a.B = B; a.T = T; a.Hq = Hq; a.Hkv = Hkv;
    a.left = left; a.right = 0;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.lse = lse; a.gidx = nullptr; a.g = n_sink;
    a.q = q; a.k = k; a.v = v; a.o = o;
    if ((st = ctl(&a.ctl)) != SWA_OK) return st;
    return from_cuda(swa::launch_prefill_tc(d, 0, a, swa::RingArgs{}, s));
}

swa_status swa_prefill_chunk(const void *q, const void *k, const void *v, void *o, float *lse, const void *k_cache,
                             const void *v_cache, const int32_t *pos, int B, int n, int Hq, int Hkv, int d, int W,
                             float scale, swa_dtype dt, void *stream)
{
    SWA_NVTX_RANGE("swa_prefill_chunk");
    swa_status st = check_prefill(q, k, v, o, lse, B, n, Hq, Hkv, d, W, scale, dt);
    if (st != SWA_OK || B == 0 || n == 0) return st;
    if (!k_cache || !v_cache || !pos) return SWA_ERR_INVALID_ARG;
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(pos, 4)) return SWA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dt == SWA_DTYPE_F32) {
        swa::F32PrefillArgs a{static_cast<const float *>(q), static_cast<const float *>(k),
                              static_cast<const float *>(v), static_cast<float *>(o), lse, B, n, Hq, Hkv, d, W - 1, 0,
                              nullptr, 0, scale};
        a.pos = pos;
        a.kc = static_cast<const float *>(k_cache);
        a.vc = static_cast<const float *>(v_cache);
        a.W_ring = W;
        if ((st = ctl(&a.ctl)) != SWA_OK) return st;
        return from_cuda(swa::launch_prefill_f32(a, s));
    }
    swa::TcPrefillArgs a{};
    a.B = B; a.T = n; a.Hq = Hq; a.Hkv = Hkv;
    a.left = W - 1; a.right = 0;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.lse = lse; a.gidx = nullptr; a.g = 0;
    a.q = q; a.k = k; a.v = v; a.o = o;
    if ((st = ctl(&a.ctl)) != SWA_OK) return st;
    return from_cuda(swa::launch_prefill_tc(d, 0, a, swa::RingArgs{pos, k_cache, v_cache, W}, s));
}

swa_status swa_cache_append(void *k_cache, void *v_cache, const void *k_new, const void *v_new, const int32_t *pos,
                            int32_t *slot_out, int B, int n, int Hkv, int d, int W, swa_dtype dt, void *stream)
{
    SWA_NVTX_RANGE("swa_cache_append");
    if (!valid_dtype(dt)) return SWA_ERR_INVALID_ARG;
    if (B < 0 || n < 0 || Hkv < 1 || d < 1 || W < 1) return SWA_ERR_INVALID_ARG;
    if ((d * elt_size(dt)) % 16 != 0) return SWA_ERR_UNSUPPORTED;
    if (B == 0 || n == 0) return SWA_OK;
    if (!k_cache || !v_cache || !k_new || !v_new || !pos) return SWA_ERR_INVALID_ARG;
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(k_new, 16) || !aligned(v_new, 16) ||
        !aligned(pos, 4) || (slot_out && !aligned(slot_out, 4)))
        return SWA_ERR_INVALID_ARG;
    swa::AppendArgs a{k_cache, v_cache, k_new, v_new, pos, slot_out, B, n, Hkv, W,
                      static_cast<int>(d * elt_size(dt)), {}};
    swa_status st = ctl(&a.ctl);
    if (st != SWA_OK) return st;
    return from_cuda(swa::launch_append(a, static_cast<cudaStream_t>(stream)));
}

swa_status swa_cache_append_paged(void *k_pages, void *v_pages, const void *k_new, const void *v_new,
                                  const int32_t *pos, const int32_t *page_table, int32_t *slot_out, int B, int n,
                                  int Hkv, int d, int W, int page_size, int num_pages, swa_dtype dt, void *stream)
{
    SWA_NVTX_RANGE("swa_cache_append_paged");
    if (!valid_dtype(dt)) return SWA_ERR_INVALID_ARG;
    if (B < 0 || n < 0 || Hkv < 1 || d < 1 || W < 1 || num_pages < 1) return SWA_ERR_INVALID_ARG;
    const int shift = page_shift_of(page_size, W);
    if (shift < 0) return SWA_ERR_INVALID_ARG;
    if ((d * elt_size(dt)) % 16 != 0) return SWA_ERR_UNSUPPORTED;
    if (B == 0 || n == 0) return SWA_OK;
    if (!k_pages || !v_pages || !k_new || !v_new || !pos || !page_table) return SWA_ERR_INVALID_ARG;
    if (!aligned(k_pages, 16) || !aligned(v_pages, 16) || !aligned(k_new, 16) || !aligned(v_new, 16) ||
        !aligned(pos, 4) || !aligned(page_table, 4) || (slot_out && !aligned(slot_out, 4)))
        return SWA_ERR_INVALID_ARG;
    swa::AppendArgs a{k_pages, v_pages, k_new, v_new, pos, slot_out, B, n, Hkv, W,
                      static_cast<int>(d * elt_size(dt)), {}, page_table, shift, num_pages};
    swa_status st = ctl(&a.ctl);
    if (st != SWA_OK) return st;
    return from_cuda(swa::launch_append(a, static_cast<cudaStream_t>(stream)));
}

size_t swa_decode_workspace_bytes(int B, int Hq, int Hkv, int d, int W)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || d < 1 || W < 1 || Hq % Hkv) return 0;
    return swa::decode_workspace_bytes(B, Hq, Hkv, d, W);
}

}  // extern "C"

namespace {

// swa_decode, swa_decode_sinks (n_sink = 0: no sinks) and swa_decode_paged
// (page_table not null: k_cache / v_cache are page pools).
swa_status decode_impl(const void *q, const void *k_cache, const void *v_cache, const void *k_sink,
                       const void *v_sink, int n_sink, void *o, float *lse, const int32_t *pos, int B, int Hq, int Hkv,
                       int d, int W, float scale, swa_dtype dt, void *workspace, size_t workspace_bytes, void *stream,
                       const int32_t *page_table = nullptr, int page_size = 0, int num_pages = 0)
{
    if (!valid_dtype(dt)) return SWA_ERR_INVALID_ARG;
    if (n_sink < 0) return SWA_ERR_INVALID_ARG;
    if (B < 0 || Hq < 1 || Hkv < 1 || W < 1 || d < 1 || Hq % Hkv != 0) return SWA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !isfinite(scale)) return SWA_ERR_INVALID_ARG;
    const int G = Hq / Hkv;
    if (d != 32 && d != 64 && d != 128) return SWA_ERR_UNSUPPORTED;
    if (G != 1 && G != 2 && G != 4 && G != 8) return SWA_ERR_UNSUPPORTED;
    if (B == 0) return SWA_OK;
    if (!q || !k_cache || !v_cache || !o || !pos) return SWA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) || !aligned(pos, 4) ||
        (lse && !aligned(lse, 4)))
        return SWA_ERR_INVALID_ARG;
    const size_t need = swa::decode_workspace_bytes(B, Hq, Hkv, d, W);
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 16))) return SWA_ERR_INVALID_ARG;
    swa::DecodeArgs a{};
    a.q = q; a.kc = k_cache; a.vc = v_cache; a.o = o; a.lse = lse; a.pos = pos;
    a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.d = d; a.W = W;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.splits = swa::decode_splits(B, Hq, Hkv, d, W);
    a.partial = static_cast<float *>(workspace);
    if (n_sink > 0) {
        if (!k_sink || !v_sink || !aligned(k_sink, 16) || !aligned(v_sink, 16)) return SWA_ERR_INVALID_ARG;
        a.ks = k_sink; a.vs = v_sink; a.n_sink = n_sink;
    }
    if (page_table) {
        if (!aligned(page_table, 4)) return SWA_ERR_INVALID_ARG;
        a.ptable = page_table;
        a.page_shift = page_shift_of(page_size, W);
        a.num_pages = num_pages;
    }
    swa_status st = ctl(&a.ctl);
    if (st != SWA_OK) return st;
    return from_cuda(swa::launch_decode(dt == SWA_DTYPE_BF16, a, static_cast<cudaStream_t>(stream)));
}

}  // namespace

extern "C" {

swa_status swa_decode(const void *q, const void *k_cache, const void *v_cache, void *o, float *lse,
                      const int32_t *pos, int B, int Hq, int Hkv, int d, int W, float scale, swa_dtype dt,
                      void *workspace, size_t workspace_bytes, void *stream)
{
    SWA_NVTX_RANGE("swa_decode");
    return decode_impl(q, k_cache, v_cache, nullptr, nullptr, 0, o, lse, pos, B, Hq, Hkv, d, W, scale, dt, workspace,
                       workspace_bytes, stream);
}

swa_status swa_decode_sinks(const void *q, const void *k_cache, const void *v_cache, const void *k_sink,
                            const void *v_sink, int n_sink, void *o, float *lse, const int32_t *pos, int B, int Hq,
                            int Hkv, int d, int W, float scale, swa_dtype dt, void *workspace, size_t workspace_bytes,
                            void *stream)
{
    SWA_NVTX_RANGE("swa_decode_sinks");
    return decode_impl(q, k_cache, v_cache, k_sink, v_sink, n_sink, o, lse, pos, B, Hq, Hkv, d, W, scale, dt,
                       workspace, workspace_bytes, stream);
}

swa_status swa_decode_paged(const void *q, const void *k_pages, const void *v_pages, const int32_t *page_table,
                            void *o, float *lse, const int32_t *pos, int B, int Hq, int Hkv, int d, int W,
                            int page_size, int num_pages, float scale, swa_dtype dt, void *workspace,
                            size_t workspace_bytes, void *stream)
{
    SWA_NVTX_RANGE("swa_decode_paged");
    if (W < 1 || num_pages < 1 || page_shift_of(page_size, W) < 0) return SWA_ERR_INVALID_ARG;
    if (B > 0 && !page_table) return SWA_ERR_INVALID_ARG;
    return decode_impl(q, k_pages, v_pages, nullptr, nullptr, 0, o, lse, pos, B, Hq, Hkv, d, W, scale, dt, workspace,
                       workspace_bytes, stream, B > 0 ? page_table : nullptr, page_size, num_pages);
}

swa_status swa_mask_export(uint8_t *mask, int T, int W, int symmetric, const int32_t *global_idx, int g,
                           void *stream)
{
    SWA_NVTX_RANGE("swa_mask_export");
    if (T < 0 || T > 65536 || W < 1 || (symmetric != 0 && symmetric != 1)) return SWA_ERR_INVALID_ARG;
    if (g < 0 || g > T || (g > 0 && !symmetric)) return SWA_ERR_INVALID_ARG;
    if (T == 0) return SWA_OK;
    if (!mask || (g > 0 && (!global_idx || !aligned(global_idx, 4)))) return SWA_ERR_INVALID_ARG;
    int left, right;
    if (symmetric) {
        left = right = (W / 2 < T ? W / 2 : T);
    } else {
        left = W - 1 < T ? W - 1 : T;
        right = 0;
    }
    return from_cuda(
        swa::launch_mask_export(mask, T, left, right, g > 0 ? global_idx : nullptr, g, static_cast<cudaStream_t>(stream)));
}

swa_status swa_get_device_status(void *stream)
{
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SWA_ERR_CUDA;
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_swa_status, sizeof(int)) != cudaSuccess) return SWA_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_swa_status, &zero, sizeof(int)) != cudaSuccess) return SWA_ERR_CUDA;
    if (v >= SWA_STATUS_TIMEOUT) return SWA_ERR_TIMEOUT;
    if (v == SWA_STATUS_DEBUG_CHECK) return SWA_ERR_INTERNAL;
    if (v == SWA_STATUS_BAD_INPUT) return SWA_ERR_INVALID_ARG;
    return SWA_OK;
}

swa_status swa_debug_expire_wait(int timeout_us, void *stream)
{
    if (timeout_us < 1 || timeout_us > 10000000) return SWA_ERR_INVALID_ARG;
    swa::DeviceCtl c{};
    swa_status st = status_ptr(&c.status);
    if (st != SWA_OK) return st;
    c.limit_ns = static_cast<unsigned long long>(timeout_us) * 1000ull;
    return from_cuda(swa::launch_debug_expire_wait(c, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
