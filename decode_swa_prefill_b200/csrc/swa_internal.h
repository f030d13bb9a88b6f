// Internal declarations shared by the C-ABI layer and the kernel files.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include <nvtx3/nvToolsExt.h>

// A named NVTX range around one C-ABI call, so a timeline (Nsight Systems,
// ncu's NVTX filters) shows which call launched which kernels.  NVTX v3 is
// header-only; without a tool attached each push/pop is a cheap no-op.
struct SwaNvtxRange {
    explicit SwaNvtxRange(const char *name) { nvtxRangePushA(name); }
    ~SwaNvtxRange() { nvtxRangePop(); }
    SwaNvtxRange(const SwaNvtxRange &) = delete;
    SwaNvtxRange &operator=(const SwaNvtxRange &) = delete;
};
#define SWA_NVTX_RANGE(name) SwaNvtxRange swa_nvtx_range_(name)

// Device status word values (ordered: the worst one wins via atomicMax).
#define SWA_STATUS_OK 0
#define SWA_STATUS_BAD_INPUT 1
#define SWA_STATUS_DEBUG_CHECK 2
#define SWA_STATUS_TIMEOUT 4

// Device-side consistency checks of tile, row and slot indices, compiled in
// only by the debug build (-DSWA_DEBUG, libswa_debug.so).  A failed check
// records SWA_STATUS_DEBUG_CHECK in the status word (read by
// swa_get_device_status as SWA_ERR_INTERNAL); it never traps.  In the release
// build the checks compile to nothing.
#ifdef SWA_DEBUG
#define SWA_DCHECK(cond, status)                                                                                      \
    do {                                                                                                              \
        if (!(cond)) atomicMax((status), SWA_STATUS_DEBUG_CHECK);                                                     \
    } while (0)
#else
#define SWA_DCHECK(cond, status)                                                                                      \
    do {                                                                                                              \
    } while (0)
#endif

namespace swa {

// Key j is visible to query i when i-left <= j <= i+right (both in [0,T)).
// Causal window W: left = W-1, right = 0.  Symmetric window W: left = right
// = W/2.  Global tokens are handled by the callers (see the kernels).
__host__ __device__ __forceinline__ bool band_contains(long long i, long long j, int left, int right)
{
    return j >= i - left && j <= i + right;
}

// One-time setup per device of a kernel launcher (kernel attributes, the SM
// count), safe when several host threads launch on the same device: the
// first call for a device runs init(dev, &n_sm) under a mutex, later calls
// read the stored SM count under the same mutex.
class DeviceOnce {
  public:
    template <typename F>
    cudaError_t get(F init, int *n_sm_out)
    {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= kMax) return cudaErrorInvalidDevice;
        std::lock_guard<std::mutex> lock(mu_);
        if (!done_[dev]) {
            int n = 0;
            if ((e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
            if ((e = init(dev)) != cudaSuccess) return e;
            n_sm_[dev] = n;
            done_[dev] = true;
        }
        if (n_sm_out) *n_sm_out = n_sm_[dev];
        return cudaSuccess;
    }

  private:
    static constexpr int kMax = 64;
    std::mutex mu_;
    bool done_[kMax] = {};
    int n_sm_[kMax] = {};
};

struct DeviceCtl {
    int *status;                 // device status word
    unsigned long long limit_ns; // bounded-wait limit
};

// ---- tcgen05 prefill (band rows, optional gathered global keys; or dense
//      global rows) ----
struct TcPrefillArgs {
    int B, T, Hq, Hkv;
    int left, right;          // band of visible keys around each query
    float scale_log2;         // softmax scale * log2(e)
    float *lse;               // [B,Hq,T] or null
    const int32_t *gidx;      // [B,g] global positions or null
    int g;
    const void *q, *k, *v;    // raw pointers (gathers)
    void *o;                  // raw output pointer (scatter in global-row mode)
    DeviceCtl ctl;
};

// A chunk continuing a ring (band mode): T is the chunk length n, query row r
// of batch b is at position pos[b]+r, and keys before pos[b] come from the
// W-slot caches kc / vc [B,Hkv,W,d].  A separate kernel argument, so that the
// other launches keep their argument layout.
struct RingArgs {
    const int32_t *pos;       // null: no ring
    const void *kc, *vc;
    int W;
};

// mode 0: one CTA per (q tile, head, batch) over band tiles (+ one gathered
//         tile of global keys per 128 globals when gidx != null)
// mode 1: one CTA per (128 global rows, head, batch): dense rows over all keys
cudaError_t launch_prefill_tc(int d, int mode, const TcPrefillArgs &a, const RingArgs &ring, cudaStream_t s);

// Causal window of at most 64 keys (left <= 63, right 0, no global keys or
// sinks), d = 32 or 64: persistent single-pass kernel whose S tile holds
// every key a 128-row query tile sees.
bool prefill_narrow_applies(int d, const TcPrefillArgs &a);
cudaError_t launch_prefill_narrow(int d, const TcPrefillArgs &a, cudaStream_t s);

// ---- backward pass of the window prefill (bf16, d = 64 or 128) ----
struct BwdArgs {
    const void *q, *k, *v, *o, *dout;   // [B,T,Hq,d] / [B,T,Hkv,d]
    const float *lse;                   // [B,Hq,T] natural log, from the forward pass
    float *delta;                       // [B,Hq,T] scratch: dout_i . o_i
    void *dq, *dk, *dv;                 // outputs, bf16
    int B, T, Hq, Hkv;
    int left, right;                    // window: keys i-left .. i+right
    float scale, scale_log2;
    DeviceCtl ctl;
};
cudaError_t launch_prefill_backward(int d, const BwdArgs &a, cudaStream_t s);

// Band prefill with 128-key tiles and the two query tiles in alternation (no
// global keys, sinks or packed sequences; optionally a chunk continuing a
// ring, ring.pos not null): d = 32, 64 or 128 and windows of at least 256
// keys.
bool prefill_pp_applies(int d, const TcPrefillArgs &a);
cudaError_t launch_prefill_pp(int d, const TcPrefillArgs &a, const RingArgs &ring, cudaStream_t s);

// Packed variable-length sequences (causal band mode): q/k/v/o are
// [total,H,d] (TcPrefillArgs.T = total, B = number of sequences) and
// sequence b holds rows cu[b] .. cu[b+1]-1, none longer than max_len.
struct VarlenArgs {
    const int32_t *cu;        // device [B+1]
    int max_len;
    const int32_t *wseq;      // device [B]: window of each sequence, or null (TcPrefillArgs.left for all)
};
cudaError_t launch_prefill_varlen(int d, const TcPrefillArgs &a, const VarlenArgs &vl, cudaStream_t s);

// Is packed sequence b's entry consistent (offsets inside the rows and
// non-decreasing, length at most max_len, window at least 1)?
__device__ __forceinline__ bool varlen_ok(const VarlenArgs &vl, int b, int total)
{
    const int c0 = vl.cu[b], c1 = vl.cu[b + 1];
    return c0 >= 0 && c1 >= c0 && c1 <= total && c1 - c0 <= vl.max_len && (!vl.wseq || vl.wseq[b] >= 1);
}

// Keys before the query a row of packed sequence b sees: its own window's
// (clipped to the longest sequence, like the call's single window), or the
// call's.
__device__ __forceinline__ int varlen_left(const VarlenArgs &vl, int b, int left)
{
    return vl.wseq ? min(max(vl.wseq[b], 1) - 1, vl.max_len) : left;
}

// The same calls on the 128-key kernel (prefill_pp.cu): d = 32, 64 or 128
// and a call window (or, with one window per sequence, a longest sequence)
// of at least 256 keys.
bool prefill_pp_varlen_applies(int d, const TcPrefillArgs &a, const VarlenArgs &vl);
cudaError_t launch_prefill_pp_varlen(int d, const TcPrefillArgs &a, const VarlenArgs &vl, cudaStream_t s);

// ---- SIMT kernels ----
// Attention sinks in the prefill calls: gidx == null with g > 0 means the
// first g positions of each sequence are keys every later query sees
// (causal window only).
struct F32PrefillArgs {
    const float *q, *k, *v;
    float *o, *lse;
    int B, T, Hq, Hkv, d;
    int left, right;
    const int32_t *gidx;
    int g;
    float scale;
    // chunk continuing a ring (causal only), as in TcPrefillArgs
    const int32_t *pos;
    const float *kc, *vc;
    int W_ring;
    DeviceCtl ctl;
    // packed sequences (B == 1, T = total rows): sequence s holds rows
    // cu[s] .. cu[s+1]-1 (null: one sequence per batch row), with window
    // wseq[s] when wseq is not null (left = wseq[s]-1 instead of `left`)
    const int32_t *cu;
    int nseq;
    const int32_t *wseq;
};
cudaError_t launch_prefill_f32(const F32PrefillArgs &a, cudaStream_t s);

struct DecodeArgs {
    const void *q, *kc, *vc;
    void *o;
    float *lse;
    const int32_t *pos;
    int B, Hq, Hkv, d, W;
    float scale_log2;
    float *partial;           // [B,Hq,S,d+2] when S > 1
    int splits;
    DeviceCtl ctl;
    // attention sinks beside the ring: [B,Hkv,n_sink,d] caches of positions
    // 0..n_sink-1 (n_sink = 0: none)
    const void *ks, *vs;
    int n_sink;
    // paged ring (ptable not null): kc / vc are pools [num_pages,Hkv,P,d]
    // with P = 2^page_shift; ring slot s of sequence b is row s mod P of
    // page ptable[b*(W/P) + s/P]
    const int32_t *ptable;
    int page_shift, num_pages;
};
int decode_splits(int B, int Hq, int Hkv, int d, int W);
size_t decode_workspace_bytes(int B, int Hq, int Hkv, int d, int W);
cudaError_t launch_decode(int dtype_bf16, const DecodeArgs &a, cudaStream_t s);

struct AppendArgs {
    void *kc, *vc;
    const void *kn, *vn;
    const int32_t *pos;
    int32_t *slot_out;
    int B, n, Hkv, W;
    int row_bytes;            // d * element size
    DeviceCtl ctl;
    // paged ring, as in DecodeArgs (null: dense [B,Hkv,W,d] caches)
    const int32_t *ptable;
    int page_shift, num_pages;
};
cudaError_t launch_append(const AppendArgs &a, cudaStream_t s);

cudaError_t launch_mask_export(uint8_t *mask, int T, int left, int right, const int32_t *gidx, int g,
                               cudaStream_t s);

cudaError_t launch_debug_expire_wait(const DeviceCtl &ctl, cudaStream_t s);

// ---- dilated window: residue-major sub-sequence permutations ----
// Group of residues r0 .. r0+n-1 of a [B,T,H,...] tensor, each a sub-sequence
// of L rows at positions r0 + rr + t*dil.
struct DilateGroup {
    int B, T, H;
    int row16;   // 16-byte units per row (row bytes / 16)
    int dil, r0, n, L;
};
cudaError_t launch_dilate_rows(const void *src, void *dst, const DilateGroup &g, int to_group, cudaStream_t s);
cudaError_t launch_dilate_lse(const float *src, float *dst, const DilateGroup &g, cudaStream_t s);

// Fills the current device's status-word address and the wait limit; 0 on
// success.
int device_ctl(DeviceCtl *c);

}  // namespace swa
