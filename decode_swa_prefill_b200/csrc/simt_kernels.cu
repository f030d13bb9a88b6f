// SIMT kernels: mask export, ring-cache append, fp32 prefill, split-K decode
// over the ring with its LSE merge, and the bounded-wait test hook.
#include <cuda_bf16.h>
#include <math_constants.h>

#include <type_traits>

#include "ptx.cuh"
#include "swa_internal.h"

namespace swa {
namespace {

// Is position x one of the g sorted global positions?
__device__ __forceinline__ bool is_global_pos(const int32_t *gidx, int g, long long x)
{
    int lo = 0, hi = g;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (gidx[mid] < x) lo = mid + 1;
        else hi = mid;
    }
    return lo < g && gidx[lo] == x;
}

// --------------------------------------------------------- mask export --
// One byte per (i, j), from the band predicate the prefill kernels use plus
// the global-token rule (robocikowo.com binary-mask and global-token entries).
__global__ void mask_export_kernel(uint8_t *mask, int T, int left, int right, const int32_t *gidx, int g)
{
    const long long n = (long long)T * T;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n;
         idx += (long long)gridDim.x * blockDim.x) {
        const long long i = idx / T, j = idx % T;
        bool ok = band_contains(i, j, left, right);
        if (!ok && g > 0) ok = is_global_pos(gidx, g, i) || is_global_pos(gidx, g, j);
        mask[idx] = ok ? 1 : 0;
    }
}

// --------------------------------------------------------- cache append --
// Token t of row b goes to slot (pos[b]+t) mod W (Ultralytics ring-buffer
// paragraph); with n > W only the last W tokens are copied, so no two
// threads write one slot.  16-byte units.  A paged ring keeps slot s of
// sequence b in row s mod P of page ptable[b][s/P] of the pool; a page outside
// the pool is reported in the status word and its token is not written.
__global__ void append_kernel(AppendArgs a)
{
    const int upr = a.row_bytes / 16;
    const int n_eff = min(a.n, a.W);
    const int t0 = a.n - n_eff;
    const long long total = (long long)a.B * n_eff * a.Hkv * upr;
    const long long stride = (long long)gridDim.x * blockDim.x;
    const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (a.slot_out) {
        for (long long idx = tid; idx < (long long)a.B * a.n; idx += stride) {
            const int b = (int)(idx / a.n), t = (int)(idx % a.n);
            const long long p = a.pos[b];
            a.slot_out[idx] = p < 0 ? -1 : (int32_t)((p + t) % a.W);
        }
    }
    for (long long idx = tid; idx < total; idx += stride) {
        const int u = (int)(idx % upr);
        long long rest = idx / upr;
        const int hk = (int)(rest % a.Hkv);
        rest /= a.Hkv;
        const int t = t0 + (int)(rest % n_eff);
        const int b = (int)(rest / n_eff);
        const long long p = a.pos[b];
        if (p < 0) {
            if (u == 0 && hk == 0) atomicMax(a.ctl.status, SWA_STATUS_BAD_INPUT);
            continue;
        }
        const long long slot = (p + t) % a.W;
        SWA_DCHECK(slot >= 0 && slot < a.W && t >= 0 && t < a.n, a.ctl.status);
        long long row;  // destination row of the cache or pool
        if (a.ptable) {
            const int pg = a.ptable[(long long)b * (a.W >> a.page_shift) + (slot >> a.page_shift)];
            if ((unsigned)pg >= (unsigned)a.num_pages) {
                if (u == 0) atomicMax(a.ctl.status, SWA_STATUS_BAD_INPUT);
                continue;
            }
            row = (((long long)pg * a.Hkv + hk) << a.page_shift) + (slot & ((1LL << a.page_shift) - 1));
        } else {
            row = ((long long)b * a.Hkv + hk) * a.W + slot;
        }
        const long long src = (((long long)b * a.n + t) * a.Hkv + hk) * a.row_bytes + u * 16;
        const long long dst = row * a.row_bytes + u * 16;
        const uint4 kv = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(a.kn) + src));
        const uint4 vv = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(a.vn) + src));
        *reinterpret_cast<uint4 *>(static_cast<uint8_t *>(a.kc) + dst) = kv;
        *reinterpret_cast<uint4 *>(static_cast<uint8_t *>(a.vc) + dst) = vv;
    }
}

// --------------------------------------------------------- fp32 prefill --
// One warp per query row, fp32 FMA throughout (no TF32), accurate expf.
// Keys: the band [i-left, i+right]; for a global row every key; for other
// rows also the global keys outside the band.
constexpr int F32_ROWS_PER_CTA = 4;

__global__ void __launch_bounds__(32 * F32_ROWS_PER_CTA)
    prefill_f32_kernel(F32PrefillArgs a)
{
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int i = blockIdx.x * F32_ROWS_PER_CTA + warp;
    const int h = blockIdx.y, b = blockIdx.z;
    if (i >= a.T) return;
    const int hk = h / (a.Hq / a.Hkv);
    const int32_t *gb = a.gidx ? a.gidx + (long long)b * a.g : nullptr;
    const bool row_global = gb && is_global_pos(gb, a.g, i);
    constexpr int EPL = 4; // d <= 128
    float q[EPL], acc[EPL];
    const float *qrow = a.q + (((long long)b * a.T + i) * a.Hq + h) * a.d;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
        const int c = lane + 32 * e;
        q[e] = c < a.d ? qrow[c] : 0.f;
        acc[e] = 0.f;
    }
    float m = -CUDART_INF_F, l = 0.f;
    // chunk continuing a ring: row i is at position p0 + i; positions below
    // p0 are read from ring slot (position mod W_ring)
    long long p0 = 0;
    if (a.pos) {
        p0 = a.pos[b];
        if (p0 < 0) {
            if (lane == 0 && i == 0 && h == 0) atomicMax(a.ctl.status, SWA_STATUS_BAD_INPUT);
            p0 = 0;
        }
    }
    auto visit = [&](long long j) {
        const float *krow, *vrow;
        if (j >= p0) {
            krow = a.k + (((long long)b * a.T + (j - p0)) * a.Hkv + hk) * a.d;
            vrow = a.v + (((long long)b * a.T + (j - p0)) * a.Hkv + hk) * a.d;
        } else {
            const long long sl = j % a.W_ring;
            krow = a.kc + (((long long)b * a.Hkv + hk) * a.W_ring + sl) * a.d;
            vrow = a.vc + (((long long)b * a.Hkv + hk) * a.W_ring + sl) * a.d;
        }
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
            const int c = lane + 32 * e;
            if (c < a.d) dot = fmaf(q[e], krow[c], dot);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
        const float s = dot * a.scale;
        const float mn = fmaxf(m, s);
        const float corr = expf(m - mn);
        const float p = expf(s - mn);
        l = l * corr + p;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
            const int c = lane + 32 * e;
            acc[e] = acc[e] * corr + (c < a.d ? p * vrow[c] : 0.f);
        }
        m = mn;
    };
    if (row_global) {
        for (long long j = 0; j < a.T; ++j) visit(j);
    } else {
        const long long ip = p0 + i;  // absolute position of the row
        long long first = 0, last = p0 + a.T - 1;  // the row's sequence
        int left = a.left;
        if (a.cu) {
            // packed sequences: the one holding row i (kept inside the rows
            // even for an inconsistent cu)
            int s0 = 0, s1 = a.nseq;
            while (s1 - s0 > 1) {
                const int mid = (s0 + s1) / 2;
                if (a.cu[mid] <= i) s0 = mid;
                else s1 = mid;
            }
            first = max(0LL, (long long)a.cu[s0]);
            last = min((long long)a.T - 1, (long long)a.cu[s0 + 1] - 1);
            if (a.wseq) {
                // the sequence's own window; below 1: rows left untouched,
                // reported in the status word
                const int wv = a.wseq[s0];
                if (wv < 1) {
                    if (lane == 0) atomicMax(a.ctl.status, SWA_STATUS_BAD_INPUT);
                    return;
                }
                left = (int)min((long long)wv - 1, (long long)a.left);
            }
        }
        const long long lo = max(first, ip - left);
        const long long hi = min(last, ip + a.right);
        if (!gb && a.g > 0)  // sinks older than the window
            for (long long j = 0; j < min((long long)a.g, lo); ++j) visit(j);
        for (long long j = lo; j <= hi; ++j) visit(j);
        if (gb)
            for (int c = 0; c < a.g; ++c)
                if (!band_contains(i, gb[c], a.left, a.right)) visit(gb[c]);
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float *orow = a.o + (((long long)b * a.T + i) * a.Hq + h) * a.d;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
        const int c = lane + 32 * e;
        if (c < a.d) orow[c] = acc[e] * inv;
    }
    if (a.lse && lane == 0) a.lse[((long long)b * a.Hq + h) * a.T + i] = l > 0.f ? m + logf(l) : -CUDART_INF_F;
}

// ---------------------------------------------------------------- decode --
// One CTA per (split, kv head, batch row); 4 warps.  Every query head of the
// GQA group shares the kv head's ring, so one pass over each slot serves all
// G of them.  Lane l holds elements [l*EPL, (l+1)*EPL) of a head row; a warp
// reads a whole K or V row per load (coalesced).  A batch of NB = 32/G slots
// gives NB*G = 32 partial dot products per lane; a reduce-scatter across the
// warp (31 shuffles) leaves lane L with the full score of (slot L/G, head
// L%G).  Softmax runs in log2 units with q pre-scaled by scale*log2(e).
constexpr int DEC_WARPS = 4;

template <typename T>
struct Ld;
template <>
struct Ld<__nv_bfloat16> {
    template <int EPL>
    __device__ __forceinline__ static void row(const __nv_bfloat16 *p, float *out)
    {
        if constexpr (EPL == 4) {
            const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
            out[0] = __uint_as_float(u.x << 16);
            out[1] = __uint_as_float(u.x & 0xffff0000u);
            out[2] = __uint_as_float(u.y << 16);
            out[3] = __uint_as_float(u.y & 0xffff0000u);
        } else if constexpr (EPL == 2) {
            const uint32_t u = __ldg(reinterpret_cast<const unsigned int *>(p));
            out[0] = __uint_as_float(u << 16);
            out[1] = __uint_as_float(u & 0xffff0000u);
        } else {
            const unsigned short u = __ldg(reinterpret_cast<const unsigned short *>(p));
            out[0] = __uint_as_float((uint32_t)u << 16);
        }
    }
    __device__ __forceinline__ static void store(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
};
template <>
struct Ld<float> {
    template <int EPL>
    __device__ __forceinline__ static void row(const float *p, float *out)
    {
#pragma unroll
        for (int e = 0; e < EPL; ++e) out[e] = __ldg(p + e);
    }
    __device__ __forceinline__ static void store(float *p, float x) { *p = x; }
};

// Where a decode reads its key/value rows: the dense ring, the dense ring
// plus sink caches, or a paged ring (pool + page table).
constexpr int SRC_RING = 0, SRC_SINKS = 1, SRC_PAGED = 2;

// Row (in rows of d elements) of ring slot sl of (sequence b, kv head hk) in
// a paged pool; a page outside the pool reads page 0 and sets *bad.
__device__ __forceinline__ long long paged_row(const DecodeArgs &a, const int32_t *tbl, int hk, int sl, bool *bad)
{
    int pg = __ldg(tbl + (sl >> a.page_shift));
    if ((unsigned)pg >= (unsigned)a.num_pages) {
        *bad = true;
        pg = 0;
    }
    return (((long long)pg * a.Hkv + hk) << a.page_shift) + (sl & ((1 << a.page_shift) - 1));
}

// The end of a decode CTA: merge the warps' partials (running max m in log2
// units, sum l, unnormalised accumulator) held in shared memory, then write
// o (and lse) when the (sequence, kv head) has one split, else the split's
// partial for decode_combine_kernel.  (Merging the splits inside a
// thread-block cluster through distributed shared memory instead measured
// slower: 219-238 us against 189-195 us at the 64-sequence decode workload,
// the cluster's CTAs being scheduled together and waiting for the slowest at
// the merge.)
template <typename T, int D, int G>
__device__ __forceinline__ void decode_finish(const DecodeArgs &a, int b, int hk, int split,
                                              const float (*sm_m)[G], const float (*sm_l)[G],
                                              const float (*sm_acc)[G][D])
{
    const int Hq = a.Hq;
    for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
        const int g = idx / D, e = idx % D;
        float M = -CUDART_INF_F;
#pragma unroll
        for (int w = 0; w < DEC_WARPS; ++w) M = fmaxf(M, sm_m[w][g]);
        const float Mu = M == -CUDART_INF_F ? 0.f : M;
        float L = 0.f, O = 0.f;
#pragma unroll
        for (int w = 0; w < DEC_WARPS; ++w) {
            const float f = ex2_approx(sm_m[w][g] - Mu);
            L += sm_l[w][g] * f;
            O += sm_acc[w][g][e] * f;
        }
        const int h = hk * G + g;
        if (a.splits == 1) {
            T *o = static_cast<T *>(a.o) + ((long long)b * Hq + h) * D;
            Ld<T>::store(o + e, L > 0.f ? O / L : 0.f);
            if (a.lse && e == 0)
                a.lse[(long long)b * Hq + h] = L > 0.f ? (M + __log2f(L)) * 0.69314718055994530942f : -CUDART_INF_F;
        } else {
            float *part = a.partial + (((long long)b * Hq + h) * a.splits + split) * (D + 2);
            part[e] = O;
            if (e == 0) {
                part[D] = M;
                part[D + 1] = L;
            }
        }
    }
}

template <typename T, int D, int G, int SRC>
__global__ void __launch_bounds__(32 * DEC_WARPS)
    decode_kernel(DecodeArgs a)
{
    constexpr bool SINKS = SRC == SRC_SINKS;
    constexpr bool PAGED = SRC == SRC_PAGED;
    constexpr int EPL = D / 32;
    constexpr int NB = 32 / G;
    const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int Hq = a.Hq;

    const long long p = a.pos[b];
    if (p < 0 && threadIdx.x == 0 && split == 0 && hk == 0) atomicMax(a.ctl.status, SWA_STATUS_BAD_INPUT);
    const int n_valid = p < 0 ? 0 : (int)(p + 1 < a.W ? p + 1 : a.W);
    // virtual slots: the ring's filled slots, then the sinks older than the
    // window (positions < p-W+1), which the last split takes on top of its
    // share of the ring (the ring keeps the plain decode's split boundaries)
    const int ns = SINKS ? (int)max(0LL, min((long long)a.n_sink, p - a.W + 1)) : 0;
    const int chunk = (a.W + a.splits - 1) / a.splits;
    const int s_begin = split * chunk;
    const int s_end = (SINKS && split == a.splits - 1) ? n_valid + ns : min(n_valid, s_begin + chunk);

    const T *qb = static_cast<const T *>(a.q) + ((long long)b * Hq + (long long)hk * G) * D;
    const T *kb = static_cast<const T *>(a.kc) + ((long long)b * a.Hkv + hk) * (long long)a.W * D;
    const T *vb = static_cast<const T *>(a.vc) + ((long long)b * a.Hkv + hk) * (long long)a.W * D;
    const long long sink0 = ((long long)b * a.Hkv + hk) * (long long)a.n_sink * D;
    const int32_t *tbl = PAGED ? a.ptable + (long long)b * (a.W >> a.page_shift) : nullptr;
    bool bad_page = false;
    auto krow = [&](int sl) -> const T * {
        if (SINKS && sl >= n_valid) return static_cast<const T *>(a.ks) + sink0 + (long long)(sl - n_valid) * D;
        if (PAGED) return static_cast<const T *>(a.kc) + paged_row(a, tbl, hk, sl, &bad_page) * D;
        return kb + (long long)sl * D;
    };
    auto vrow = [&](int sl) -> const T * {
        if (SINKS && sl >= n_valid) return static_cast<const T *>(a.vs) + sink0 + (long long)(sl - n_valid) * D;
        if (PAGED) return static_cast<const T *>(a.vc) + paged_row(a, tbl, hk, sl, &bad_page) * D;
        return vb + (long long)sl * D;
    };

    float q[G][EPL];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        Ld<T>::template row<EPL>(qb + g * D + lane * EPL, q[g]);
#pragma unroll
        for (int e = 0; e < EPL; ++e) q[g][e] *= a.scale_log2;
    }
    float acc[G][EPL];
    float m[G], l[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m[g] = -CUDART_INF_F;
        l[g] = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[g][e] = 0.f;
    }

    for (int base = s_begin + warp * NB; base < s_end; base += DEC_WARPS * NB) {
        float kr[NB][EPL], vr[NB][EPL];
#pragma unroll
        for (int n = 0; n < NB; ++n) {
            const int sl = min(base + n, s_end - 1); // clamp: masked below
            SWA_DCHECK(sl >= 0 && sl < (SINKS ? a.W + a.n_sink : a.W), a.ctl.status);
            Ld<T>::template row<EPL>(krow(sl) + lane * EPL, kr[n]);
            Ld<T>::template row<EPL>(vrow(sl) + lane * EPL, vr[n]);
        }
        // partial dot products, value index n*G + g
        float v[32];
#pragma unroll
        for (int n = 0; n < NB; ++n)
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float s = 0.f;
#pragma unroll
                for (int e = 0; e < EPL; ++e) s = fmaf(q[g][e], kr[n][e], s);
                v[n * G + g] = s;
            }
        // reduce-scatter: after the step with offset k, lane keeps the half
        // selected by its bit k; finally lane L holds the sum for index L
#pragma unroll
        for (int k = 16; k >= 1; k >>= 1) {
            const bool upper = (lane & k) != 0;
#pragma unroll
            for (int x = 0; x < k; ++x) {
                const float send = upper ? v[x] : v[x + k];
                const float keep = upper ? v[x + k] : v[x];
                v[x] = keep + __shfl_xor_sync(0xffffffffu, send, k);
            }
        }
        const int my_n = lane / G, my_g = lane % G;
        float sc = (base + my_n < s_end) ? v[0] : -CUDART_INF_F;
        // per-head batch max over the NB lanes sharing my_g
        float bm = sc;
#pragma unroll
        for (int k = G; k < 32; k <<= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, k));
        // running max of my head (m[] is replicated; pick mine)
        float m_old = m[0];
#pragma unroll
        for (int g = 1; g < G; ++g)
            if (my_g == g) m_old = m[g];
        const float m_new = fmaxf(m_old, bm);
        const float m_use = m_new == -CUDART_INF_F ? 0.f : m_new;
        float pr = ex2_approx(sc - m_use);
        const float al = ex2_approx(m_old - m_use);
        float ps = pr;
#pragma unroll
        for (int k = G; k < 32; k <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, k);
        // every lane gets each head's alpha, new max and batch sum
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float alg = __shfl_sync(0xffffffffu, al, g);
            const float psg = __shfl_sync(0xffffffffu, ps, g);
            m[g] = __shfl_sync(0xffffffffu, m_new, g);
            l[g] = l[g] * alg + psg;
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[g][e] *= alg;
        }
#pragma unroll
        for (int n = 0; n < NB; ++n)
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float pn = __shfl_sync(0xffffffffu, pr, n * G + g);
#pragma unroll
                for (int e = 0; e < EPL; ++e) acc[g][e] = fmaf(pn, vr[n][e], acc[g][e]);
            }
    }

    if (PAGED && bad_page) atomicMax(a.ctl.status, SWA_STATUS_BAD_INPUT);

    // merge the warps' partials in shared memory
    __shared__ float sm_m[DEC_WARPS][G], sm_l[DEC_WARPS][G];
    __shared__ float sm_acc[DEC_WARPS][G][D];
    if (lane == 0)
#pragma unroll
        for (int g = 0; g < G; ++g) {
            sm_m[warp][g] = m[g];
            sm_l[warp][g] = l[g];
        }
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < EPL; ++e) sm_acc[warp][g][lane * EPL + e] = acc[g][e];
    __syncthreads();
    decode_finish<T, D, G>(a, b, hk, split, sm_m, sm_l, sm_acc);
}

// bf16 decode with 16-byte loads (used when G <= d/8).  A row of d bf16 is
// read by LPR = d/8 lanes (8 elements, 16 bytes each), so one warp load
// covers RPW = 32/LPR consecutive ring slots.  Each lane takes NBL = LPR/G
// slots of a batch (stride RPW), giving NBL*G = LPR partial scores, which a
// reduce-scatter over the LPR lanes of its row group (log2 LPR shuffles per
// value pair) turns into one full score per lane.  q.k uses sm_100's mixed
// precision FMA (bf16 x bf16 + fp32) straight from the packed pairs; P.V
// runs as paired fp32 FMAs.  Same split-K partials as decode_kernel.
__device__ __forceinline__ float dot2_bf16(uint32_t a, uint32_t b, float c)
{
    float d;
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
        "mov.b32 {al, ah}, %1;\n\t"
        "mov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %3;\n\t"
        "fma.rn.f32.bf16 %0, ah, bh, %0;\n\t}"
        : "=f"(d)
        : "r"(a), "r"(b), "f"(c));
    return d;
}

__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w)
{
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

template <int D, int G, int SRC>
__global__ void __launch_bounds__(32 * DEC_WARPS)
    decode_bf16_kernel(DecodeArgs a)
{
    constexpr bool SINKS = SRC == SRC_SINKS;
    constexpr bool PAGED = SRC == SRC_PAGED;
    constexpr int LPR = D / 8;          // lanes per row
    constexpr int RPW = 32 / LPR;       // rows per warp load
    constexpr int NBL = LPR / G;        // slots per lane per batch
    constexpr int BATCH = NBL * RPW;    // slots per warp per batch
    static_assert(NBL >= 1 && NBL * G == LPR, "layout");
    const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int part = lane % LPR;        // which 8 elements of a row
    const int rgrp = lane / LPR;        // which row of a warp load
    const int Hq = a.Hq;

    const long long p = a.pos[b];
    if (p < 0 && threadIdx.x == 0 && split == 0 && hk == 0) atomicMax(a.ctl.status, SWA_STATUS_BAD_INPUT);
    const int n_valid = p < 0 ? 0 : (int)(p + 1 < a.W ? p + 1 : a.W);
    // virtual slots: the ring's filled slots, then the sinks older than the
    // window (positions < p-W+1), which the last split takes on top of its
    // share of the ring (the ring keeps the plain decode's split boundaries)
    const int ns = SINKS ? (int)max(0LL, min((long long)a.n_sink, p - a.W + 1)) : 0;
    const int chunk = (a.W + a.splits - 1) / a.splits;
    const int s_begin = split * chunk;
    const int s_end = (SINKS && split == a.splits - 1) ? n_valid + ns : min(n_valid, s_begin + chunk);

    const __nv_bfloat16 *qb = static_cast<const __nv_bfloat16 *>(a.q) + ((long long)b * Hq + (long long)hk * G) * D;
    const __nv_bfloat16 *kb = static_cast<const __nv_bfloat16 *>(a.kc) + ((long long)b * a.Hkv + hk) * (long long)a.W * D;
    const __nv_bfloat16 *vb = static_cast<const __nv_bfloat16 *>(a.vc) + ((long long)b * a.Hkv + hk) * (long long)a.W * D;
    const long long sink0 = ((long long)b * a.Hkv + hk) * (long long)a.n_sink * D;
    // row sources: the ring (dense, or paged through the page table), or
    // (the last split of a call with sinks) the ring and then the sink caches
    const int32_t *tbl = PAGED ? a.ptable + (long long)b * (a.W >> a.page_shift) : nullptr;
    bool bad_page = false;
    auto ring_k = [&](int sl) -> const __nv_bfloat16 * {
        if (PAGED) return static_cast<const __nv_bfloat16 *>(a.kc) + paged_row(a, tbl, hk, sl, &bad_page) * D;
        return kb + (long long)sl * D;
    };
    auto ring_v = [&](int sl) -> const __nv_bfloat16 * {
        if (PAGED) return static_cast<const __nv_bfloat16 *>(a.vc) + paged_row(a, tbl, hk, sl, &bad_page) * D;
        return vb + (long long)sl * D;
    };
    auto tail_k = [&](int sl) -> const __nv_bfloat16 * {
        if (sl >= n_valid) return static_cast<const __nv_bfloat16 *>(a.ks) + sink0 + (long long)(sl - n_valid) * D;
        return kb + (long long)sl * D;
    };
    auto tail_v = [&](int sl) -> const __nv_bfloat16 * {
        if (sl >= n_valid) return static_cast<const __nv_bfloat16 *>(a.vs) + sink0 + (long long)(sl - n_valid) * D;
        return vb + (long long)sl * D;
    };

    uint4 q[G];
#pragma unroll
    for (int g = 0; g < G; ++g) q[g] = __ldg(reinterpret_cast<const uint4 *>(qb + g * D + part * 8));
    float2 acc[G][4];
    float m[G], l[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m[g] = -CUDART_INF_F;
        l[g] = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[g][e] = make_float2(0.f, 0.f);
    }

    auto run = [&](auto krow, auto vrow) {
    for (int base = s_begin + warp * BATCH; base < s_end; base += DEC_WARPS * BATCH) {
        uint4 kr[NBL], vr[NBL];
#pragma unroll
        for (int n = 0; n < NBL; ++n) {
            const int sl = min(base + n * RPW + rgrp, s_end - 1); // clamp: masked below
            SWA_DCHECK(sl >= 0 && sl < (SINKS ? a.W + a.n_sink : a.W), a.ctl.status);
            kr[n] = __ldg(reinterpret_cast<const uint4 *>(krow(sl) + part * 8));
            vr[n] = __ldg(reinterpret_cast<const uint4 *>(vrow(sl) + part * 8));
        }
        // partial dot products over this lane's 8 elements, index n*G + g
        float v[LPR];
#pragma unroll
        for (int n = 0; n < NBL; ++n)
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float t = 0.f;
                t = dot2_bf16(q[g].x, kr[n].x, t);
                t = dot2_bf16(q[g].y, kr[n].y, t);
                t = dot2_bf16(q[g].z, kr[n].z, t);
                t = dot2_bf16(q[g].w, kr[n].w, t);
                v[n * G + g] = t;
            }
        // reduce-scatter over the LPR lanes of the row group: afterwards
        // lane part holds the full score of value index part
#pragma unroll
        for (int k = LPR / 2; k >= 1; k >>= 1) {
            const bool upper = (part & k) != 0;
#pragma unroll
            for (int x = 0; x < k; ++x) {
                const float send = upper ? v[x] : v[x + k];
                const float keep = upper ? v[x + k] : v[x];
                v[x] = keep + __shfl_xor_sync(0xffffffffu, send, k);
            }
        }
        const int my_n = part / G, my_g = part % G;
        const float sc = (base + my_n * RPW + rgrp < s_end) ? v[0] * a.scale_log2 : -CUDART_INF_F;
        // per-head batch max over the lanes holding the same head
        float bm = sc;
#pragma unroll
        for (int k = G; k < 32; k <<= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, k));
        float m_old = m[0];
#pragma unroll
        for (int g = 1; g < G; ++g)
            if (my_g == g) m_old = m[g];
        const float m_new = fmaxf(m_old, bm);
        const float m_use = m_new == -CUDART_INF_F ? 0.f : m_new;
        const float pr = ex2_approx(sc - m_use);
        const float al = ex2_approx(m_old - m_use);
        float ps = pr;
#pragma unroll
        for (int k = G; k < 32; k <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, k);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float alg = __shfl_sync(0xffffffffu, al, g);
            const float psg = __shfl_sync(0xffffffffu, ps, g);
            m[g] = __shfl_sync(0xffffffffu, m_new, g);
            l[g] = l[g] * alg + psg;
            const float2 a2 = make_float2(alg, alg);
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[g][e] = mul2(acc[g][e], a2);
        }
        // P.V for this lane's slots (probabilities from its row group)
#pragma unroll
        for (int n = 0; n < NBL; ++n) {
            const float2 v0 = bf16x2_to_float2(vr[n].x), v1 = bf16x2_to_float2(vr[n].y);
            const float2 v2 = bf16x2_to_float2(vr[n].z), v3 = bf16x2_to_float2(vr[n].w);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float pn = __shfl_sync(0xffffffffu, pr, rgrp * LPR + n * G + g);
                const float2 p2 = make_float2(pn, pn);
                acc[g][0] = fma2(p2, v0, acc[g][0]);
                acc[g][1] = fma2(p2, v1, acc[g][1]);
                acc[g][2] = fma2(p2, v2, acc[g][2]);
                acc[g][3] = fma2(p2, v3, acc[g][3]);
            }
        }
    }
    };
    if constexpr (SINKS) {
        if (split == a.splits - 1) run(tail_k, tail_v);
        else run(ring_k, ring_v);
    } else {
        run(ring_k, ring_v);
    }
    if (PAGED && bad_page) atomicMax(a.ctl.status, SWA_STATUS_BAD_INPUT);
    // sum the row groups' accumulators (same softmax reference per head)
#pragma unroll
    for (int k = LPR; k < 32; k <<= 1)
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc[g][e].x += __shfl_xor_sync(0xffffffffu, acc[g][e].x, k);
                acc[g][e].y += __shfl_xor_sync(0xffffffffu, acc[g][e].y, k);
            }

    // merge the warps' partials in shared memory
    __shared__ float sm_m[DEC_WARPS][G], sm_l[DEC_WARPS][G];
    __shared__ float sm_acc[DEC_WARPS][G][D];
    if (lane == 0)
#pragma unroll
        for (int g = 0; g < G; ++g) {
            sm_m[warp][g] = m[g];
            sm_l[warp][g] = l[g];
        }
    if (rgrp == 0)
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                sm_acc[warp][g][part * 8 + 2 * e] = acc[g][e].x;
                sm_acc[warp][g][part * 8 + 2 * e + 1] = acc[g][e].y;
            }
    __syncthreads();
    decode_finish<__nv_bfloat16, D, G>(a, b, hk, split, sm_m, sm_l, sm_acc);
}

// bf16 decode over a dense ring with the ring rows staged in shared memory.
// Same CTAs (split, kv head, sequence), same slots per warp and the same
// arithmetic as decode_bf16_kernel, but a fifth warp is a producer: each
// stage of SS = 4*BATCH consecutive slots is one contiguous run of K rows and
// one of V rows in the [B,Hkv,W,d] ring, copied with two cp.async.bulk
// (no multicast) into a ring of BULK_NST stages; the four compute warps read
// their rows from shared memory.  The bytes in flight per SM are then set by
// the stages (up to 3 CTAs x 4 stages x 16 KB) instead of the compute warps'
// registers (measured at the 64-sequence decode workload: 189 us back to
// back against 195 us for decode_bf16_kernel).  Waits are bounded
// (wait_bounded); on expiry the CTA records SWA_STATUS_TIMEOUT and the
// producer lets its own copies land before the CTA exits.
constexpr int BULK_NST = 4;
constexpr int BULK_THREADS = 32 * (DEC_WARPS + 1);

template <int D, int G>
struct BulkCfg {
    static constexpr int LPR = D / 8, RPW = 32 / LPR, NBL = LPR / G, BATCH = NBL * RPW;
    static constexpr int SS = DEC_WARPS * BATCH;   // slots per stage
    static constexpr int ROWB = D * 2;             // bytes per row
    static constexpr int STAGE = SS * ROWB;        // bytes of K (or V) per stage
    static constexpr int SMEM = 2 * BULK_NST * STAGE + 2 * BULK_NST * 8;
    static constexpr bool OK = (G <= D / 8) && STAGE <= 8192;
};

template <int D, int G, bool PAGED>
__global__ void __launch_bounds__(BULK_THREADS) decode_bulk_kernel(DecodeArgs a)
{
    using C = BulkCfg<D, G>;
    constexpr int LPR = C::LPR, RPW = C::RPW, NBL = C::NBL, BATCH = C::BATCH;
    extern __shared__ __align__(128) uint8_t dsm[];
    uint8_t *sK = dsm;
    uint8_t *sV = dsm + BULK_NST * C::STAGE;
    uint64_t *full = reinterpret_cast<uint64_t *>(dsm + 2 * BULK_NST * C::STAGE);
    uint64_t *empty = full + BULK_NST;
    __shared__ int abort_flag;
    __shared__ float sm_m[DEC_WARPS][G], sm_l[DEC_WARPS][G];
    __shared__ float sm_acc[DEC_WARPS][G][D];

    const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const long long p = a.pos[b];
    if (p < 0 && threadIdx.x == 0 && split == 0 && hk == 0) atomicMax(a.ctl.status, SWA_STATUS_BAD_INPUT);
    const int n_valid = p < 0 ? 0 : (int)(p + 1 < a.W ? p + 1 : a.W);
    const int chunk = (a.W + a.splits - 1) / a.splits;
    const int s_begin = split * chunk;
    const int s_end = min(n_valid, s_begin + chunk);
    const int n_it = s_end > s_begin ? (s_end - s_begin + C::SS - 1) / C::SS : 0;

    if (threadIdx.x == 0) {
        for (int st = 0; st < BULK_NST; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], DEC_WARPS);
        }
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    WaitCtl ctl{&abort_flag, a.ctl.status, a.ctl.limit_ns};

    if (warp == DEC_WARPS) {
        // ------------------------------------------------------ producer --
        const long long ring0 = PAGED ? 0 : ((long long)b * a.Hkv + hk) * (long long)a.W * C::ROWB;
        const uint8_t *kb = static_cast<const uint8_t *>(a.kc) + ring0;
        const uint8_t *vb = static_cast<const uint8_t *>(a.vc) + ring0;
        const int32_t *tbl = PAGED ? a.ptable + (long long)b * (a.W >> a.page_shift) : nullptr;
        bool bad_page = false;
        int iss[BULK_NST] = {};
        bool ok = true;
        for (int it = 0; it < n_it && ok; ++it) {
            const int st = it % BULK_NST;
            ok = warp_wait_bounded(&empty[st], ((it / BULK_NST) & 1) ^ 1, ctl);
            if (!ok) break;
            if (lane == 0) {
                const int s0 = s_begin + it * C::SS;
                const int rows = min(C::SS, s_end - s0);
                SWA_DCHECK(s0 >= 0 && rows > 0 && s0 + rows <= a.W, a.ctl.status);
                mbar_expect_tx(&full[st], 2u * (uint32_t)(rows * C::ROWB));
                if constexpr (PAGED) {
                    // one copy per run of slots inside one page
                    const int P = 1 << a.page_shift;
                    for (int r = 0; r < rows;) {
                        const int sl = s0 + r;
                        const int n = min(P - (sl & (P - 1)), rows - r);
                        const long long row = paged_row(a, tbl, hk, sl, &bad_page);
                        bulk_load(sK + st * C::STAGE + r * C::ROWB, kb + row * C::ROWB, (uint32_t)(n * C::ROWB),
                                  &full[st]);
                        bulk_load(sV + st * C::STAGE + r * C::ROWB, vb + row * C::ROWB, (uint32_t)(n * C::ROWB),
                                  &full[st]);
                        r += n;
                    }
                } else {
                    const uint32_t bytes = (uint32_t)(rows * C::ROWB);
                    bulk_load(sK + st * C::STAGE, kb + (long long)s0 * C::ROWB, bytes, &full[st]);
                    bulk_load(sV + st * C::STAGE, vb + (long long)s0 * C::ROWB, bytes, &full[st]);
                }
            }
            iss[st]++;
        }
        if (PAGED && bad_page) atomicMax(a.ctl.status, SWA_STATUS_BAD_INPUT);
        if (!ok && lane == 0)
            // let our own copies land before the CTA's shared memory goes away
            for (int st = 0; st < BULK_NST; ++st) {
                if (iss[st] == 0) continue;
                const unsigned long long t0 = globaltimer();
                while (!mbar_try_wait(&full[st], (iss[st] - 1) & 1))
                    if (globaltimer() - t0 > a.ctl.limit_ns) break;
            }
    } else {
        // ----------------------------------------------------- compute --
        const int part = lane % LPR;        // which 8 elements of a row
        const int rgrp = lane / LPR;        // which row of a warp load
        const __nv_bfloat16 *qb = static_cast<const __nv_bfloat16 *>(a.q) + ((long long)b * a.Hq + (long long)hk * G) * D;
        uint4 q[G];
#pragma unroll
        for (int g = 0; g < G; ++g) q[g] = __ldg(reinterpret_cast<const uint4 *>(qb + g * D + part * 8));
        float2 acc[G][4];
        float m[G], l[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            m[g] = -CUDART_INF_F;
            l[g] = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[g][e] = make_float2(0.f, 0.f);
        }
        for (int it = 0; it < n_it; ++it) {
            const int st = it % BULK_NST;
            if (!warp_wait_bounded(&full[st], (it / BULK_NST) & 1, ctl)) break;
            const int rows = min(C::SS, s_end - (s_begin + it * C::SS));
            const int r0 = warp * BATCH;    // this warp's first row of the stage
            if (r0 < rows) {
                const uint8_t *kst = sK + st * C::STAGE + part * 16;
                const uint8_t *vst = sV + st * C::STAGE + part * 16;
                uint4 kr[NBL], vr[NBL];
#pragma unroll
                for (int n = 0; n < NBL; ++n) {
                    const int r = min(r0 + n * RPW + rgrp, rows - 1); // clamp: masked below
                    kr[n] = *reinterpret_cast<const uint4 *>(kst + r * C::ROWB);
                    vr[n] = *reinterpret_cast<const uint4 *>(vst + r * C::ROWB);
                }
                float v[LPR];
#pragma unroll
                for (int n = 0; n < NBL; ++n)
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        float t = 0.f;
                        t = dot2_bf16(q[g].x, kr[n].x, t);
                        t = dot2_bf16(q[g].y, kr[n].y, t);
                        t = dot2_bf16(q[g].z, kr[n].z, t);
                        t = dot2_bf16(q[g].w, kr[n].w, t);
                        v[n * G + g] = t;
                    }
#pragma unroll
                for (int k = LPR / 2; k >= 1; k >>= 1) {
                    const bool upper = (part & k) != 0;
#pragma unroll
                    for (int x = 0; x < k; ++x) {
                        const float send = upper ? v[x] : v[x + k];
                        const float keep = upper ? v[x + k] : v[x];
                        v[x] = keep + __shfl_xor_sync(0xffffffffu, send, k);
                    }
                }
                const int my_n = part / G, my_g = part % G;
                const float sc = (r0 + my_n * RPW + rgrp < rows) ? v[0] * a.scale_log2 : -CUDART_INF_F;
                float bm = sc;
#pragma unroll
                for (int k = G; k < 32; k <<= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, k));
                float m_old = m[0];
#pragma unroll
                for (int g = 1; g < G; ++g)
                    if (my_g == g) m_old = m[g];
                const float m_new = fmaxf(m_old, bm);
                const float m_use = m_new == -CUDART_INF_F ? 0.f : m_new;
                const float pr = ex2_approx(sc - m_use);
                const float al = ex2_approx(m_old - m_use);
                float ps = pr;
#pragma unroll
                for (int k = G; k < 32; k <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, k);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float alg = __shfl_sync(0xffffffffu, al, g);
                    const float psg = __shfl_sync(0xffffffffu, ps, g);
                    m[g] = __shfl_sync(0xffffffffu, m_new, g);
                    l[g] = l[g] * alg + psg;
                    const float2 a2 = make_float2(alg, alg);
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[g][e] = mul2(acc[g][e], a2);
                }
#pragma unroll
                for (int n = 0; n < NBL; ++n) {
                    const float2 v0 = bf16x2_to_float2(vr[n].x), v1 = bf16x2_to_float2(vr[n].y);
                    const float2 v2 = bf16x2_to_float2(vr[n].z), v3 = bf16x2_to_float2(vr[n].w);
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float pn = __shfl_sync(0xffffffffu, pr, rgrp * LPR + n * G + g);
                        const float2 p2 = make_float2(pn, pn);
                        acc[g][0] = fma2(p2, v0, acc[g][0]);
                        acc[g][1] = fma2(p2, v1, acc[g][1]);
                        acc[g][2] = fma2(p2, v2, acc[g][2]);
                        acc[g][3] = fma2(p2, v3, acc[g][3]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        // sum the row groups' accumulators (same softmax reference per head)
#pragma unroll
        for (int k = LPR; k < 32; k <<= 1)
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    acc[g][e].x += __shfl_xor_sync(0xffffffffu, acc[g][e].x, k);
                    acc[g][e].y += __shfl_xor_sync(0xffffffffu, acc[g][e].y, k);
                }
        if (lane == 0)
#pragma unroll
            for (int g = 0; g < G; ++g) {
                sm_m[warp][g] = m[g];
                sm_l[warp][g] = l[g];
            }
        if (rgrp == 0)
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    sm_acc[warp][g][part * 8 + 2 * e] = acc[g][e].x;
                    sm_acc[warp][g][part * 8 + 2 * e + 1] = acc[g][e].y;
                }
    }
    __syncthreads();
    decode_finish<__nv_bfloat16, D, G>(a, b, hk, split, sm_m, sm_l, sm_acc);
}

// LSE merge of the split partials: o = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s
template <typename T, int D>
__global__ void decode_combine_kernel(DecodeArgs a)
{
    // launched as a programmatic dependent of the split kernel: its launch
    // overlaps the split kernel's tail, and this wait returns once that
    // kernel has completed and its partials are visible
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int bh = blockIdx.x;
    const int e = threadIdx.x;
    const float *part = a.partial + (long long)bh * a.splits * (D + 2);
    float M = -CUDART_INF_F;
    for (int s = 0; s < a.splits; ++s) M = fmaxf(M, part[s * (D + 2) + D]);
    const float Mu = M == -CUDART_INF_F ? 0.f : M;
    float L = 0.f, O = 0.f;
    for (int s = 0; s < a.splits; ++s) {
        const float f = ex2_approx(part[s * (D + 2) + D] - Mu);
        L += part[s * (D + 2) + D + 1] * f;
        O += part[s * (D + 2) + e] * f;
    }
    T *o = static_cast<T *>(a.o) + (long long)bh * D;
    Ld<T>::store(o + e, L > 0.f ? O / L : 0.f);
    if (a.lse && e == 0) a.lse[bh] = L > 0.f ? (M + __log2f(L)) * 0.69314718055994530942f : -CUDART_INF_F;
}

// One decode launch: grid (splits, Hkv, B).
template <typename K>
cudaError_t launch_decode_grid(K kernel, const DecodeArgs &a, cudaStream_t s, int threads = 32 * DEC_WARPS,
                               int smem = 0)
{
    kernel<<<dim3(a.splits, a.Hkv, a.B), threads, smem, s>>>(a);
    return cudaGetLastError();
}

// The split merge, launched as a programmatic dependent of the split kernel
// before it on the stream (its griddepcontrol.wait orders it after that
// kernel's completion).
template <typename T, int D>
cudaError_t launch_combine(const DecodeArgs &a, cudaStream_t s)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.B * a.Hq);
    cfg.blockDim = dim3(D);
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_combine_kernel<T, D>, a);
}

template <typename T, int D, int G>
cudaError_t launch_decode_t(const DecodeArgs &a, cudaStream_t s)
{
    const int src = a.ptable ? SRC_PAGED : a.n_sink > 0 ? SRC_SINKS : SRC_RING;
    cudaError_t e;
    if constexpr (std::is_same<T, __nv_bfloat16>::value && BulkCfg<D, G>::OK) {
        if (src == SRC_RING || src == SRC_PAGED) {
            using C = BulkCfg<D, G>;
            static DeviceOnce once;
            e = once.get(
                [&](int) {
                    cudaError_t r = cudaFuncSetAttribute(decode_bulk_kernel<D, G, false>,
                                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
                    if (r != cudaSuccess) return r;
                    return cudaFuncSetAttribute(decode_bulk_kernel<D, G, true>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
                },
                nullptr);
            if (e == cudaSuccess)
                e = src == SRC_PAGED ? launch_decode_grid(decode_bulk_kernel<D, G, true>, a, s, BULK_THREADS, C::SMEM)
                                     : launch_decode_grid(decode_bulk_kernel<D, G, false>, a, s, BULK_THREADS, C::SMEM);
            if (e != cudaSuccess || a.splits == 1) return e;
            return launch_combine<T, D>(a, s);
        }
    }
    if constexpr (std::is_same<T, __nv_bfloat16>::value && G <= D / 8) {
        if (src == SRC_PAGED) e = launch_decode_grid(decode_bf16_kernel<D, G, SRC_PAGED>, a, s);
        else if (src == SRC_SINKS) e = launch_decode_grid(decode_bf16_kernel<D, G, SRC_SINKS>, a, s);
        else e = launch_decode_grid(decode_bf16_kernel<D, G, SRC_RING>, a, s);
    } else {
        if (src == SRC_PAGED) e = launch_decode_grid(decode_kernel<T, D, G, SRC_PAGED>, a, s);
        else if (src == SRC_SINKS) e = launch_decode_grid(decode_kernel<T, D, G, SRC_SINKS>, a, s);
        else e = launch_decode_grid(decode_kernel<T, D, G, SRC_RING>, a, s);
    }
    if (e != cudaSuccess || a.splits == 1) return e;
    return launch_combine<T, D>(a, s);
}

template <typename T, int D>
cudaError_t launch_decode_g(const DecodeArgs &a, cudaStream_t s)
{
    switch (a.Hq / a.Hkv) {
    case 1: return launch_decode_t<T, D, 1>(a, s);
    case 2: return launch_decode_t<T, D, 2>(a, s);
    case 4: return launch_decode_t<T, D, 4>(a, s);
    case 8: return launch_decode_t<T, D, 8>(a, s);
    default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t launch_decode_d(const DecodeArgs &a, cudaStream_t s)
{
    switch (a.d) {
    case 32: return launch_decode_g<T, 32>(a, s);
    case 64: return launch_decode_g<T, 64>(a, s);
    case 128: return launch_decode_g<T, 128>(a, s);
    default: return cudaErrorInvalidValue;
    }
}

// ------------------------------------------------------ bounded-wait hook --
__global__ void expire_wait_kernel(DeviceCtl c)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        WaitCtl ctl{&abort_flag, c.status, c.limit_ns};
        (void)wait_bounded(&bar, 0, ctl); // nothing arrives: expires
    }
}

}  // namespace

int decode_splits(int B, int Hq, int Hkv, int d, int W)
{
    (void)Hq;
    (void)d;
    // enough CTAs for several waves over 148 SMs; each split keeps at least
    // one full batch of slots per warp
    const long long units = (long long)B * Hkv;
    long long want = (148LL * 16 + units - 1) / units;
    int s = 1;
    while (s < want && s * 2 * 32 * DEC_WARPS <= W) s *= 2;
    return s;
}

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int d, int W)
{
    const int s = decode_splits(B, Hq, Hkv, d, W);
    if (s <= 1) return 0;
    return (size_t)B * Hq * s * (d + 2) * sizeof(float);
}

cudaError_t launch_decode(int dtype_bf16, const DecodeArgs &a, cudaStream_t s)
{
    return dtype_bf16 ? launch_decode_d<__nv_bfloat16>(a, s) : launch_decode_d<float>(a, s);
}

cudaError_t launch_prefill_f32(const F32PrefillArgs &a, cudaStream_t s)
{
    dim3 grid((a.T + F32_ROWS_PER_CTA - 1) / F32_ROWS_PER_CTA, a.Hq, a.B);
    prefill_f32_kernel<<<grid, 32 * F32_ROWS_PER_CTA, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_append(const AppendArgs &a, cudaStream_t s)
{
    const long long total = (long long)a.B * min(a.n, a.W) * a.Hkv * (a.row_bytes / 16);
    long long blocks = (total + 255) / 256;
    if (blocks < 1) blocks = 1;
    if (blocks > 148 * 32) blocks = 148 * 32;
    append_kernel<<<(int)blocks, 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_mask_export(uint8_t *mask, int T, int left, int right, const int32_t *gidx, int g,
                               cudaStream_t s)
{
    const long long n = (long long)T * T;
    long long blocks = (n + 255) / 256;
    if (blocks > 148 * 64) blocks = 148 * 64;
    if (blocks < 1) blocks = 1;
    mask_export_kernel<<<(int)blocks, 256, 0, s>>>(mask, T, left, right, gidx, g);
    return cudaGetLastError();
}

cudaError_t launch_debug_expire_wait(const DeviceCtl &ctl, cudaStream_t s)
{
    expire_wait_kernel<<<1, 32, 0, s>>>(ctl);
    return cudaGetLastError();
}

}  // namespace swa
