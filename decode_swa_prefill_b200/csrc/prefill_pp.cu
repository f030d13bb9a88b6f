// Sliding-window prefill on tcgen05 tensor cores with 128-key tiles and two
// query tiles in alternation (sm_100a).
//
// What it computes (the pages' definition): for query row i, softmax over the
// keys of its window of scale*q.k, logits outside the window being -inf, then
// the weighted sum of value rows ("Sliding Window Attention", robocikowo.com,
// opening definition).  The [T,T] score matrix never exists: a CTA streams
// only the 128-key tiles that intersect its query tiles' windows (the
// fused-kernel point of the same page and of the Ultralytics glossary's
// FlashAttention entry); work per query tile is O(W*d).
//
// CTA anatomy (320 threads, one CTA per SM), two 128-row query tiles X = A, B
// sharing one kv head, hence every K/V tile: the two query heads of a GQA pair
// at the same rows, or (odd group size) two consecutive row tiles of one head.
//   warps 0-3  softmax + epilogue of tile A: thread r owns row r = TMEM lane r
//   warps 4-7  the same for tile B
//   warp 8     producer: TMA tile loads of Q (once), K and V (128 keys per
//              tile, two stages each); no multicast
//   warp 9     TMEM allocator and the single MMA issuer (lane 0)
// TMEM (all 512 columns):
//   S[X]  columns 128X .. 128X+127: fp32 scores of one 128-key tile
//   P[X]  the first 64 columns of S[X]: bf16 probabilities (pairs)
//   O[X]  columns 256+128X: fp32 output accumulator (d <= 128)
// Per key tile t the issuer runs, in this order,
//   PV_A(t-1), QK_A(t), PV_B(t-1), QK_B(t)
// (PV_X: O[X] += P[X] V, A operand from TMEM; QK_X: S[X] = Q_X K^T), so the
// softmax of one tile runs while the tensor core computes the other tile's
// PV and next QK^T.  QK_X(t) overwrites the S[X] columns that PV_X(t-1) reads
// P from; both come from the one issuing thread, and the tensor core executes
// one thread's tcgen05.mma operations in issue order, so no wait separates
// them.  With 128-key tiles every QK^T has N = 128: both operands come from
// shared memory at the rate the tensor core consumes them (an N = 64 QK^T is
// limited by shared-memory bandwidth instead).
//
// Softmax (one row per thread, 128 scores per tile, one streaming pass over
// four 32-key chunks): running maximum in log2 units, raised only when a
// chunk's maximum exceeds it by more than 2^8 (P stays <= 256 in bf16), by a
// whole power of two, which rescales l, the P chunks already written and the
// O row in TMEM after the previous PV; -inf outside the window on edge tiles
// only; per warp, 32-key chunks no row of the warp can see are skipped (their
// P is written as 0).
// Every exponential runs on the MUFU (ex2.approx): moving a quarter of them
// to a cubic on the FMA pipe measured 2% slower here (the issue slots, not
// the MUFU, are what the softmax runs short of).
//
// Every mbarrier wait is bounded (wait_bounded): on expiry the CTA records
// SWA_STATUS_TIMEOUT, drains its own in-flight copies and MMAs with a second
// bound, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math_constants.h>

#include <type_traits>

#include "ptx.cuh"
#include "swa_internal.h"
#include "tma_map.h"

namespace swa {
namespace {

constexpr int PP_BM = 128;               // query rows per tile (= TMEM lanes)
constexpr int PP_BN = 128;               // keys per key tile
constexpr int PP_NSTAGE = 2;             // K and V pipeline depth
constexpr int PP_THREADS = 320;
constexpr float PP_RESCALE_LOG2 = 8.0f;  // raise the running max only beyond 2^8
// where the keys come from: the prefill's own k/v; or (a chunk of new tokens)
// its k/v and the W-slot ring before it; or its k/v plus one gathered tile
// of the first n_sink positions (attention sinks)
constexpr int PP_PLAIN = 0, PP_RING = 1, PP_SINKS = 2, PP_VARLEN = 3;

template <int D>
struct PCfg {
    static constexpr int RB = (D * 2 >= 128) ? 128 : D * 2; // bytes per swizzled row
    static constexpr int E = RB / 2;                         // elements per chunk row
    static constexpr int NCH = D / E;                        // chunks per head row
    static constexpr int QCH = PP_BM * RB;                   // one chunk of a 128-row Q tile
    static constexpr int KCH = PP_BN * RB;                   // one chunk of a 128-key tile
    static constexpr int QTILE = PP_BM * D * 2;
    static constexpr int KTILE = PP_BN * D * 2;
    static constexpr uint32_t LAYOUT = (RB == 128) ? UMMA_SW128 : UMMA_SW64;
    static constexpr int OFF_Q = 0;                          // Q_A, Q_B
    static constexpr int OFF_K = OFF_Q + 2 * QTILE;
    static constexpr int OFF_V = OFF_K + PP_NSTAGE * KTILE;
    static constexpr int OFF_BAR = OFF_V + PP_NSTAGE * KTILE;
    // + room to align the base to 1 KiB; more than half the SM's shared
    // memory so that a second CTA never shares the SM (each CTA takes all
    // 512 TMEM columns)
    static constexpr int SMEM_NEED = OFF_BAR + 256 + 1024;
    static constexpr int SMEM_BYTES = SMEM_NEED > 120 * 1024 ? SMEM_NEED : 120 * 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(D == 32 || D == 64 || D == 128, "head dim");
    static_assert(SMEM_BYTES + 1024 <= 228 * 1024, "fits one SM");
    static_assert(2 * (SMEM_BYTES + 1024) > 228 * 1024, "never two CTAs per SM");
};

__host__ __device__ constexpr uint32_t pp_col_s(int x) { return 128u * x; }
__host__ __device__ constexpr uint32_t pp_col_o(int x) { return 256u + 128u * x; }

// Byte offset of element e of row r inside a swizzled [rows][D] tile whose
// E-element chunks are `ch_bytes` apart (the layout of a TMA SWIZZLE_128B /
// SWIZZLE_64B load).
template <int D>
__device__ __forceinline__ uint32_t pp_tile_offset(int r, int e, int ch_bytes)
{
    using C = PCfg<D>;
    const int ch = e / C::E;
    const int u = (e % C::E) / 8;
    const int phys = (C::RB == 128) ? (u ^ (r & 7)) : (u ^ ((r >> 1) & 3));
    return ch * ch_bytes + r * C::RB + phys * 16;
}

// Producer-warp gather of a 128-key tile, one row at a time, into the
// swizzled layout of a TMA tile load: 16-byte cp.async copies, all in flight
// at once; row_src(r) gives key row r's source, or null for zeros.  All 32
// lanes; returns once the copies have landed.
template <int D, typename RowSrc>
__device__ __forceinline__ void pp_gather_rows(uint8_t *dst, const __nv_bfloat16 *any_valid, int lane, RowSrc row_src)
{
    using C = PCfg<D>;
    constexpr int GR = D / 8;   // 16-byte granules per row
    for (int idx = lane; idx < PP_BN * GR; idx += 32) {
        const int r = idx / GR, u = idx % GR;
        const __nv_bfloat16 *src = row_src(r);
        cp_async16(dst + pp_tile_offset<D>(r, u * 8, C::KCH), src ? src + u * 8 : any_valid, src ? 16u : 0u);
    }
    cp_async_wait_all();
}

struct PPBars {
    uint64_t q_full[2];    // [tile] (the one-unit kernel loads both on q_full[0])
    uint64_t q_empty[2];   // [tile] (persistent kernel): the unit's output store has read Q_X's buffer
    uint64_t k_full[PP_NSTAGE];
    uint64_t k_empty[PP_NSTAGE];
    uint64_t v_full[PP_NSTAGE];
    uint64_t v_empty[PP_NSTAGE];
    uint64_t s_full[2];    // [tile]
    uint64_t p_full[2];    // [tile], one arrival per softmax warp
    uint64_t pv_done[2];   // [tile]
    uint64_t epi[2];       // [tile]: the output tile is staged (one arrival per warp)
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

// Bulk stores of this thread have finished reading their shared memory.
__device__ __forceinline__ void pp_store_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

__device__ __forceinline__ void pp_drain_wait(uint64_t *bar, uint32_t parity, unsigned long long limit)
{
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > limit) return;
    }
}

// One 128-row query tile of a CTA: key tiles [ts, te) relative to j_lo.
struct PPTile {
    int h, m0, nrows, ts, te;
    bool active;
};

struct PPWork {
    int b, hk;
    PPTile q[2];
    int j_lo;      // first key tile (absolute, 128-key units)
    int n_band;    // window key tiles; a sink tile follows them
    int n_tiles;   // key tiles the CTA streams
    long long p0;  // position of query row 0 (a chunk continuing a ring; else 0)
    long long kend; // one past the last key position (p0 + T; a packed sequence: its length)
};

// Does query tile q use key tile t (window tiles [ts, te), then the sink
// tile, which every query tile takes)?
template <int SRC>
__device__ __forceinline__ bool pp_active(const PPTile &q, int n_band, int t)
{
    if constexpr (SRC == PP_SINKS)
        if (t >= n_band) return q.active;
    return q.active && t >= q.ts && t < q.te;
}

// Units: pairs of query heads of one kv head (even group size) or pairs of
// consecutive row tiles of one head; query tiles in descending order, so the
// short CTAs at the start of a causal sequence run last and fill the tail.
// RING: the rows are a chunk of new tokens at positions pos[b] .. (a
// negative entry is read as 0; the producer records it), and key tiles are
// counted in absolute positions.  VARLEN: b is a packed sequence, tiles are
// counted from its first row, and those past its end are inactive (an
// inconsistent entry makes the sequence empty; the CTA records it).
template <int SRC>
__device__ __forceinline__ PPWork pp_make_work(const TcPrefillArgs &a, const RingArgs &ring, const VarlenArgs &vl,
                                               int unit)
{
    constexpr bool RING = SRC == PP_RING;
    constexpr bool VARLEN = SRC == PP_VARLEN;
    PPWork w;
    const int G = a.Hq / a.Hkv;
    const int nqt = ((VARLEN ? vl.max_len : a.T) + PP_BM - 1) / PP_BM;
    const int bid = unit;
    for (int x = 0; x < 2; ++x) w.q[x] = PPTile{0, 0, 0, 0, 0, false};
    if (G % 2 == 0) {
        const int hp = bid % (a.Hq / 2);
        const int qt = nqt - 1 - (bid / (a.Hq / 2)) % nqt;
        w.b = bid / ((a.Hq / 2) * nqt);
        for (int x = 0; x < 2; ++x) w.q[x] = PPTile{2 * hp + x, qt * PP_BM, min(PP_BM, a.T - qt * PP_BM), 0, 0, true};
    } else {
        const int h = bid % a.Hq;
        const int nqp = (nqt + 1) / 2;
        const int qp = nqp - 1 - (bid / a.Hq) % nqp;
        w.b = bid / (a.Hq * nqp);
        for (int x = 0; x < 2; ++x) {
            const int qt = 2 * qp + x;
            if (qt < nqt) w.q[x] = PPTile{h, qt * PP_BM, min(PP_BM, a.T - qt * PP_BM), 0, 0, true};
        }
    }
    int left = a.left;
    int TT = a.T;   // rows of this sequence
    if constexpr (VARLEN) {
        TT = varlen_ok(vl, w.b, a.T) ? vl.cu[w.b + 1] - vl.cu[w.b] : 0;
        left = varlen_left(vl, w.b, a.left);
        for (int x = 0; x < 2; ++x) {
            if (w.q[x].m0 >= TT) w.q[x].active = false;
            w.q[x].nrows = min(PP_BM, TT - w.q[x].m0);
        }
    }
    // positions: 64-bit only for a chunk continuing a ring
    typedef typename std::conditional<RING, long long, int>::type kpos_t;
    w.p0 = 0;
    if constexpr (RING) w.p0 = max((long long)ring.pos[w.b], 0LL);
    w.kend = w.p0 + TT;
    const kpos_t p0 = (kpos_t)w.p0, kend = (kpos_t)w.kend;
    kpos_t lo = kend, hi = -1;
    kpos_t lo_x[2] = {0, 0}, hi_x[2] = {0, 0};
    for (int x = 0; x < 2; ++x) {
        if (!w.q[x].active) continue;
        lo_x[x] = max((kpos_t)0, (kpos_t)(p0 + w.q[x].m0 - left));
        hi_x[x] = min(kend - 1, (kpos_t)(p0 + w.q[x].m0 + PP_BM - 1 + a.right));
        lo = min(lo, lo_x[x]);
        hi = max(hi, hi_x[x]);
    }
    w.j_lo = (int)(lo / PP_BN);
    w.n_band = (int)(hi / PP_BN) - w.j_lo + 1;
    w.n_tiles = w.n_band + ((SRC == PP_SINKS && a.g > 0) ? 1 : 0);
    for (int x = 0; x < 2; ++x)
        if (w.q[x].active) {
            w.q[x].ts = (int)(lo_x[x] / PP_BN) - w.j_lo;
            w.q[x].te = (int)(hi_x[x] / PP_BN) - w.j_lo + 1;
        }
    w.hk = w.q[0].h / G;
    return w;
}

// Softmax of one 128-key tile for one row, one streaming pass over its four
// 32-key chunks: chunk cc+1's TMEM load is in flight while chunk cc's scores
// become exponentials and P (bf16 pairs in columns 16cc .. 16cc+15 of S,
// inside S chunks already read), so at most 64 scores are held in registers
// and one TMEM round trip per tile is exposed.  There is no separate maximum
// pass: the running maximum m (log2 units) is raised when a chunk's own
// maximum exceeds it by more than 2^8 -- after a row's first chunk that only
// happens when its scores jump by that much -- by a whole number k of log2
// units, and then l, this tile's sum so far and this tile's P chunks already
// written are scaled by 2^-k, exactly (the caller scales the O row after the
// previous PV).  P stays <= 256.
// FULL: every key of the tile is visible to every row of the warp (no
// masking, all chunks live), the common case, compiled without masking.
template <bool FULL>
__device__ __forceinline__ void pp_softmax_tile(uint32_t s_addr, int c_lo, int c_hi, int col_lo, int col_hi,
                                                float scale_log2, float &m, float &l, bool &rescale, float &alpha,
                                                bool first)
{
    auto live = [&](int cc) { return FULL || (cc >= c_lo && cc <= c_hi); };
    const float2 sc2 = make_float2(scale_log2, scale_log2);
    float2 acc2 = make_float2(0.f, 0.f), acc2b = make_float2(0.f, 0.f);
    float atot = 1.f;    // product of this tile's raises
    // chunk maximum (log2 units, before the scale), -inf for a dead chunk;
    // masked keys become -inf in place
    auto cmax = [&](float *v, int cc) -> float {
        if (!live(cc)) return -CUDART_INF_F;
        if (!FULL) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int xx = cc * 32 + e;
                if (xx < col_lo || xx > col_hi) v[e] = -CUDART_INF_F;
            }
        }
        float mx4[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) mx4[j] = fmax3(v[j], v[4 + j], v[8 + j]);
#pragma unroll
        for (int e = 12; e + 8 <= 32; e += 8)
#pragma unroll
            for (int j = 0; j < 4; ++j) mx4[j] = fmax3(mx4[j], v[e + j], v[e + 4 + j]);
#pragma unroll
        for (int j = 0; j < 4; ++j) mx4[j] = fmaxf(mx4[j], v[28 + j]);
        return fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
    };
    // raise the running maximum for the pair of chunks from c0 on (maximum mc)
    auto raise_to = [&](float mc, int c0) {
        const bool raise = mc > m + PP_RESCALE_LOG2;
        if (!__any_sync(0xffffffffu, raise)) return;
        float a = 1.f;
        if (raise) {
            if (m == -CUDART_INF_F) {
                a = 0.f;
                m = mc;
            } else {
                const int k = (int)ceilf(mc - m);
                a = k < 126 ? __int_as_float((127 - k) << 23) : 0.f;
                m += (float)k;
            }
            l *= a;
            acc2 = mul2(acc2, make_float2(a, a));
            acc2b = mul2(acc2b, make_float2(a, a));
            atot *= a;
        }
        if (c0 > 0) {
            tmem_st_wait();
#pragma unroll 1
            for (int pc = 0; pc < c0; ++pc) {
                float pv[16];
                tmem_ld16(s_addr + pc * 16, pv);
                tmem_ld_wait_dep16(pv);
                uint32_t pu[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const uint32_t w = __float_as_uint(pv[e]);
                    pu[e] = pack_bf16x2(__uint_as_float(w << 16) * a, __uint_as_float(w & 0xffff0000u) * a);
                }
                tmem_st16u(s_addr + pc * 16, pu);
            }
        }
    };
    auto exps = [&](float *v, int cc) {
        uint32_t pk[16];
        if (live(cc)) {
            const float ref = (m == -CUDART_INF_F) ? 0.f : m;
            const float2 nr2 = make_float2(-ref, -ref);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
                float2 y = fma2(make_float2(v[e], v[e + 1]), sc2, nr2);
                y.x = ex2_approx(y.x);
                y.y = ex2_approx(y.y);
                if (e & 2) acc2b = add2(acc2b, y);
                else acc2 = add2(acc2, y);
                pk[e / 2] = pack_bf16x2(y.x, y.y);
            }
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) pk[j] = 0u;
        }
        tmem_st16u(s_addr + cc * 16, pk);
    };
    float va[32], vb[32];
    if (live(0)) tmem_ld32(s_addr, va);
    if (live(1)) tmem_ld32(s_addr + 32, vb);
    tmem_ld_wait_dep(va);
    reg_fence32(vb);
    raise_to(fmaxf(cmax(va, 0), cmax(vb, 1)) * scale_log2, 0);
    exps(va, 0);
    if (live(2)) tmem_ld32(s_addr + 64, va);
    exps(vb, 1);
    if (live(3)) tmem_ld32(s_addr + 96, vb);
    tmem_ld_wait_dep(va);
    reg_fence32(vb);
    raise_to(fmaxf(cmax(va, 2), cmax(vb, 3)) * scale_log2, 2);
    exps(va, 2);
    exps(vb, 3);
    const float2 tot = add2(acc2, acc2b);
    l += tot.x + tot.y;
    alpha = atot;
    rescale = !first && atot != 1.f;
}

// RING: a chunk of new tokens whose earlier keys are in the W-slot ring
// (position p in slot p mod W): key tiles wholly in the chunk or wholly in
// the ring (without wrapping round its end) come by TMA, the others by row
// gathers.
template <int D, int SRC>
__global__ void __launch_bounds__(PP_THREADS, 1)
    swa_prefill_pp_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                          const __grid_constant__ CUtensorMap tmKr, const __grid_constant__ CUtensorMap tmVr,
                          const TcPrefillArgs a, const RingArgs ring, const VarlenArgs vl)
{
    using C = PCfg<D>;
    constexpr bool RING = SRC == PP_RING;
    constexpr bool VARLEN = SRC == PP_VARLEN;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + C::OFF_Q;   // Q_X at sQ + X * QTILE
    uint8_t *sK = smem + C::OFF_K;
    uint8_t *sV = smem + C::OFF_V;
    PPBars *bars = reinterpret_cast<PPBars *>(smem + C::OFF_BAR);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const PPWork w = pp_make_work<SRC>(a, ring, vl, blockIdx.x);
    if constexpr (VARLEN) {
        if (threadIdx.x == 0 && !varlen_ok(vl, w.b, a.T)) atomicMax(a.ctl.status, SWA_STATUS_BAD_INPUT);
        // a unit past its sequence's end has nothing to do
        if (!w.q[0].active) return;
    }
    const int tb = VARLEN ? 0 : w.b;            // batch coordinate of the tensors
    const int row0 = VARLEN ? vl.cu[w.b] : 0;   // tensor row of position 0
    WaitCtl ctl{&bars->abort, a.ctl.status, a.ctl.limit_ns};

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full[0], 1);
        for (int s = 0; s < PP_NSTAGE; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&bars->s_full[x], 1);
            mbar_init(&bars->p_full[x], PP_BM / 32);
            mbar_init(&bars->pv_done[x], 1);
            mbar_init(&bars->epi[x], PP_BM / 32);
        }
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        fence_mbar_init();
    }
    if (warp == 8 && lane == 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        prefetch_tensormap(&tmO);
    }
    if (warp == 9) tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 8) {
        // ------------------------------------------------------ producer --
        int nk = 0, nv = 0;   // K and V tiles issued (tile t goes to stage t % PP_NSTAGE)
        bool ok = true;
        if (lane == 0) {
            int nq = 0;
            for (int x = 0; x < 2; ++x) nq += w.q[x].active ? 1 : 0;
            mbar_expect_tx(&bars->q_full[0], nq * C::QTILE);
            for (int x = 0; x < 2; ++x)
                if (w.q[x].active)
                    for (int ch = 0; ch < C::NCH; ++ch) {
                        SWA_DCHECK(w.q[x].m0 >= 0 && row0 + w.q[x].m0 < a.T && w.q[x].h < a.Hq, a.ctl.status);
                        tma_load_4d(sQ + x * C::QTILE + ch * C::QCH, &tmQ, &bars->q_full[0], ch * C::E, w.q[x].h,
                                    row0 + w.q[x].m0, tb);
                    }
        }
        if (RING && lane == 0 && ring.pos[w.b] < 0) atomicMax(a.ctl.status, SWA_STATUS_BAD_INPUT);
        // one K or V tile into stage st
        auto load_tile = [&](bool is_v, int st, long long key0) {
            uint8_t *dst = (is_v ? sV : sK) + st * C::KTILE;
            uint64_t *bar = is_v ? &bars->v_full[st] : &bars->k_full[st];
            if constexpr (RING) {
                const bool ring_tile = key0 < w.p0;
                const long long slot0 = ring_tile ? key0 % ring.W : 0;
                if (!ring_tile || (key0 + PP_BN <= w.p0 && slot0 + PP_BN <= ring.W)) {
                    SWA_DCHECK(ring_tile || key0 - w.p0 < a.T, a.ctl.status);
                    if (lane == 0) {
                        mbar_expect_tx(bar, C::KTILE);
                        for (int ch = 0; ch < C::NCH; ++ch) {
                            if (ring_tile)
                                tma_load_4d(dst + ch * C::KCH, is_v ? &tmVr : &tmKr, bar, ch * C::E, (int)slot0, w.hk,
                                            w.b);
                            else
                                tma_load_4d(dst + ch * C::KCH, is_v ? &tmV : &tmK, bar, ch * C::E, w.hk,
                                            (int)(key0 - w.p0), w.b);
                        }
                    }
                    return;
                }
                // a tile that meets the chunk's first row or wraps round the
                // ring's end: rows from wherever each position lives
                const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(is_v ? a.v : a.k);
                const __nv_bfloat16 *rc = static_cast<const __nv_bfloat16 *>(is_v ? ring.vc : ring.kc);
                pp_gather_rows<D>(dst, src, lane, [&](int r) -> const __nv_bfloat16 * {
                    const long long p = key0 + r;
                    if (p >= w.p0) {
                        const long long row = p - w.p0;
                        return row < a.T ? src + (((long long)w.b * a.T + row) * a.Hkv + w.hk) * D : nullptr;
                    }
                    return rc + (((long long)w.b * a.Hkv + w.hk) * ring.W + p % ring.W) * D;
                });
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar);
            } else {
                SWA_DCHECK(key0 >= 0 && row0 + key0 < a.T, a.ctl.status);
                if (lane == 0) {
                    mbar_expect_tx(bar, C::KTILE);
                    for (int ch = 0; ch < C::NCH; ++ch)
                        tma_load_4d(dst + ch * C::KCH, is_v ? &tmV : &tmK, bar, ch * C::E, w.hk,
                                    row0 + (int)key0, tb);
                }
            }
        };
        // the sink tile: positions 0 .. n_sink-1, zeros after
        auto load_sinks = [&](bool is_v, int st) {
            uint8_t *dst = (is_v ? sV : sK) + st * C::KTILE;
            const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(is_v ? a.v : a.k);
            pp_gather_rows<D>(dst, src, lane, [&](int r) -> const __nv_bfloat16 * {
                return r < a.g ? src + (((long long)w.b * a.T + r) * a.Hkv + w.hk) * D : nullptr;
            });
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(is_v ? &bars->v_full[st] : &bars->k_full[st]);
        };
        for (int t = 0; t < w.n_tiles && ok; ++t) {
            const long long key0 = (long long)(w.j_lo + t) * PP_BN;
            const int st = t % PP_NSTAGE;
            const uint32_t par = ((t / PP_NSTAGE) & 1) ^ 1;
            const bool sink_tile = SRC == PP_SINKS && t >= w.n_band;
            ok = warp_wait_bounded(&bars->k_empty[st], par, ctl);
            if (!ok) break;
            if (sink_tile) load_sinks(false, st);
            else load_tile(false, st, key0);
            nk++;
            ok = warp_wait_bounded(&bars->v_empty[st], par, ctl);
            if (!ok) break;
            if (sink_tile) load_sinks(true, st);
            else load_tile(true, st, key0);
            nv++;
        }
        if (!ok && lane == 0) {
            // let our own copies land before the CTA's shared memory goes away
            for (int s = 0; s < PP_NSTAGE; ++s) {
                // copies issued into stage s: tiles s, s + PP_NSTAGE, ...
                const int ks = nk > s ? (nk - s + PP_NSTAGE - 1) / PP_NSTAGE : 0;
                const int vs = nv > s ? (nv - s + PP_NSTAGE - 1) / PP_NSTAGE : 0;
                if (ks > 0) pp_drain_wait(&bars->k_full[s], (ks - 1) & 1, a.ctl.limit_ns);
                if (vs > 0) pp_drain_wait(&bars->v_full[s], (vs - 1) & 1, a.ctl.limit_ns);
            }
        }
    } else if (warp == 9) {
        // ----------------------------------------------------------- MMA --
        // The whole warp runs the schedule (waits, descriptor arithmetic) in
        // lock step; lane 0 alone issues MMAs and commits.
        constexpr uint32_t idesc_qk = umma_idesc_bf16(PP_BM, PP_BN, 0, 0);
        constexpr uint32_t idesc_pv = umma_idesc_bf16(PP_BM, D, 0, 1);
        // descriptors are built once; a k-step or stage only adds a constant
        // to the 14-bit start-address field (addresses < 2^18)
        const uint64_t dq0 = umma_smem_desc(smem_u32(sQ), 16, 8 * C::RB, C::LAYOUT);
        const uint64_t dk0 = umma_smem_desc(smem_u32(sK), 16, 8 * C::RB, C::LAYOUT);
        const uint64_t dv0 = umma_smem_desc(smem_u32(sV), C::KCH, 8 * C::RB, C::LAYOUT);
        const bool leader = lane == 0;
        int cnt[2] = {0, 0};   // key tiles each query tile has multiplied by V so far
        bool ok = warp_wait_bounded(&bars->q_full[0], 0, ctl);
        auto qk = [&](int x, int t) {
            const int st = t % PP_NSTAGE;
            const uint64_t dq = dq0 + (uint64_t)((x * C::QTILE) >> 4);
            const uint64_t dk = dk0 + (uint64_t)((st * C::KTILE) >> 4);
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int byte = kk * 32;
                    const uint64_t qo = (uint64_t)(((byte / C::RB) * C::QCH + (byte % C::RB)) >> 4);
                    const uint64_t ko = (uint64_t)(((byte / C::RB) * C::KCH + (byte % C::RB)) >> 4);
                    mma_bf16_ss(tmem + pp_col_s(x), dq + qo, dk + ko, idesc_qk, kk > 0 ? 1u : 0u);
                }
                mma_commit(&bars->s_full[x]);
            }
        };
        auto pv = [&](int x, int t) -> bool {
            if (!warp_wait_bounded(&bars->p_full[x], cnt[x] & 1, ctl)) return false;
            tc_fence_after();
            const int st = t % PP_NSTAGE;
            const uint64_t dv = dv0 + (uint64_t)((st * C::KTILE) >> 4);
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < PP_BN / 16; ++kk)
                    mma_bf16_ts(tmem + pp_col_o(x), tmem + pp_col_s(x) + kk * 8,
                                dv + (uint64_t)((kk * 16 * C::RB) >> 4), idesc_pv, (cnt[x] > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&bars->pv_done[x]);
            }
            cnt[x]++;
            return true;
        };
        // prologue: QK^T of the first key tile for both query tiles
        if (ok && w.n_tiles > 0) {
            ok = warp_wait_bounded(&bars->k_full[0], 0, ctl);
            if (ok) {
                tc_fence_after();
                for (int x = 0; x < 2; ++x)
                    if (pp_active<SRC>(w.q[x], w.n_band, 0)) qk(x, 0);
                if (leader) mma_commit(&bars->k_empty[0]);
            }
        }
        for (int t = 0; t < w.n_tiles && ok; ++t) {
            const int st = t % PP_NSTAGE;
            const bool more = t + 1 < w.n_tiles;
            ok = warp_wait_bounded(&bars->v_full[st], (t / PP_NSTAGE) & 1, ctl);
            // the next K tile is waited for while tile A's softmax still runs
            if (ok && more) ok = warp_wait_bounded(&bars->k_full[(t + 1) % PP_NSTAGE], ((t + 1) / PP_NSTAGE) & 1, ctl);
            if (!ok) break;
            // tile A: PV of key tile t, then QK^T of key tile t+1 into the
            // same S columns (issue order keeps them apart)
            if (pp_active<SRC>(w.q[0], w.n_band, t)) ok = pv(0, t);
            if (!ok) break;
            if (more) {
                tc_fence_after();
                if (pp_active<SRC>(w.q[0], w.n_band, t + 1)) qk(0, t + 1);
            }
            // tile B likewise, half a step behind
            if (pp_active<SRC>(w.q[1], w.n_band, t)) ok = pv(1, t);
            if (!ok) break;
            if (leader) mma_commit(&bars->v_empty[st]);
            if (more) {
                if (pp_active<SRC>(w.q[1], w.n_band, t + 1)) qk(1, t + 1);
                if (leader) mma_commit(&bars->k_empty[(t + 1) % PP_NSTAGE]);
            }
            __syncwarp();
        }
        // all MMAs lane 0 issued are complete before TMEM is freed
        if (leader) {
            mma_commit(&bars->drain);
            pp_drain_wait(&bars->drain, 0, a.ctl.limit_ns);
        }
        __syncwarp();
    } else {
        // ------------------------------------------- softmax + epilogue --
        const int x = warp / 4;                 // query tile of this warpgroup
        const int quarter = warp % 4;
        const int r = quarter * 32 + lane;      // row in tile = TMEM lane
        // a select, not w.q[x]: a run-time index would keep the work record
        // in local memory (96 more bytes of stack per thread, in an L1 that
        // the 198 KB of shared memory leave small)
        const PPTile qt = x ? w.q[1] : w.q[0];
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t s_addr = tmem + lane_off + pp_col_s(x);
        const uint32_t o_addr = tmem + lane_off + pp_col_o(x);
        // key positions: 64-bit only for a chunk continuing a ring
        typedef typename std::conditional<RING, long long, int>::type kpos_t;
        const kpos_t p0 = RING ? (kpos_t)w.p0 : 0;
        const kpos_t kend = (RING || VARLEN) ? (kpos_t)w.kend : (kpos_t)a.T;   // one past the last key
        const int left = VARLEN ? varlen_left(vl, w.b, a.left) : a.left;   // keys before the query
        const int i_row = qt.m0 + r;            // row in q / o / lse
        const kpos_t ip = p0 + i_row;           // query position
        const bool row_real = qt.active && r < qt.nrows;
        const bool warp_has_rows = qt.active && quarter * 32 < qt.nrows;
        const kpos_t wi0 = p0 + qt.m0 + quarter * 32, wi1 = wi0 + 31;
        float m = -CUDART_INF_F, l = 0.f;
        bool ok = true;
        int c = 0;
        for (int t = 0; t < w.n_tiles && qt.active; ++t) {
            if (!pp_active<SRC>(qt, w.n_band, t)) continue;
            ok = warp_wait_bounded(&bars->s_full[x], c & 1, ctl);
            if (!ok) break;
            tc_fence_after();
            // which 32-key chunks can any row of this warp see
            const kpos_t key0 = (kpos_t)(w.j_lo + t) * PP_BN;
            int c_lo = 0, c_hi = -1;
            bool interior = false;
            if (warp_has_rows) {
                const kpos_t lo = max(max(key0, (kpos_t)(wi0 - left)), (kpos_t)0);
                const kpos_t hi = min(min(key0 + PP_BN - 1, (kpos_t)(wi1 + a.right)), kend - 1);
                if (lo <= hi) {
                    c_lo = (int)((lo - key0) / 32);
                    c_hi = (int)((hi - key0) / 32);
                }
                interior = (key0 + PP_BN - 1 < kend) && band_contains(wi1, key0, left, a.right) &&
                           band_contains(wi0, key0 + PP_BN - 1, left, a.right);
            }
            SWA_DCHECK(c_lo >= 0 && c_hi < PP_BN / 32, a.ctl.status);
            // visible columns of this row
            int col_lo = (int)max(ip - left - key0, (kpos_t)0);
            int col_hi = (int)min(min((kpos_t)(ip + a.right), kend - 1) - key0, (kpos_t)(PP_BN - 1));
            if (SRC == PP_SINKS && t >= w.n_band) {
                // sink positions 0 .. n_sink-1 below the row's window (the
                // ones inside it were counted there; causal: all <= the row)
                col_lo = 0;
                col_hi = min(a.g, (int)(ip - a.left)) - 1;
                const int last = warp_has_rows ? min(a.g, (int)(wi1 - a.left)) - 1 : -1;
                c_lo = 0;
                c_hi = last >= 0 ? last / 32 : -1;
                interior = false;
            }
            bool rescale_o;
            float alpha;
            if (interior && c_lo == 0 && c_hi == PP_BN / 32 - 1)
                pp_softmax_tile<true>(s_addr, c_lo, c_hi, col_lo, col_hi, a.scale_log2, m, l, rescale_o, alpha,
                                      c == 0);
            else
                pp_softmax_tile<false>(s_addr, c_lo, c_hi, col_lo, col_hi, a.scale_log2, m, l, rescale_o, alpha,
                                       c == 0);
            // O rescale (rare): wait for the previous tile's PV, which
            // accumulates into O; this tile's PV waits for P
            if (__any_sync(0xffffffffu, rescale_o)) {
                ok = warp_wait_bounded(&bars->pv_done[x], (c - 1) & 1, ctl);
                if (!ok) break;
                tc_fence_after();
                const float f = rescale_o ? alpha : 1.f;
#pragma unroll 1
                for (int cc = 0; cc < D / 16; ++cc) {
                    float ov[16];
                    tmem_ld16(o_addr + cc * 16, ov);
                    tmem_ld_wait_dep16(ov);
                    uint32_t ou[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) ou[e] = __float_as_uint(ov[e] * f);
                    tmem_st16u(o_addr + cc * 16, ou);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->p_full[x]);
            c++;
        }

        // ---- epilogue: O / l -> bf16 -> shared memory -> TMA store ----
        if (ok && c > 0) ok = warp_wait_bounded(&bars->pv_done[x], (c - 1) & 1, ctl);
        uint8_t *stage = sQ + x * C::QTILE;    // Q_X is no longer read: its last QK^T is complete
        // the last tile of a packed sequence is written row by row (a tile
        // store would run into the next sequence)
        const bool direct = VARLEN && qt.nrows < PP_BM;
        if (ok && qt.active) {
            tc_fence_after();
            const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll 1
            for (int cc = 0; cc < D / 16; ++cc) {
                float ov[16];
                tmem_ld16(o_addr + cc * 16, ov);
                tmem_ld_wait_dep16(ov);
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    uint4 pk;
                    pk.x = pack_bf16x2(ov[u * 8 + 0] * inv, ov[u * 8 + 1] * inv);
                    pk.y = pack_bf16x2(ov[u * 8 + 2] * inv, ov[u * 8 + 3] * inv);
                    pk.z = pack_bf16x2(ov[u * 8 + 4] * inv, ov[u * 8 + 5] * inv);
                    pk.w = pack_bf16x2(ov[u * 8 + 6] * inv, ov[u * 8 + 7] * inv);
                    if (direct) {
                        if (row_real) {
                            SWA_DCHECK(row0 + i_row < a.T, a.ctl.status);
                            __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(a.o) +
                                                 ((long long)(row0 + i_row) * a.Hq + qt.h) * D + cc * 16 + u * 8;
                            *reinterpret_cast<uint4 *>(dst) = pk;
                        }
                    } else {
                        *reinterpret_cast<uint4 *>(stage + pp_tile_offset<D>(r, cc * 16 + u * 8, C::QCH)) = pk;
                    }
                }
            }
            if (a.lse && row_real)
                a.lse[((long long)tb * a.Hq + qt.h) * a.T + row0 + i_row] =
                    (l > 0.f) ? (m + __log2f(l)) * 0.69314718055994530942f : -CUDART_INF_F;
        }
        // staging tile complete -> one thread per warpgroup stores it
        // (rows past T are clipped by the tensor map; an abort anywhere in
        // the CTA skips the store)
        if (!direct && qt.active) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->epi[x]);
            if (r == 0 && wait_bounded(&bars->epi[x], 0, ctl) && !bars->abort) {
                for (int ch = 0; ch < C::NCH; ++ch)
                    tma_store_4d(&tmO, stage + ch * C::QCH, ch * C::E, qt.h, row0 + qt.m0, tb);
                tma_store_commit();
                tma_store_wait_all();
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Persistent form, for windows of at most PP_PERSIST_MAX_WINDOW keys (short
// units): one CTA per SM takes units blockIdx.x, blockIdx.x + gridDim.x, ...
// with the same roles, tiles and softmax.  Barriers and TMEM are set up once;
// the K/V stage rings and every barrier phase run on across units.  Each
// query tile's epilogue stages O in Q_X's buffer, as above, and hands the
// buffer back to the producer once its store has read it (q_empty); the
// producer then loads the next unit's Q_X, while the next unit's first K and
// V tiles are already in flight.  No shared memory is added, so the L1 that
// holds the spills keeps its size.

// What the MMA issuer needs of a unit, as scalars (kept in registers; the
// query tile index is always a compile-time constant there).
struct PPSched {
    int n_tiles, n_band;
    int ts0, te0, ts1, te1;
    bool act0, act1;
};

template <int SRC>
__device__ __forceinline__ PPSched pp_sched(const PPWork &w)
{
    PPSched s;
    s.n_tiles = w.n_tiles;
    s.n_band = w.n_band;
    s.ts0 = w.q[0].ts; s.te0 = w.q[0].te; s.act0 = w.q[0].active;
    s.ts1 = w.q[1].ts; s.te1 = w.q[1].te; s.act1 = w.q[1].active;
    return s;
}

// Does query tile X use key tile t (as pp_active)?
template <int SRC, int X>
__device__ __forceinline__ bool pp_sched_on(const PPSched &s, int t)
{
    const bool act = X ? s.act1 : s.act0;
    if constexpr (SRC == PP_SINKS)
        if (t >= s.n_band) return act;
    return act && t >= (X ? s.ts1 : s.ts0) && t < (X ? s.te1 : s.te0);
}

// The next unit this CTA takes after `unit` (units unit, unit + gridDim.x,
// ...), skipping packed-sequence units that lie past their sequence's end;
// false when there is none.
template <int SRC>
__device__ __forceinline__ bool pp_next_unit(const TcPrefillArgs &a, const RingArgs &ring, const VarlenArgs &vl,
                                             int n_units, int &unit, PPWork &w)
{
    for (unit += gridDim.x; unit < n_units; unit += gridDim.x) {
        w = pp_make_work<SRC>(a, ring, vl, unit);
        if constexpr (SRC == PP_VARLEN) {
            // thread 0 visits every unit of the CTA: it records an
            // inconsistent entry (whose sequence is then empty)
            if (threadIdx.x == 0 && !varlen_ok(vl, w.b, a.T)) atomicMax(a.ctl.status, SWA_STATUS_BAD_INPUT);
            if (!w.q[0].active) continue;
        }
        return true;
    }
    return false;
}

template <int D, int SRC>
__global__ void __launch_bounds__(PP_THREADS, 1)
    swa_prefill_pp_persistent_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                          const __grid_constant__ CUtensorMap tmKr,
                          const __grid_constant__ CUtensorMap tmVr, const TcPrefillArgs a, const RingArgs ring,
                          const VarlenArgs vl, const int n_units)
{
    using C = PCfg<D>;
    constexpr bool RING = SRC == PP_RING;
    constexpr bool VARLEN = SRC == PP_VARLEN;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + C::OFF_Q;   // Q_X at sQ + X * QTILE
    uint8_t *sK = smem + C::OFF_K;
    uint8_t *sV = smem + C::OFF_V;
    PPBars *bars = reinterpret_cast<PPBars *>(smem + C::OFF_BAR);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    WaitCtl ctl{&bars->abort, a.ctl.status, a.ctl.limit_ns};

    if (threadIdx.x == 0) {
        for (int x = 0; x < 2; ++x) {
            mbar_init(&bars->q_full[x], 1);
            mbar_init(&bars->q_empty[x], 1);
        }
        for (int s = 0; s < PP_NSTAGE; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&bars->s_full[x], 1);
            mbar_init(&bars->p_full[x], PP_BM / 32);
            mbar_init(&bars->pv_done[x], 1);
            mbar_init(&bars->epi[x], PP_BM / 32);
        }
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        fence_mbar_init();
    }
    if (warp == 8 && lane == 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        prefetch_tensormap(&tmO);
    }
    if (warp == 9) tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 8) {
        // ------------------------------------------------------ producer --
        // Per unit: its first K tile, then Q_A and Q_B (each once the
        // previous unit's output store has read Q_X's buffer), then V and K
        // tiles alternately through the two-stage rings, whose phases run on
        // across units.
        int kiss[PP_NSTAGE] = {}, viss[PP_NSTAGE] = {}, nq[2] = {0, 0};
        bool ok = true;
        int g = 0;   // key tiles loaded so far
        int unit = (int)blockIdx.x - (int)gridDim.x;
        PPWork w;
        while (ok && pp_next_unit<SRC>(a, ring, vl, n_units, unit, w)) {
            if (RING && lane == 0 && ring.pos[w.b] < 0) atomicMax(a.ctl.status, SWA_STATUS_BAD_INPUT);
            const int tb = VARLEN ? 0 : w.b;             // batch coordinate of the tensors
            const int row0 = VARLEN ? vl.cu[w.b] : 0;    // tensor row of position 0
            // one K or V tile into stage st
            auto load_tile = [&](bool is_v, int st, long long key0) {
                uint8_t *dst = (is_v ? sV : sK) + st * C::KTILE;
                uint64_t *bar = is_v ? &bars->v_full[st] : &bars->k_full[st];
                if constexpr (RING) {
                    const bool ring_tile = key0 < w.p0;
                    const long long slot0 = ring_tile ? key0 % ring.W : 0;
                    if (!ring_tile || (key0 + PP_BN <= w.p0 && slot0 + PP_BN <= ring.W)) {
                        SWA_DCHECK(ring_tile || key0 - w.p0 < a.T, a.ctl.status);
                        if (lane == 0) {
                            mbar_expect_tx(bar, C::KTILE);
                            for (int ch = 0; ch < C::NCH; ++ch) {
                                if (ring_tile)
                                    tma_load_4d(dst + ch * C::KCH, is_v ? &tmVr : &tmKr, bar, ch * C::E, (int)slot0,
                                                w.hk, w.b);
                                else
                                    tma_load_4d(dst + ch * C::KCH, is_v ? &tmV : &tmK, bar, ch * C::E, w.hk,
                                                (int)(key0 - w.p0), w.b);
                            }
                        }
                        return;
                    }
                    // a tile that meets the chunk's first row or wraps round
                    // the ring's end: rows from wherever each position lives
                    const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(is_v ? a.v : a.k);
                    const __nv_bfloat16 *rc = static_cast<const __nv_bfloat16 *>(is_v ? ring.vc : ring.kc);
                    pp_gather_rows<D>(dst, src, lane, [&](int r) -> const __nv_bfloat16 * {
                        const long long p = key0 + r;
                        if (p >= w.p0) {
                            const long long row = p - w.p0;
                            return row < a.T ? src + (((long long)w.b * a.T + row) * a.Hkv + w.hk) * D : nullptr;
                        }
                        return rc + (((long long)w.b * a.Hkv + w.hk) * ring.W + p % ring.W) * D;
                    });
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar);
                } else {
                    SWA_DCHECK(key0 >= 0 && row0 + key0 < a.T, a.ctl.status);
                    if (lane == 0) {
                        mbar_expect_tx(bar, C::KTILE);
                        for (int ch = 0; ch < C::NCH; ++ch)
                            tma_load_4d(dst + ch * C::KCH, is_v ? &tmV : &tmK, bar, ch * C::E, w.hk,
                                        row0 + (int)key0, tb);
                    }
                }
            };
            // the sink tile: positions 0 .. n_sink-1, zeros after
            auto load_sinks = [&](bool is_v, int st) {
                uint8_t *dst = (is_v ? sV : sK) + st * C::KTILE;
                const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(is_v ? a.v : a.k);
                pp_gather_rows<D>(dst, src, lane, [&](int r) -> const __nv_bfloat16 * {
                    return r < a.g ? src + (((long long)w.b * a.T + r) * a.Hkv + w.hk) * D : nullptr;
                });
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(is_v ? &bars->v_full[st] : &bars->k_full[st]);
            };
            for (int t = 0; t < w.n_tiles && ok; ++t, ++g) {
                const long long key0 = (long long)(w.j_lo + t) * PP_BN;
                const int st = g % PP_NSTAGE;
                const uint32_t par = ((g / PP_NSTAGE) & 1) ^ 1;
                const bool sink_tile = SRC == PP_SINKS && t >= w.n_band;
                ok = warp_wait_bounded(&bars->k_empty[st], par, ctl);
                if (!ok) break;
                if (sink_tile) load_sinks(false, st);
                else load_tile(false, st, key0);
                kiss[st]++;
                if (t == 0) {
                    for (int x = 0; x < 2 && ok; ++x) {
                        if (!w.q[x].active) continue;
                        if (nq[x] > 0) ok = warp_wait_bounded(&bars->q_empty[x], (nq[x] - 1) & 1, ctl);
                        if (!ok) break;
                        if (lane == 0) {
                            mbar_expect_tx(&bars->q_full[x], C::QTILE);
                            for (int ch = 0; ch < C::NCH; ++ch) {
                                SWA_DCHECK(w.q[x].m0 >= 0 && row0 + w.q[x].m0 < a.T && w.q[x].h < a.Hq,
                                           a.ctl.status);
                                tma_load_4d(sQ + x * C::QTILE + ch * C::QCH, &tmQ, &bars->q_full[x], ch * C::E,
                                            w.q[x].h, row0 + w.q[x].m0, tb);
                            }
                        }
                        nq[x]++;
                    }
                    if (!ok) break;
                }
                ok = warp_wait_bounded(&bars->v_empty[st], par, ctl);
                if (!ok) break;
                if (sink_tile) load_sinks(true, st);
                else load_tile(true, st, key0);
                viss[st]++;
            }
        }
        if (!ok && lane == 0) {
            // let our own copies land before the CTA's shared memory goes away
            for (int s = 0; s < PP_NSTAGE; ++s) {
                if (kiss[s] > 0) pp_drain_wait(&bars->k_full[s], (kiss[s] - 1) & 1, a.ctl.limit_ns);
                if (viss[s] > 0) pp_drain_wait(&bars->v_full[s], (viss[s] - 1) & 1, a.ctl.limit_ns);
            }
            for (int x = 0; x < 2; ++x)
                if (nq[x] > 0) pp_drain_wait(&bars->q_full[x], (nq[x] - 1) & 1, a.ctl.limit_ns);
        }
    } else if (warp == 9) {
        // ----------------------------------------------------------- MMA --
        // The whole warp runs the schedule (waits, descriptor arithmetic) in
        // lock step; lane 0 alone issues MMAs and commits.  The key tiles of
        // the CTA's units form one sequence through the stage rings; a
        // unit's first QK^T waits for its Q tiles, which the producer reloads
        // as each of the previous unit's epilogues lets go of its buffer.
        constexpr uint32_t idesc_qk = umma_idesc_bf16(PP_BM, PP_BN, 0, 0);
        constexpr uint32_t idesc_pv = umma_idesc_bf16(PP_BM, D, 0, 1);
        // descriptors are built once; a k-step or stage only adds a constant
        // to the 14-bit start-address field (addresses < 2^18)
        const uint64_t dq0 = umma_smem_desc(smem_u32(sQ), 16, 8 * C::RB, C::LAYOUT);
        const uint64_t dk0 = umma_smem_desc(smem_u32(sK), 16, 8 * C::RB, C::LAYOUT);
        const uint64_t dv0 = umma_smem_desc(smem_u32(sV), C::KCH, 8 * C::RB, C::LAYOUT);
        const bool leader = lane == 0;
        int cnt0 = 0, cnt1 = 0;       // PVs of each query tile so far (all units)
        bool acc0 = false, acc1 = false; // O of the tile holds this unit's sum
        int nq0 = 0, nq1 = 0;         // Q tiles consumed
        bool qw0 = false, qw1 = false; // Q_X of this unit waited for
        bool ok = true;
        PPSched cur;
        // QK^T of query tile X against the key tile in stage st (the unit's
        // first one waits for Q_X)
        auto qk = [&](auto xc, int st) -> bool {
            constexpr int X = decltype(xc)::value;
            bool &qw = X ? qw1 : qw0;
            int &nq = X ? nq1 : nq0;
            if (!qw) {
                if (!warp_wait_bounded(&bars->q_full[X], nq & 1, ctl)) return false;
                nq++;
                qw = true;
                tc_fence_after();
            }
            const uint64_t dq = dq0 + (uint64_t)((X * C::QTILE) >> 4);
            const uint64_t dk = dk0 + (uint64_t)((st * C::KTILE) >> 4);
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int byte = kk * 32;
                    const uint64_t qo = (uint64_t)(((byte / C::RB) * C::QCH + (byte % C::RB)) >> 4);
                    const uint64_t ko = (uint64_t)(((byte / C::RB) * C::KCH + (byte % C::RB)) >> 4);
                    mma_bf16_ss(tmem + pp_col_s(X), dq + qo, dk + ko, idesc_qk, kk > 0 ? 1u : 0u);
                }
                mma_commit(&bars->s_full[X]);
            }
            return true;
        };
        auto pv = [&](auto xc, int st) -> bool {
            constexpr int X = decltype(xc)::value;
            int &cnt = X ? cnt1 : cnt0;
            bool &acc = X ? acc1 : acc0;
            if (!warp_wait_bounded(&bars->p_full[X], cnt & 1, ctl)) return false;
            tc_fence_after();
            const uint64_t dv = dv0 + (uint64_t)((st * C::KTILE) >> 4);
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < PP_BN / 16; ++kk)
                    mma_bf16_ts(tmem + pp_col_o(X), tmem + pp_col_s(X) + kk * 8,
                                dv + (uint64_t)((kk * 16 * C::RB) >> 4), idesc_pv, (acc || kk > 0) ? 1u : 0u);
                mma_commit(&bars->pv_done[X]);
            }
            cnt++;
            acc = true;
            return true;
        };
        const std::integral_constant<int, 0> xA;
        const std::integral_constant<int, 1> xB;
        int unit = (int)blockIdx.x - (int)gridDim.x;
        PPWork wk;
        int g = 0;   // sequence number of the unit's first key tile
        while (ok && pp_next_unit<SRC>(a, ring, vl, n_units, unit, wk)) {
            cur = pp_sched<SRC>(wk);
            qw0 = qw1 = false;
            acc0 = acc1 = false;
            // prologue: QK^T of the unit's first key tile for both query
            // tiles, as soon as their Q tiles are in
            ok = warp_wait_bounded(&bars->k_full[g % PP_NSTAGE], (g / PP_NSTAGE) & 1, ctl);
            if (!ok) break;
            tc_fence_after();
            if (pp_sched_on<SRC, 0>(cur, 0)) ok = qk(xA, g % PP_NSTAGE);
            if (ok && pp_sched_on<SRC, 1>(cur, 0)) ok = qk(xB, g % PP_NSTAGE);
            if (!ok) break;
            if (leader) mma_commit(&bars->k_empty[g % PP_NSTAGE]);
            for (int t = 0; t < cur.n_tiles && ok; ++t) {
                const int gt = g + t;
                const int st = gt % PP_NSTAGE;
                const bool more = t + 1 < cur.n_tiles;
                ok = warp_wait_bounded(&bars->v_full[st], (gt / PP_NSTAGE) & 1, ctl);
                // the next K tile is waited for while tile A's softmax still runs
                if (ok && more) ok = warp_wait_bounded(&bars->k_full[(gt + 1) % PP_NSTAGE], ((gt + 1) / PP_NSTAGE) & 1, ctl);
                if (!ok) break;
                // tile A: PV of key tile t, then QK^T of key tile t+1 into the
                // same S columns (issue order keeps them apart)
                if (pp_sched_on<SRC, 0>(cur, t)) ok = pv(xA, st);
                if (!ok) break;
                if (more) {
                    tc_fence_after();
                    if (pp_sched_on<SRC, 0>(cur, t + 1)) ok = qk(xA, (gt + 1) % PP_NSTAGE);
                    if (!ok) break;
                }
                // tile B likewise, half a step behind
                if (pp_sched_on<SRC, 1>(cur, t)) ok = pv(xB, st);
                if (!ok) break;
                if (leader) mma_commit(&bars->v_empty[st]);
                if (more) {
                    if (pp_sched_on<SRC, 1>(cur, t + 1)) ok = qk(xB, (gt + 1) % PP_NSTAGE);
                    if (!ok) break;
                    if (leader) mma_commit(&bars->k_empty[(gt + 1) % PP_NSTAGE]);
                }
                __syncwarp();
            }
            g += cur.n_tiles;
        }
        // all MMAs lane 0 issued are complete before TMEM is freed
        if (leader) {
            mma_commit(&bars->drain);
            pp_drain_wait(&bars->drain, 0, a.ctl.limit_ns);
        }
        __syncwarp();
    } else {
        // ------------------------------------------- softmax + epilogue --
        const int x = warp / 4;                 // query tile of this warpgroup
        const int quarter = warp % 4;
        const int r = quarter * 32 + lane;      // row in tile = TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t s_addr = tmem + lane_off + pp_col_s(x);
        const uint32_t o_addr = tmem + lane_off + pp_col_o(x);
        // key positions: 64-bit only for a chunk continuing a ring
        typedef typename std::conditional<RING, long long, int>::type kpos_t;
        bool ok = true;
        int cs = 0;   // key tiles of this query tile so far (all units)
        int ns = 0;   // output tiles staged so far
        int unit = (int)blockIdx.x - (int)gridDim.x;
        PPWork w;
        while (ok && pp_next_unit<SRC>(a, ring, vl, n_units, unit, w)) {
            const PPTile qt = x ? w.q[1] : w.q[0];
            if (!qt.active) continue;
            const int tb = VARLEN ? 0 : w.b;             // batch coordinate of the tensors
            const int row0 = VARLEN ? vl.cu[w.b] : 0;    // tensor row of position 0
            const kpos_t p0 = RING ? (kpos_t)w.p0 : 0;
            const kpos_t kend = (RING || VARLEN) ? (kpos_t)w.kend : (kpos_t)a.T;   // one past the last key
            const int left = VARLEN ? varlen_left(vl, w.b, a.left) : a.left;   // keys before the query
            const int i_row = qt.m0 + r;            // row in q / o / lse
            const kpos_t ip = p0 + i_row;           // query position
            const bool row_real = r < qt.nrows;
            const bool warp_has_rows = quarter * 32 < qt.nrows;
            const kpos_t wi0 = p0 + qt.m0 + quarter * 32, wi1 = wi0 + 31;
            float m = -CUDART_INF_F, l = 0.f;
            int c = 0;   // key tiles of this query tile in this unit
            for (int t = 0; t < w.n_tiles; ++t) {
                if (!pp_active<SRC>(qt, w.n_band, t)) continue;
                ok = warp_wait_bounded(&bars->s_full[x], cs & 1, ctl);
                if (!ok) break;
                tc_fence_after();
                // which 32-key chunks can any row of this warp see
                const kpos_t key0 = (kpos_t)(w.j_lo + t) * PP_BN;
                int c_lo = 0, c_hi = -1;
                bool interior = false;
                if (warp_has_rows) {
                    const kpos_t lo = max(max(key0, (kpos_t)(wi0 - left)), (kpos_t)0);
                    const kpos_t hi = min(min(key0 + PP_BN - 1, (kpos_t)(wi1 + a.right)), kend - 1);
                    if (lo <= hi) {
                        c_lo = (int)((lo - key0) / 32);
                        c_hi = (int)((hi - key0) / 32);
                    }
                    interior = (key0 + PP_BN - 1 < kend) && band_contains(wi1, key0, left, a.right) &&
                               band_contains(wi0, key0 + PP_BN - 1, left, a.right);
                }
                SWA_DCHECK(c_lo >= 0 && c_hi < PP_BN / 32, a.ctl.status);
                // visible columns of this row
                int col_lo = (int)max(ip - left - key0, (kpos_t)0);
                int col_hi = (int)min(min((kpos_t)(ip + a.right), kend - 1) - key0, (kpos_t)(PP_BN - 1));
                if (SRC == PP_SINKS && t >= w.n_band) {
                    // sink positions 0 .. n_sink-1 below the row's window (the
                    // ones inside it were counted there; causal: all <= the row)
                    col_lo = 0;
                    col_hi = min(a.g, (int)(ip - a.left)) - 1;
                    const int last = warp_has_rows ? min(a.g, (int)(wi1 - a.left)) - 1 : -1;
                    c_lo = 0;
                    c_hi = last >= 0 ? last / 32 : -1;
                    interior = false;
                }
                bool rescale_o;
                float alpha;
                if (interior && c_lo == 0 && c_hi == PP_BN / 32 - 1)
                    pp_softmax_tile<true>(s_addr, c_lo, c_hi, col_lo, col_hi, a.scale_log2, m, l, rescale_o, alpha,
                                          c == 0);
                else
                    pp_softmax_tile<false>(s_addr, c_lo, c_hi, col_lo, col_hi, a.scale_log2, m, l, rescale_o, alpha,
                                           c == 0);
                // O rescale (rare): wait for the previous tile's PV, which
                // accumulates into O; this tile's PV waits for P
                if (__any_sync(0xffffffffu, rescale_o)) {
                    ok = warp_wait_bounded(&bars->pv_done[x], (cs - 1) & 1, ctl);
                    if (!ok) break;
                    tc_fence_after();
                    const float f = rescale_o ? alpha : 1.f;
#pragma unroll 1
                    for (int cc = 0; cc < D / 16; ++cc) {
                        float ov[16];
                        tmem_ld16(o_addr + cc * 16, ov);
                        tmem_ld_wait_dep16(ov);
                        uint32_t ou[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) ou[e] = __float_as_uint(ov[e] * f);
                        tmem_st16u(o_addr + cc * 16, ou);
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->p_full[x]);
                c++;
                cs++;
            }
            if (!ok) break;

            // ---- epilogue: O / l -> bf16 -> Q_X's buffer -> TMA store ----
            // Q_X is no longer read (its last QK^T precedes the last PV); the
            // producer reloads it for the next unit once the store has read
            // it.  The last tile of a packed sequence goes row by row (a tile
            // store would run into the next sequence).  The next unit's first
            // PV, which overwrites O, waits for this warpgroup's next P, so it
            // comes after these reads.
            if (c > 0) ok = warp_wait_bounded(&bars->pv_done[x], (cs - 1) & 1, ctl);
            if (!ok) break;
            tc_fence_after();
            const bool direct = VARLEN && qt.nrows < PP_BM;
            const float inv = (l > 0.f) ? 1.f / l : 0.f;
            uint8_t *stg = sQ + x * C::QTILE;
            __nv_bfloat16 *orow = static_cast<__nv_bfloat16 *>(a.o) +
                                  (((long long)tb * a.T + row0 + i_row) * a.Hq + qt.h) * D;
            SWA_DCHECK(!row_real || row0 + i_row < a.T, a.ctl.status);
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
                float ov[32];
                tmem_ld32(o_addr + cc * 32, ov);
                tmem_ld_wait_dep(ov);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    uint4 pk;
                    pk.x = pack_bf16x2(ov[u * 8 + 0] * inv, ov[u * 8 + 1] * inv);
                    pk.y = pack_bf16x2(ov[u * 8 + 2] * inv, ov[u * 8 + 3] * inv);
                    pk.z = pack_bf16x2(ov[u * 8 + 4] * inv, ov[u * 8 + 5] * inv);
                    pk.w = pack_bf16x2(ov[u * 8 + 6] * inv, ov[u * 8 + 7] * inv);
                    if (direct) {
                        if (row_real) *reinterpret_cast<uint4 *>(orow + cc * 32 + u * 8) = pk;
                    } else {
                        *reinterpret_cast<uint4 *>(stg + pp_tile_offset<D>(r, cc * 32 + u * 8, C::QCH)) = pk;
                    }
                }
            }
            if (a.lse && row_real)
                a.lse[((long long)tb * a.Hq + qt.h) * a.T + row0 + i_row] =
                    (l > 0.f) ? (m + __log2f(l)) * 0.69314718055994530942f : -CUDART_INF_F;
            // tile staged -> one thread stores it (rows past T are clipped by
            // the tensor map; an abort skips the store) and hands Q_X's
            // buffer back to the producer
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->epi[x]);
            if (r == 0) {
                if (wait_bounded(&bars->epi[x], ns & 1, ctl) && !bars->abort && !direct) {
                    for (int ch = 0; ch < C::NCH; ++ch)
                        tma_store_4d(&tmO, stg + ch * C::QCH, ch * C::E, qt.h, row0 + qt.m0, tb);
                    tma_store_commit();
                    pp_store_wait_read();
                }
                mbar_arrive(&bars->q_empty[x]);
            }
            ns++;
        }
        // the output stores are complete before the CTA ends
        if (r == 0) tma_store_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// Ring cache [B,Hkv,W,D] bf16 viewed as (D, W, Hkv, B); box = one chunk of
// 128 consecutive slots of one kv head.
template <int D>
bool pp_make_ring_map(CUtensorMap *m, const void *ptr, int B, int Hkv, int W)
{
    using C = PCfg<D>;
    EncodeTiledFn enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)W, (cuuint64_t)Hkv, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)W * D * 2, (cuuint64_t)Hkv * W * D * 2};
    cuuint32_t box[4] = {(cuuint32_t)C::E, (cuuint32_t)PP_BN, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE,
                     C::RB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Windows of at most this many keys take the persistent kernel: its units
// are short, so the start and end it saves per unit pay; measured (T =
// 16384, ms, persistent against one CTA per unit) d = 128 W = 256 / 512 /
// 1024: 0.182 / 0.240 / 0.355 against 0.217 / 0.274 / 0.380; d = 64 W = 256:
// 0.164 against 0.192; d = 32 W = 256 / 1024: 0.158 / 0.310 against 0.179 /
// 0.324; symmetric W = 512 (Longformer shapes, no globals) d = 128 / 64:
// 0.212 / 0.197 against 0.228 / 0.205; but W = 2048 about equal (d = 128
// 0.577 against 0.585, d = 64 0.533 against 0.528) and the Mistral-7B
// prefill (W = 4096) 2.030 against 1.991 ms.
constexpr int PP_PERSIST_MAX_WINDOW = 1024;

template <int D, int SRC, bool PERSIST>
cudaError_t launch_pp_d(const TcPrefillArgs &a, const RingArgs &ring, const VarlenArgs &vl, cudaStream_t s)
{
    using C = PCfg<D>;
    constexpr bool RING = SRC == PP_RING;
    constexpr bool VARLEN = SRC == PP_VARLEN;
    // packed sequences: the tensors as one sequence of `total` rows
    const int TB = VARLEN ? 1 : a.B;
    CUtensorMap mq, mk, mv, mo, mkr, mvr;
    if (!make_bthd_map(&mq, a.q, TB, a.T, a.Hq, D, PP_BM) || !make_bthd_map(&mk, a.k, TB, a.T, a.Hkv, D, PP_BN) ||
        !make_bthd_map(&mv, a.v, TB, a.T, a.Hkv, D, PP_BN) || !make_bthd_map(&mo, a.o, TB, a.T, a.Hq, D, PP_BM))
        return cudaErrorInvalidValue;
    if (RING) {
        if (!pp_make_ring_map<D>(&mkr, ring.kc, a.B, a.Hkv, ring.W) ||
            !pp_make_ring_map<D>(&mvr, ring.vc, a.B, a.Hkv, ring.W))
            return cudaErrorInvalidValue;
    } else {
        mkr = mk;   // unused without a ring
        mvr = mv;
    }
    static DeviceOnce once;
    int n_sm = 0;
    cudaError_t e = once.get(
        [&](int) {
            return PERSIST ? cudaFuncSetAttribute(swa_prefill_pp_persistent_kernel<D, SRC>,
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES)
                           : cudaFuncSetAttribute(swa_prefill_pp_kernel<D, SRC>,
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        },
        &n_sm);
    if (e != cudaSuccess) return e;
    const int G = a.Hq / a.Hkv;
    // units over (sequence, query tile [pair], head [pair]); for packed
    // sequences the longest one sets the tiles and units past a sequence's
    // end return at once (are skipped, persistent)
    const int nqt = ((VARLEN ? vl.max_len : a.T) + PP_BM - 1) / PP_BM;
    const long long units = (long long)a.B * ((G % 2 == 0) ? (a.Hq / 2) * nqt : a.Hq * ((nqt + 1) / 2));
    if (units == 0) return cudaSuccess;
    if (units > 0x7fffffffLL) return cudaErrorInvalidValue;
    if constexpr (PERSIST) {
        // one CTA per SM takes units blockIdx.x, blockIdx.x + gridDim.x, ...
        const int grid = (int)(units < n_sm ? units : n_sm);
        swa_prefill_pp_persistent_kernel<D, SRC><<<grid, PP_THREADS, C::SMEM_BYTES, s>>>(mq, mk, mv, mo, mkr, mvr, a,
                                                                                           ring, vl, (int)units);
    } else {
        swa_prefill_pp_kernel<D, SRC><<<(int)units, PP_THREADS, C::SMEM_BYTES, s>>>(mq, mk, mv, mo, mkr, mvr, a,
                                                                                      ring, vl);
    }
    return cudaGetLastError();
}

}  // namespace

// Measured on B200 against the 64-key band kernel (same process, same
// inputs, T = 16384 unless stated, ms): d = 128, causal W = 256 / 512: 0.220 /
// 0.278 against 0.238 / 0.312; W = 1024 equal; Mistral-7B prefill (W = 4096,
// T = 32768) 2.007 against 2.666; d = 64, W = 256 / 512: 0.194 / 0.246
// against 0.206 / 0.273; d = 32, W = 256 / 1024: 0.181 / 0.327 against 0.196
// / 0.397; symmetric W = 512 (Longformer shapes, no globals) d = 64 0.207
// against 0.225, d = 128 0.230 against 0.250.  So it takes every plain band
// prefill (no global tokens) whose window spans at least 256 keys.
bool prefill_pp_applies(int d, const TcPrefillArgs &a)
{
    // no global keys; attention sinks (gidx null, g > 0) with a causal window
    // and at most one key tile of them
    const bool keys_ok = a.gidx == nullptr && (a.g == 0 || (a.g <= PP_BN && a.right == 0));
    return (d == 32 || d == 64 || d == 128) && keys_ok && a.left + a.right + 1 >= 256;
}

template <int SRC, bool PERSIST>
cudaError_t launch_pp_src(int d, const TcPrefillArgs &a, const RingArgs &ring, const VarlenArgs &vl, cudaStream_t s)
{
    return d == 128 ? launch_pp_d<128, SRC, PERSIST>(a, ring, vl, s)
           : d == 64 ? launch_pp_d<64, SRC, PERSIST>(a, ring, vl, s)
                     : launch_pp_d<32, SRC, PERSIST>(a, ring, vl, s);
}

template <int SRC>
cudaError_t launch_pp_any(int d, const TcPrefillArgs &a, const RingArgs &ring, const VarlenArgs &vl, cudaStream_t s)
{
    return a.left + a.right + 1 <= PP_PERSIST_MAX_WINDOW ? launch_pp_src<SRC, true>(d, a, ring, vl, s)
                                                         : launch_pp_src<SRC, false>(d, a, ring, vl, s);
}

cudaError_t launch_prefill_pp(int d, const TcPrefillArgs &a, const RingArgs &ring, cudaStream_t s)
{
    if (!prefill_pp_applies(d, a)) return cudaErrorInvalidValue;
    const VarlenArgs vl{nullptr, 0, nullptr};
    if (ring.pos) {
        if (a.g > 0) return cudaErrorInvalidValue;
        return launch_pp_any<PP_RING>(d, a, ring, vl, s);
    }
    if (a.g > 0) return launch_pp_any<PP_SINKS>(d, a, ring, vl, s);
    return launch_pp_any<PP_PLAIN>(d, a, ring, vl, s);
}

// Packed sequences (causal, no sinks): the call's window, clipped to the
// longest sequence, or with one window per sequence the longest sequence
// itself, spans at least 256 keys.  With one window per sequence the host
// does not read the windows, so short ones run here too (correct, though
// below 256 keys the 64-key kernel would be the faster one).
bool prefill_pp_varlen_applies(int d, const TcPrefillArgs &a, const VarlenArgs &vl)
{
    return (d == 32 || d == 64 || d == 128) && vl.cu != nullptr && a.gidx == nullptr && a.g == 0 && a.right == 0 &&
           a.left + 1 >= 256;
}

cudaError_t launch_prefill_pp_varlen(int d, const TcPrefillArgs &a, const VarlenArgs &vl, cudaStream_t s)
{
    if (!prefill_pp_varlen_applies(d, a, vl)) return cudaErrorInvalidValue;
    const RingArgs ring{nullptr, nullptr, nullptr, 0};
    return launch_pp_any<PP_VARLEN>(d, a, ring, vl, s);
}

}  // namespace swa
