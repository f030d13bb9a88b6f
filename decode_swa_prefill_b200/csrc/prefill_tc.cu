// Sliding-window prefill on tcgen05 tensor cores (sm_100a).
//
// What it computes (the pages' definition): for query row i, softmax over the
// keys of its window of scale*q.k, logits outside the window being -inf, then
// the weighted sum of value rows ("Sliding Window Attention", robocikowo.com,
// opening definition).  The [T,T] score matrix never exists: a CTA streams
// only the 64-key tiles that intersect its query tiles' windows, skipping
// every tile that lies fully outside them (the fused-kernel point of the same
// page and of the Ultralytics glossary's FlashAttention entry).  Work per
// query tile is O(W*d), total O(T*W*d).
//
// CTA anatomy (384 threads, one CTA per SM), two 128-row query tiles X = A, B
// that share one kv head, hence every K/V tile: the two query heads of a GQA
// pair at the same rows, or (odd group size) two consecutive row tiles of one
// head, whose key ranges are then merged.
//   warps 0-3  softmax + epilogue of tile A: thread r owns row r = TMEM lane r
//   warps 4-7  the same for tile B (warp w touches TMEM lanes 32(w%4)...)
//   warp 8     producer: TMA tile loads of Q, K, V (no multicast), or
//              cp.async gathers for global keys / global query rows
//   warp 9     TMEM allocator; with warp 10, the MMA issuers: warp 9 + X runs
//              tile X's schedule and its lane 0 issues X's tcgen05.mma, so a
//              wait on one tile never holds up the other tile's MMAs
//   warp 11    idle: it completes warpgroup 2 (warps 8-11), which hands
//              registers to the softmax warpgroups (setmaxnreg) -- three
//              warps on a sub-partition cap a thread at 168 registers, where
//              the softmax spilled
// TMEM (all 512 columns):
//   S[X][b]  columns 128X + 64b: fp32 scores of one 64-key tile, b = buffer
//   P[X][b]  the first 32 columns of S[X][b]: bf16 probabilities (pairs)
//   O[X]     columns 256 + 128X: fp32 output accumulator (d <= 128)
// Per key tile t, for each query tile X, with c = X's running tile count and
// b = c & 1:
//   S[X][b] = Q_X K_t^T             (A, B operands from shared memory)
//   softmax: S -> registers (one TMEM round trip), -inf outside the window
//            (edge tiles only), running row max in log2 units,
//            P = 2^(S*scale*log2e - m) -> bf16 -> TMEM over S[X][b]
//   O[X] += P[X][b] V_t             (A from TMEM, B from shared memory)
// QK^T of the next tile runs while the softmax of this one works, and the two
// softmax warpgroups of the CTA hide each other's latencies.  S[X][b] is only
// recomputed once the PV that read P[X][b] two tiles earlier has completed.
// Every barrier that alternates between the two S buffers is kept per buffer,
// so no waiter can fall two phases behind (the parity of an mbarrier phase
// only names the phase modulo two).
//
// The running max is only raised when a tile's max exceeds it by more than
// 2^8; P then stays <= 256 and O, l share one reference, so the final O/l is
// exact; raising it rescales l and the O row in TMEM.  Per warp, 32-key
// chunks that no row of the warp can see are skipped.  Three quarters of the
// exponentials run on the MUFU (ex2.approx), one quarter as a range-reduced
// cubic on the FMA pipe (exp2_poly2), which shortens the MUFU time per tile.
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

constexpr int BM = 128;              // query rows per tile (= TMEM lanes)
constexpr int BN = 64;               // keys per key tile
constexpr int NSTAGE = 3;            // K and V pipeline depth
constexpr int NTHREADS = 384;
// registers per thread after the split: 256 x 200 + 128 x 104 = 384 x 168,
// the block's launch total (checked on the host before each launch: an
// increase the block cannot cover would wait for ever).  Measured against
// 11 warps at 168: Longformer prefill 0.316 -> 0.293 ms, causal W = 128 (d
// = 128) 0.201 -> 0.193 ms, W = 192 (d = 64) 0.190 -> 0.180 ms (T = 16384).
constexpr int TC_REG_SOFTMAX = 200, TC_REG_OTHER = 104;
constexpr float RESCALE_LOG2 = 8.0f; // raise the running max only beyond 2^8
constexpr int POLY_EVERY = 4;        // every 4th pair of exponentials on the FMA pipe
constexpr int SM_SMEM = 228 * 1024;  // shared memory per SM

template <int D>
struct Cfg {
    static constexpr int RB = (D * 2 >= 128) ? 128 : D * 2; // bytes per swizzled row
    static constexpr int E = RB / 2;                         // elements per chunk row
    static constexpr int NCH = D / E;                        // chunks per head row
    static constexpr int QCH = BM * RB;                      // one chunk of a 128-row tile
    static constexpr int KCH = BN * RB;                      // one chunk of a 64-row tile
    static constexpr int QTILE = BM * D * 2;
    static constexpr int KTILE = BN * D * 2;
    static constexpr uint32_t LAYOUT = (RB == 128) ? UMMA_SW128 : UMMA_SW64;
    static constexpr int OFF_Q = 0;                          // Q_A, Q_B
    static constexpr int OFF_K = OFF_Q + 2 * QTILE;
    static constexpr int OFF_V = OFF_K + NSTAGE * KTILE;
    static constexpr int OFF_BAR = OFF_V + NSTAGE * KTILE;
    // + room to align the base to 1 KiB; more than half the SM's shared
    // memory so that a second CTA never shares the SM (each CTA takes all
    // 512 TMEM columns)
    static constexpr int SMEM_NEED = OFF_BAR + 512 + 1024;
    static constexpr int SMEM_BYTES = SMEM_NEED > 120 * 1024 ? SMEM_NEED : 120 * 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(D == 32 || D == 64 || D == 128, "head dim");
    static_assert(SMEM_BYTES + 1024 <= SM_SMEM, "fits one SM");
    static_assert(2 * (SMEM_BYTES + 1024) > SM_SMEM, "never two CTAs per SM");
};

__host__ __device__ constexpr uint32_t col_s(int x, int b) { return 128u * x + 64u * b; }
__host__ __device__ constexpr uint32_t col_o(int x) { return 256u + 128u * x; }

// Byte offset of element e of row r inside a swizzled [rows][D] tile whose
// E-element chunks are `ch_bytes` apart (the layout of a TMA SWIZZLE_128B /
// SWIZZLE_64B load).
template <int D>
__device__ __forceinline__ uint32_t tile_offset(int r, int e, int ch_bytes)
{
    using C = Cfg<D>;
    const int ch = e / C::E;
    const int u = (e % C::E) / 8;
    const int phys = (C::RB == 128) ? (u ^ (r & 7)) : (u ^ ((r >> 1) & 3));
    return ch * ch_bytes + r * C::RB + phys * 16;
}

struct Bars {
    uint64_t q_full;
    uint64_t k_full[NSTAGE];
    uint64_t k_empty[NSTAGE];
    uint64_t v_full[NSTAGE];
    uint64_t v_empty[NSTAGE];
    uint64_t s_full[2][2];   // [tile][buffer]
    uint64_t p_full[2][2];   // [tile][buffer], one arrival per softmax warp
    uint64_t pv_done[2][2];  // [tile][buffer]
    uint64_t drain[2];
    uint64_t epi[2];
    uint64_t a_first;        // tile A's first QK^T complete (used once)
    uint32_t tmem_base;
    int abort;
};

// Time-only bound (ignores the abort flag): used to drain after an abort.
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity, unsigned long long limit)
{
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > limit) return;
    }
}

// One 128-row query tile of a CTA.
struct QTile {
    int h;        // query head
    int m0;       // first row (band mode)
    int gt;       // group of 128 global rows (dense-row mode)
    int nrows;    // real rows
    int ts, te;   // band key tiles [ts, te) it needs, relative to j_lo
    bool active;
};

// The per-CTA work description every role derives identically.
struct Work {
    int mode;     // 0 band tiles, 1 dense global rows
    int b, hk;
    QTile q[2];
    int j_lo;     // first band key tile (absolute, 64-key units)
    int n_band;   // band key tiles streamed by TMA
    int n_glob;   // gathered tiles of global keys (band mode with globals)
    int n_tiles;
    long long p0;   // position of query row 0 (a chunk continuing a ring; else 0)
    long long kend; // one past the last key position (p0 + T)
};

// Does query tile q use key tile t, and which of its tiles is it?
__device__ __forceinline__ bool tile_active(const QTile &q, int n_band, int t)
{
    return q.active && (t >= n_band || (t >= q.ts && t < q.te));
}
__device__ __forceinline__ int tile_count(const QTile &q, int n_band, int t)
{
    return t < n_band ? t - q.ts : (q.te - q.ts) + (t - n_band);
}
__device__ __forceinline__ int tiles_of(const QTile &q, int n_glob)
{
    return q.active ? (q.te - q.ts) + n_glob : 0;
}

template <bool RING, bool SINKS, bool VARLEN>
__device__ __forceinline__ Work make_work(const TcPrefillArgs &a, const RingArgs &ring, const VarlenArgs &vl,
                                          int n_mode1)
{
    Work w;
    const int G = a.Hq / a.Hkv;
    const bool pair_heads = (G % 2) == 0;
    // query tiles per sequence (the longest one for packed sequences)
    const int nqt = ((VARLEN ? vl.max_len : a.T) + BM - 1) / BM;
    const int nkt = (a.T + BN - 1) / BN;
    const int ngt = (a.g + BM - 1) / BM;
    int bid = blockIdx.x;
    for (int x = 0; x < 2; ++x) w.q[x] = QTile{0, 0, 0, 0, 0, 0, false};
    if (bid < n_mode1) {
        w.mode = 1;
        if (pair_heads) {
            const int hp = bid % (a.Hq / 2);
            const int gt = (bid / (a.Hq / 2)) % ngt;
            w.b = bid / ((a.Hq / 2) * ngt);
            for (int x = 0; x < 2; ++x) w.q[x] = QTile{2 * hp + x, 0, gt, min(BM, a.g - gt * BM), 0, nkt, true};
        } else {
            const int h = bid % a.Hq;
            const int ngp = (ngt + 1) / 2;
            const int gp = (bid / a.Hq) % ngp;
            w.b = bid / (a.Hq * ngp);
            for (int x = 0; x < 2; ++x) {
                const int gt = 2 * gp + x;
                if (gt < ngt) w.q[x] = QTile{h, 0, gt, min(BM, a.g - gt * BM), 0, nkt, true};
            }
        }
        w.j_lo = 0;
        w.n_band = nkt;
        w.n_glob = 0;
        w.p0 = 0;
        w.kend = a.T;
    } else {
        bid -= n_mode1;
        w.mode = 0;
        // query tiles in descending order: the CTAs the hardware starts last
        // are the short ones at the start of a causal sequence, which fill
        // the tail of the grid instead of full-window CTAs
        if (pair_heads) {
            const int hp = bid % (a.Hq / 2);
            const int qt = nqt - 1 - (bid / (a.Hq / 2)) % nqt;
            w.b = bid / ((a.Hq / 2) * nqt);
            for (int x = 0; x < 2; ++x)
                w.q[x] = QTile{2 * hp + x, qt * BM, 0, min(BM, a.T - qt * BM), 0, 0, true};
        } else {
            const int h = bid % a.Hq;
            const int nqp = (nqt + 1) / 2;
            const int qp = nqp - 1 - (bid / a.Hq) % nqp;
            w.b = bid / (a.Hq * nqp);
            for (int x = 0; x < 2; ++x) {
                const int qt = 2 * qp + x;
                if (qt < nqt) w.q[x] = QTile{h, qt * BM, 0, min(BM, a.T - qt * BM), 0, 0, true};
            }
        }
        if constexpr (RING) {
            // a chunk continuing a ring starts at position pos[b] (a
            // negative entry is read as 0; the producer records it); key
            // tiles are counted in absolute positions
            const long long p0 = max((long long)ring.pos[w.b], 0LL);
            w.p0 = p0;
            w.kend = p0 + a.T;
            long long lo = w.kend, hi = -1;
            long long lo_x[2] = {0, 0}, hi_x[2] = {0, 0};
            for (int x = 0; x < 2; ++x) {
                if (!w.q[x].active) continue;
                lo_x[x] = max(0LL, p0 + w.q[x].m0 - a.left);
                hi_x[x] = min(w.kend - 1, p0 + w.q[x].m0 + BM - 1 + a.right);
                lo = min(lo, lo_x[x]);
                hi = max(hi, hi_x[x]);
            }
            w.j_lo = (int)(lo / BN);
            w.n_band = (int)(hi / BN) - w.j_lo + 1;
            for (int x = 0; x < 2; ++x)
                if (w.q[x].active) {
                    w.q[x].ts = (int)(lo_x[x] / BN) - w.j_lo;
                    w.q[x].te = (int)(hi_x[x] / BN) - w.j_lo + 1;
                }
        } else {
            // sequence length (a packed sequence: its own; tiles past it idle)
            int TT = a.T;
            int left = a.left;
            if constexpr (VARLEN) {
                // an inconsistent entry (decreasing, past the rows, longer
                // than max_len, a window below 1) makes the sequence empty;
                // the CTA reports it
                TT = varlen_ok(vl, w.b, a.T) ? vl.cu[w.b + 1] - vl.cu[w.b] : 0;
                left = varlen_left(vl, w.b, a.left);
                for (int x = 0; x < 2; ++x) {
                    if (w.q[x].m0 >= TT) w.q[x].active = false;
                    w.q[x].nrows = min(BM, TT - w.q[x].m0);
                }
            }
            w.p0 = 0;
            w.kend = TT;
            int lo = TT, hi = -1;
            int lo_x[2] = {0, 0}, hi_x[2] = {0, 0};
            for (int x = 0; x < 2; ++x) {
                if (!w.q[x].active) continue;
                lo_x[x] = max(0, w.q[x].m0 - left);
                hi_x[x] = min(TT - 1, w.q[x].m0 + BM - 1 + a.right);
                lo = min(lo, lo_x[x]);
                hi = max(hi, hi_x[x]);
            }
            w.j_lo = lo / BN;
            w.n_band = hi / BN - w.j_lo + 1;
            for (int x = 0; x < 2; ++x)
                if (w.q[x].active) {
                    w.q[x].ts = lo_x[x] / BN - w.j_lo;
                    w.q[x].te = hi_x[x] / BN - w.j_lo + 1;
                }
        }
        // gathered tiles of global keys, or (SINKS) of the first g positions
        w.n_glob = ((SINKS || a.gidx != nullptr) && a.g > 0) ? (a.g + BN - 1) / BN : 0;
    }
    w.hk = w.q[0].h / G;
    w.n_tiles = w.n_band + w.n_glob;
    return w;
}

// Key columns of tile t that the MMAs compute (a multiple of 32): all 64 of a
// band tile, the real global keys of a gathered tile rounded up.
__device__ __forceinline__ int tile_cols(const Work &w, const TcPrefillArgs &a, int t)
{
    if (t < w.n_band) return BN;
    const int n = min(BN, a.g - (t - w.n_band) * BN);
    return (n + 31) & ~31;
}

// Producer-warp gather of up to `rows` rows (positions from `rows_idx`) of
// one head into a swizzled tile with 16-byte cp.async copies, all in flight
// at once; rows past `nrows` are zero-filled.  All 32 lanes.
template <int D>
__device__ __forceinline__ void gather_tile(uint8_t *dst, int rows, int ch_bytes, const __nv_bfloat16 *base,
                                            const int32_t *rows_idx, int nrows, int b, int T, int H, int head,
                                            int lane, int *status)
{
    constexpr int GR = D / 8; // 16-byte granules per row
    (void)status;
    for (int idx = lane; idx < rows * GR; idx += 32) {
        const int r = idx / GR, u = idx % GR;
        const long long pos = r < nrows ? rows_idx[r] : 0;
        SWA_DCHECK(pos >= 0 && pos < T, status);
        const __nv_bfloat16 *src = base + (((long long)b * T + pos) * H + head) * D + u * 8;
        cp_async16(dst + tile_offset<D>(r, u * 8, ch_bytes), src, r < nrows ? 16u : 0u);
    }
    cp_async_wait_all();
}

// Producer-warp gather of `rows` rows into a swizzled tile with 16-byte
// cp.async copies; row_src(r) gives row r's source, or null for zeros.  All
// 32 lanes.
template <int D, typename RowSrc>
__device__ __forceinline__ void gather_rows(uint8_t *dst, int rows, int ch_bytes, const __nv_bfloat16 *any_valid,
                                            int lane, RowSrc row_src)
{
    constexpr int GR = D / 8; // 16-byte granules per row
    for (int idx = lane; idx < rows * GR; idx += 32) {
        const int r = idx / GR, u = idx % GR;
        const __nv_bfloat16 *src = row_src(r);
        cp_async16(dst + tile_offset<D>(r, u * 8, ch_bytes), src ? src + u * 8 : any_valid, src ? 16u : 0u);
    }
    cp_async_wait_all();
}

// Gathered key tile of sink positions first .. first+nrows-1 (zeros after).
template <int D>
__device__ __forceinline__ void gather_sinks(uint8_t *dst, const __nv_bfloat16 *base, int first, int nrows, int b,
                                             int T, int H, int head, int lane)
{
    gather_rows<D>(dst, BN, Cfg<D>::KCH, base, lane, [&](int r) -> const __nv_bfloat16 * {
        return r < nrows ? base + (((long long)b * T + first + r) * H + head) * D : nullptr;
    });
}

// Everything the softmax of one 64-key tile needs besides the scores.
struct TileCtx {
    uint32_t s_addr;      // TMEM address of this warp's lanes of S[X][b]
    int c_lo, c_hi;       // live 32-key chunks of the warp
    int col_lo, col_hi;   // visible columns of this row (band / dense tiles)
    bool by_range;        // mask by [col_lo, col_hi] (else: global-key tile)
    int gc_base;          // first global index of a gathered tile
    long long i_row;
};

// Softmax of one tile for one row: scores -> running max / sum -> P (bf16)
// over the first 32 columns of the tile's TMEM buffer.  FULL: every key of
// the tile is visible to every row of the warp (no masking, all chunks live),
// the common case, compiled without any of the masking branches.
template <bool FULL, bool SINKS>
__device__ __forceinline__ void softmax_tile(const TileCtx &k, const TcPrefillArgs &a, const int32_t *gb, float &m,
                                             float &l, bool &rescale, float &alpha, bool first)
{
    auto live = [&](int cc) { return FULL || (cc >= k.c_lo && cc <= k.c_hi); };
    float sr[BN];
#pragma unroll
    for (int cc = 0; cc < BN / 32; ++cc)
        if (live(cc)) tmem_ld32(k.s_addr + cc * 32, sr + cc * 32);
    tmem_ld_wait_dep(sr);
#pragma unroll
    for (int cc = 1; cc < BN / 32; ++cc) reg_fence32(sr + cc * 32);
    if (!FULL) {
#pragma unroll
        for (int cc = 0; cc < BN / 32; ++cc) {
            if (!live(cc)) {
#pragma unroll
                for (int e = 0; e < 32; ++e) sr[cc * 32 + e] = -CUDART_INF_F;
            } else if (k.by_range) {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int xx = cc * 32 + e;
                    if (xx < k.col_lo || xx > k.col_hi) sr[xx] = -CUDART_INF_F;
                }
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int gc = k.gc_base + cc * 32 + e;
                    bool keep;
                    if constexpr (SINKS) // sink position gc: up to the query's own position
                        keep = gc < a.g && gc <= k.i_row && !band_contains(k.i_row, gc, a.left, a.right);
                    else
                        keep = gc < a.g && !band_contains(k.i_row, __ldg(gb + gc), a.left, a.right);
                    if (!keep) sr[cc * 32 + e] = -CUDART_INF_F;
                }
            }
        }
    }
    float mx4[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) mx4[j] = fmax3(sr[j], sr[4 + j], sr[8 + j]);
#pragma unroll
    for (int cc = 12; cc + 8 <= BN; cc += 8)
#pragma unroll
        for (int j = 0; j < 4; ++j) mx4[j] = fmax3(mx4[j], sr[cc + j], sr[cc + 4 + j]);
#pragma unroll
    for (int cc = 12 + ((BN - 12) / 8) * 8; cc < BN; cc += 4)
#pragma unroll
        for (int j = 0; j < 4; ++j) mx4[j] = fmaxf(mx4[j], sr[cc + j]);
    const float mt = fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3])) * a.scale_log2;
    rescale = false;
    alpha = 1.f;
    if (mt > m + RESCALE_LOG2) {
        alpha = ex2_approx(m - mt);     // 0 when m was -inf
        l *= alpha;
        rescale = !first;
        m = mt;
    }
    const float ref = (m == -CUDART_INF_F) ? 0.f : m;
    const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
    const float2 nr2 = make_float2(-ref, -ref);
    float2 acc2 = make_float2(0.f, 0.f), acc2b = make_float2(0.f, 0.f);
#pragma unroll
    for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t pk[16];
        if (live(cc)) {
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
                const int xx = cc * 32 + e;
                float2 y = fma2(make_float2(sr[xx], sr[xx + 1]), sc2, nr2);
                if ((e / 2) % POLY_EVERY == POLY_EVERY - 1) {
                    y = exp2_poly2(y);
                } else {
                    y.x = ex2_approx(y.x);
                    y.y = ex2_approx(y.y);
                }
                if (e & 2) acc2b = add2(acc2b, y);
                else acc2 = add2(acc2, y);
                pk[e / 2] = pack_bf16x2(y.x, y.y);
            }
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) pk[j] = 0u;
        }
        tmem_st16u(k.s_addr + cc * 16, pk);
    }
    const float2 tot = add2(acc2, acc2b);
    l += tot.x + tot.y;
}

// The whole CTA program.  RING: a chunk continuing a ring
// (swa_prefill_chunk), compiled as its own kernel so that the other calls
// keep 32-bit key positions, no ring branches and their four-map argument
// list (two more tensor-map arguments alone cost those launches 2%).
template <int D, bool RING, bool SINKS, bool VARLEN>
__device__ __forceinline__ void prefill_cta(const CUtensorMap *tmQ, const CUtensorMap *tmK, const CUtensorMap *tmV,
                                            const CUtensorMap *tmO, const CUtensorMap *tmKr, const CUtensorMap *tmVr,
                                            const TcPrefillArgs &a, const RingArgs &ring, const VarlenArgs &vl,
                                            const int n_mode1)
{
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + C::OFF_Q;   // Q_X at sQ + X * QTILE
    uint8_t *sK = smem + C::OFF_K;
    uint8_t *sV = smem + C::OFF_V;
    Bars *bars = reinterpret_cast<Bars *>(smem + C::OFF_BAR);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const Work w = make_work<RING, SINKS, VARLEN>(a, ring, vl, n_mode1);
    if constexpr (VARLEN) {
        if (!varlen_ok(vl, w.b, a.T) && threadIdx.x == 0) atomicMax(a.ctl.status, SWA_STATUS_BAD_INPUT);
    }
    // keys before the query (packed sequences: the sequence's own window)
    const int left = VARLEN ? varlen_left(vl, w.b, a.left) : a.left;
    // a packed-sequence unit past its sequence's end has nothing to do
    if (VARLEN && !w.q[0].active) return;
    const int tb = VARLEN ? 0 : w.b;         // batch coordinate of the tensors
    const int trow0 = VARLEN ? vl.cu[w.b] : 0; // row of query/key position 0
    WaitCtl ctl{&bars->abort, a.ctl.status, a.ctl.limit_ns};

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 2);   // one commit per MMA issuer
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 2);
        }
        for (int x = 0; x < 2; ++x) {
            for (int b = 0; b < 2; ++b) {
                mbar_init(&bars->s_full[x][b], 1);
                mbar_init(&bars->p_full[x][b], BM / 32);
                mbar_init(&bars->pv_done[x][b], 1);
            }
            mbar_init(&bars->epi[x], BM / 32);
            mbar_init(&bars->drain[x], 1);
        }
        mbar_init(&bars->a_first, 1);
        bars->abort = 0;
        fence_mbar_init();
    }
    if (warp == 8 && lane == 0) {
        prefetch_tensormap(tmQ);
        prefetch_tensormap(tmK);
        prefetch_tensormap(tmV);
        prefetch_tensormap(tmO);
    }
    if (warp == 9) tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    const int32_t *gb = a.gidx ? a.gidx + (long long)w.b * a.g : nullptr;

    // warpgroup 2 (producer, MMA issuers, idle warp 11) gives registers up
    if (warp >= 8) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(TC_REG_OTHER) : "memory");
    if (warp == 8) {
        // ------------------------------------------------------ producer --
        int kiss[NSTAGE] = {}, viss[NSTAGE] = {};
        bool ok = true;
        if (w.mode == 0) {
            if (lane == 0) {
                int nq = 0;
                for (int x = 0; x < 2; ++x) nq += w.q[x].active ? 1 : 0;
                mbar_expect_tx(&bars->q_full, nq * C::QTILE);
                for (int x = 0; x < 2; ++x)
                    if (w.q[x].active) {
                        SWA_DCHECK(w.q[x].m0 >= 0 && w.q[x].m0 < a.T && w.q[x].h < a.Hq, a.ctl.status);
                        for (int ch = 0; ch < C::NCH; ++ch)
                            tma_load_4d(sQ + x * C::QTILE + ch * C::QCH, tmQ, &bars->q_full, ch * C::E, w.q[x].h,
                                        w.q[x].m0 + trow0, tb);
                    }
            }
        } else {
            for (int x = 0; x < 2; ++x)
                if (w.q[x].active)
                    gather_tile<D>(sQ + x * C::QTILE, BM, C::QCH, static_cast<const __nv_bfloat16 *>(a.q),
                                   gb + w.q[x].gt * BM, w.q[x].nrows, w.b, a.T, a.Hq, w.q[x].h, lane, a.ctl.status);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->q_full);
        }
        if (RING && lane == 0 && ring.pos[w.b] < 0) atomicMax(a.ctl.status, SWA_STATUS_BAD_INPUT);
        if constexpr (RING) {
            const long long p0 = RING ? w.p0 : 0;
            // One K or V key tile into stage st: a TMA tile of the key tensor or
            // of the ring, or 16-byte cp.async row copies (global keys; ring rows
            // that wrap around the ring's end or meet the chunk's first row).
            auto load_tile = [&](bool is_v, int st, int t) {
                uint8_t *dst = (is_v ? sV : sK) + st * C::KTILE;
                uint64_t *bar = is_v ? &bars->v_full[st] : &bars->k_full[st];
                const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(is_v ? a.v : a.k);
                if (t >= w.n_band) {
                    const int gt = t - w.n_band;
                    gather_tile<D>(dst, BN, C::KCH, src, gb + gt * BN, min(BN, a.g - gt * BN), w.b, a.T, a.Hkv, w.hk,
                                   lane, a.ctl.status);
                } else {
                    const long long key0 = (long long)(w.j_lo + t) * BN;
                    const bool ring_tile = RING && key0 < w.p0;
                    const long long slot0 = ring_tile ? key0 % ring.W : 0;
                    if (!RING || !ring_tile || (key0 + BN <= w.p0 && slot0 + BN <= ring.W)) {
                        SWA_DCHECK(ring_tile ? (slot0 >= 0 && slot0 + BN <= ring.W)
                                             : (key0 >= p0 && key0 - p0 < a.T),
                                   a.ctl.status);
                        if (lane == 0) {
                            mbar_expect_tx(bar, C::KTILE);
                            for (int ch = 0; ch < C::NCH; ++ch) {
                                if (ring_tile)
                                    tma_load_4d(dst + ch * C::KCH, is_v ? tmVr : tmKr, bar, ch * C::E, (int)slot0, w.hk,
                                                w.b);
                                else
                                    tma_load_4d(dst + ch * C::KCH, is_v ? tmV : tmK, bar, ch * C::E, w.hk,
                                                (int)(key0 - p0), w.b);
                            }
                        }
                        return;
                    }
                    if (!RING) return;
                    const __nv_bfloat16 *rc = static_cast<const __nv_bfloat16 *>(is_v ? ring.vc : ring.kc);
                    gather_rows<D>(dst, BN, C::KCH, src, lane, [&](int r) -> const __nv_bfloat16 * {
                        const long long p = key0 + r;
                        if (p >= p0) {
                            const long long row = p - p0;
                            return row < a.T ? src + (((long long)w.b * a.T + row) * a.Hkv + w.hk) * D : nullptr;
                        }
                        return rc + (((long long)w.b * a.Hkv + w.hk) * ring.W + p % ring.W) * D;
                    });
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar);
            };
            for (int t = 0; t < w.n_tiles && ok; ++t) {
                const int st = t % NSTAGE;
                const uint32_t par = ((t / NSTAGE) & 1) ^ 1;
                ok = warp_wait_bounded(&bars->k_empty[st], par, ctl);
                if (!ok) break;
                load_tile(false, st, t);
                kiss[st]++;
                ok = warp_wait_bounded(&bars->v_empty[st], par, ctl);
                if (!ok) break;
                load_tile(true, st, t);
                viss[st]++;
            }
        } else {
            for (int t = 0; t < w.n_tiles && ok; ++t) {
                const bool band = t < w.n_band;
                const int key0 = (w.j_lo + t) * BN;
                const int gt = t - w.n_band;
                const int nr = band ? 0 : min(BN, a.g - gt * BN);
                const int st = t % NSTAGE;
                const uint32_t par = ((t / NSTAGE) & 1) ^ 1;
                ok = warp_wait_bounded(&bars->k_empty[st], par, ctl);
                if (!ok) break;
                if (band) {
                    SWA_DCHECK(key0 >= 0 && key0 < w.kend, a.ctl.status);
                    if (lane == 0) {
                        mbar_expect_tx(&bars->k_full[st], C::KTILE);
                        for (int ch = 0; ch < C::NCH; ++ch)
                            tma_load_4d(sK + st * C::KTILE + ch * C::KCH, tmK, &bars->k_full[st], ch * C::E, w.hk,
                                        key0 + trow0, tb);
                    }
                } else {
                    if constexpr (SINKS)
                        gather_sinks<D>(sK + st * C::KTILE, static_cast<const __nv_bfloat16 *>(a.k), gt * BN, nr, w.b,
                                        a.T, a.Hkv, w.hk, lane);
                    else
                        gather_tile<D>(sK + st * C::KTILE, BN, C::KCH, static_cast<const __nv_bfloat16 *>(a.k),
                                       gb + gt * BN, nr, w.b, a.T, a.Hkv, w.hk, lane, a.ctl.status);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->k_full[st]);
                }
                kiss[st]++;
                ok = warp_wait_bounded(&bars->v_empty[st], par, ctl);
                if (!ok) break;
                if (band) {
                    if (lane == 0) {
                        mbar_expect_tx(&bars->v_full[st], C::KTILE);
                        for (int ch = 0; ch < C::NCH; ++ch)
                            tma_load_4d(sV + st * C::KTILE + ch * C::KCH, tmV, &bars->v_full[st], ch * C::E, w.hk,
                                        key0 + trow0, tb);
                    }
                } else {
                    if constexpr (SINKS)
                        gather_sinks<D>(sV + st * C::KTILE, static_cast<const __nv_bfloat16 *>(a.v), gt * BN, nr, w.b,
                                        a.T, a.Hkv, w.hk, lane);
                    else
                        gather_tile<D>(sV + st * C::KTILE, BN, C::KCH, static_cast<const __nv_bfloat16 *>(a.v),
                                       gb + gt * BN, nr, w.b, a.T, a.Hkv, w.hk, lane, a.ctl.status);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->v_full[st]);
                }
                viss[st]++;
            }
        }
        if (!ok && lane == 0) {
            // let our own copies land before the CTA's shared memory goes away
            for (int s = 0; s < NSTAGE; ++s) {
                if (kiss[s] > 0) drain_wait(&bars->k_full[s], (kiss[s] - 1) & 1, a.ctl.limit_ns);
                if (viss[s] > 0) drain_wait(&bars->v_full[s], (viss[s] - 1) & 1, a.ctl.limit_ns);
            }
        }
    } else if (warp == 9 || warp == 10) {
        // ----------------------------------------------------------- MMA --
        // Warp 9 + x issues query tile x's MMAs.  The whole warp runs the
        // schedule (waits, descriptor arithmetic) in lock step, so operands
        // are warp-uniform; lane 0 alone issues MMAs and commits.  Both
        // issuers walk every key tile and commit the stage releases for each
        // (no MMAs when their tile does not use it), so each phase of the
        // two-arrival k_empty / v_empty barriers gets exactly one commit from
        // each, in order.
        const int x = warp - 9;
        constexpr uint32_t idesc_pv = umma_idesc_bf16(BM, D, 0, 1);
        // descriptors are built once; a k-step or stage only adds a constant
        // to the 14-bit start-address field (addresses < 2^18)
        const uint64_t dq = umma_smem_desc(smem_u32(sQ) + x * C::QTILE, 16, 8 * C::RB, C::LAYOUT);
        const uint64_t dk0 = umma_smem_desc(smem_u32(sK), 16, 8 * C::RB, C::LAYOUT);
        const uint64_t dv0 = umma_smem_desc(smem_u32(sV), C::KCH, 8 * C::RB, C::LAYOUT);
        const QTile q = x ? w.q[1] : w.q[0];
        const int n_band = w.n_band;
        const bool leader = lane == 0;
        bool ok = warp_wait_bounded(&bars->q_full, 0, ctl);
        // Tile B starts once tile A's first QK^T has completed: the two
        // tiles then run half a step apart, so one tile's MMAs tend to fill
        // the tensor core while the other waits for its softmax.
        const bool offset_b = w.q[0].active && tile_active(w.q[0], n_band, 0);
        if (ok && x == 1 && offset_b) ok = warp_wait_bounded(&bars->a_first, 0, ctl);
        auto pv_step = [&](int u) -> bool {
            const int st = u % NSTAGE;
            if (!warp_wait_bounded(&bars->v_full[st], (u / NSTAGE) & 1, ctl)) return false;
            if (tile_active(q, n_band, u)) {
                const int nk = tile_cols(w, a, u) / 16;
                const uint64_t dv = dv0 + (uint64_t)((st * C::KTILE) >> 4);
                const int c = tile_count(q, n_band, u), b = c & 1;
                if (!warp_wait_bounded(&bars->p_full[x][b], (c >> 1) & 1, ctl)) return false;
                tc_fence_after();
                const uint32_t d_o = tmem + col_o(x), a_p = tmem + col_s(x, b);
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk)
                        if (kk < nk)
                            mma_bf16_ts(d_o, a_p + kk * 8, dv + (uint64_t)((kk * 16 * C::RB) >> 4), idesc_pv,
                                        (c > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(&bars->pv_done[x][b]);
                }
            }
            if (leader) mma_commit(&bars->v_empty[st]);
            __syncwarp();
            return true;
        };
        for (int t = 0; t < w.n_tiles && ok; ++t) {
            const int st = t % NSTAGE;
            ok = warp_wait_bounded(&bars->k_full[st], (t / NSTAGE) & 1, ctl);
            if (!ok) break;
            if (tile_active(q, n_band, t)) {
                const int c = tile_count(q, n_band, t), b = c & 1;
                // S[x][b] holds P of this tile's predecessor in the buffer
                // until that PV completes
                if (c >= 2) ok = warp_wait_bounded(&bars->pv_done[x][b], ((c >> 1) - 1) & 1, ctl);
                if (!ok) break;
                tc_fence_after();
                const uint32_t idesc_qk = umma_idesc_bf16(BM, tile_cols(w, a, t), 0, 0);
                const uint64_t dk = dk0 + (uint64_t)((st * C::KTILE) >> 4);
                const uint32_t d_s = tmem + col_s(x, b);
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const int byte = kk * 32;
                        const uint64_t qo = (uint64_t)(((byte / C::RB) * C::QCH + (byte % C::RB)) >> 4);
                        const uint64_t ko = (uint64_t)(((byte / C::RB) * C::KCH + (byte % C::RB)) >> 4);
                        mma_bf16_ss(d_s, dq + qo, dk + ko, idesc_qk, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&bars->s_full[x][b]);
                    if (x == 0 && t == 0) mma_commit(&bars->a_first);
                }
            }
            if (leader) mma_commit(&bars->k_empty[st]);
            __syncwarp();
            if (t >= 1) ok = pv_step(t - 1);
        }
        if (ok && w.n_tiles > 0) ok = pv_step(w.n_tiles - 1);
        // all MMAs lane 0 issued are complete before TMEM is freed
        if (leader) {
            mma_commit(&bars->drain[x]);
            drain_wait(&bars->drain[x], 0, a.ctl.limit_ns);
        }
        __syncwarp();
    } else if (warp < 8) {
        // the softmax warpgroups take them
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(TC_REG_SOFTMAX) : "memory");
        // ------------------------------------------- softmax + epilogue --
        const int x = warp / 4;                 // query tile of this warpgroup
        const int quarter = warp % 4;
        const int r = quarter * 32 + lane;      // row in tile = TMEM lane
        const QTile qt = x ? w.q[1] : w.q[0];
        const int n_band = w.n_band;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        // key positions: 64-bit only for a chunk continuing a ring
        typedef typename std::conditional<RING, long long, int>::type kpos_t;
        const long long p0 = RING ? w.p0 : 0;
#define KEND ((RING || VARLEN) ? (kpos_t)w.kend : (kpos_t)a.T) // one past the last key
        long long i_row;                        // absolute query position
        if (w.mode == 0) i_row = p0 + qt.m0 + r;
        else i_row = (qt.active && r < qt.nrows) ? gb[qt.gt * BM + r] : 0;
        const long long i_out = i_row - p0;     // row in q / o / lse
        const bool row_real = qt.active && r < qt.nrows;
        const bool warp_has_rows = qt.active && quarter * 32 < qt.nrows;
        const long long wi0 = p0 + qt.m0 + quarter * 32, wi1 = wi0 + 31;
        float m = -CUDART_INF_F, l = 0.f;
        bool ok = true;
        for (int t = 0; t < w.n_tiles && qt.active; ++t) {
            if (!tile_active(qt, n_band, t)) continue;
            const int c = tile_count(qt, n_band, t), b = c & 1;
            ok = warp_wait_bounded(&bars->s_full[x][b], (c >> 1) & 1, ctl);
            if (!ok) break;
            tc_fence_after();

            // ---- which 32-key chunks can any row of this warp see ----
            const bool band = t < w.n_band;
            const kpos_t key0 = (kpos_t)(w.j_lo + t) * BN;
            int c_lo = 0, c_hi = -1;
            bool interior = false;
            if (warp_has_rows) {
                if (w.mode == 1) {
                    c_hi = (int)((min(key0 + BN - 1, KEND - 1) - key0) / 32);
                    interior = key0 + BN <= KEND;
                } else if (band) {
                    const long long lo = max(max((long long)key0, wi0 - left), 0LL);
                    const long long hi = min(min((long long)key0 + BN - 1, wi1 + a.right), (long long)KEND - 1);
                    if (lo <= hi) {
                        c_lo = (int)((lo - key0) / 32);
                        c_hi = (int)((hi - key0) / 32);
                    }
                    interior = (key0 + BN - 1 < KEND) && band_contains(wi1, key0, left, a.right) &&
                               band_contains(wi0, key0 + BN - 1, left, a.right);
                } else {
                    c_hi = (min(BN, a.g - (t - w.n_band) * BN) - 1) / 32;
                }
            }
            SWA_DCHECK(c_lo >= 0 && c_hi < BN / 32, a.ctl.status);
            // visible columns of this row as one int range (band, dense)
            TileCtx k;
            k.s_addr = tmem + lane_off + col_s(x, b);
            k.c_lo = c_lo;
            k.c_hi = c_hi;
            k.col_lo = 0;
            k.col_hi = BN - 1;
            k.by_range = (w.mode == 1) || band;
            if (w.mode == 1) {
                k.col_hi = (int)min((kpos_t)BN - 1, KEND - 1 - key0);
            } else if (band) {
                k.col_lo = (int)max(i_row - left - key0, 0LL);
                k.col_hi = (int)min(min(i_row + a.right, (long long)KEND - 1) - key0, (long long)BN - 1);
            }
            k.gc_base = (t - w.n_band) * BN;
            k.i_row = i_row;
            bool rescale_o;
            float alpha;
            if (interior && c_lo == 0 && c_hi == BN / 32 - 1)
                softmax_tile<true, SINKS>(k, a, gb, m, l, rescale_o, alpha, c == 0);
            else
                softmax_tile<false, SINKS>(k, a, gb, m, l, rescale_o, alpha, c == 0);

            // O rescale (rare): wait for the previous tile's PV, which
            // accumulates into O; this tile's PV waits for P
            if (__any_sync(0xffffffffu, rescale_o)) {
                const int cp = c - 1, bp = cp & 1;
                ok = warp_wait_bounded(&bars->pv_done[x][bp], (cp >> 1) & 1, ctl);
                if (!ok) break;
                tc_fence_after();
                const float f = rescale_o ? alpha : 1.f;
#pragma unroll 1
                for (int cc = 0; cc < D / 16; ++cc) {
                    float ov[16];
                    tmem_ld16(tmem + lane_off + col_o(x) + cc * 16, ov);
                    tmem_ld_wait_dep16(ov);
                    uint32_t ou[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) ou[e] = __float_as_uint(ov[e] * f);
                    tmem_st16u(tmem + lane_off + col_o(x) + cc * 16, ou);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->p_full[x][b]);
        }

        // ---- epilogue ----
        const int nx = tiles_of(qt, w.n_glob);
        if (ok && nx > 0) {
            const int cl = nx - 1;
            ok = warp_wait_bounded(&bars->pv_done[x][cl & 1], (cl >> 1) & 1, ctl);
        }
        // rows written one by one: dense global rows, band rows next to global
        // ones, and the last tile of a packed sequence (a tile store would
        // run into the next sequence)
        const bool direct = (w.mode == 1) || (a.gidx != nullptr && a.g > 0) || (VARLEN && qt.nrows < BM);
        uint8_t *stage = sQ + x * C::QTILE;
        if (ok && qt.active) {
            tc_fence_after();
            const float inv = (l > 0.f) ? 1.f / l : 0.f;
            __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(a.o);
            bool skip_row = !row_real;
            if (!VARLEN && w.mode == 0 && direct && row_real) {
                // rows of global tokens are written by the dense-row CTAs
                int lo = 0, hi = a.g;
                while (lo < hi) {
                    const int mid = (lo + hi) >> 1;
                    if (gb[mid] < i_row) lo = mid + 1;
                    else hi = mid;
                }
                skip_row = (lo < a.g && gb[lo] == i_row);
            }
#pragma unroll 1
            for (int cc = 0; cc < D / 16; ++cc) {
                float ov[16];
                tmem_ld16(tmem + lane_off + col_o(x) + cc * 16, ov);
                tmem_ld_wait_dep16(ov);
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    uint4 pk;
                    pk.x = pack_bf16x2(ov[u * 8 + 0] * inv, ov[u * 8 + 1] * inv);
                    pk.y = pack_bf16x2(ov[u * 8 + 2] * inv, ov[u * 8 + 3] * inv);
                    pk.z = pack_bf16x2(ov[u * 8 + 4] * inv, ov[u * 8 + 5] * inv);
                    pk.w = pack_bf16x2(ov[u * 8 + 6] * inv, ov[u * 8 + 7] * inv);
                    const int e = cc * 16 + u * 8;
                    if (direct) {
                        if (!skip_row) {
                            SWA_DCHECK(trow0 + i_out >= 0 && trow0 + i_out < a.T, a.ctl.status);
                            __nv_bfloat16 *dst = o + (((long long)tb * a.T + trow0 + i_out) * a.Hq + qt.h) * D + e;
                            *reinterpret_cast<uint4 *>(dst) = pk;
                        }
                    } else {
                        *reinterpret_cast<uint4 *>(stage + tile_offset<D>(r, e, C::QCH)) = pk;
                    }
                }
            }
            if (a.lse && row_real && !skip_row)
                a.lse[((long long)tb * a.Hq + qt.h) * a.T + trow0 + i_out] =
                    (l > 0.f) ? (m + __log2f(l)) * 0.69314718055994530942f : -CUDART_INF_F;
        }
        // staging tile complete -> one thread per warpgroup stores it
        // (bounded; an abort anywhere in the CTA skips the store)
        if (!direct && qt.active) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->epi[x]);
            if (r == 0 && wait_bounded(&bars->epi[x], 0, ctl) && !bars->abort) {
                for (int ch = 0; ch < C::NCH; ++ch)
                    tma_store_4d(tmO, stage + ch * C::QCH, ch * C::E, qt.h, qt.m0 + trow0, tb);
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

template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    swa_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                          const TcPrefillArgs a, const int n_mode1)
{
    prefill_cta<D, false, false, false>(&tmQ, &tmK, &tmV, &tmO, nullptr, nullptr, a, RingArgs{}, VarlenArgs{}, n_mode1);
}

// Causal window plus attention sinks (a.gidx null, a.g sinks): the sink keys
// form the gathered key tiles.
template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    swa_prefill_sinks_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                             const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                             const TcPrefillArgs a, const int n_mode1)
{
    prefill_cta<D, false, true, false>(&tmQ, &tmK, &tmV, &tmO, nullptr, nullptr, a, RingArgs{}, VarlenArgs{}, n_mode1);
}

// Packed variable-length sequences: [total,H,d] tensors, sequence b in rows
// cu[b] .. cu[b+1]-1.
template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    swa_prefill_varlen_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                              const TcPrefillArgs a, const VarlenArgs vl, const int n_mode1)
{
    prefill_cta<D, false, false, true>(&tmQ, &tmK, &tmV, &tmO, nullptr, nullptr, a, RingArgs{}, vl, n_mode1);
}

template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    swa_prefill_ring_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                            const __grid_constant__ CUtensorMap tmKr, const __grid_constant__ CUtensorMap tmVr,
                            const TcPrefillArgs a, const RingArgs ring, const int n_mode1)
{
    prefill_cta<D, true, false, false>(&tmQ, &tmK, &tmV, &tmO, &tmKr, &tmVr, a, ring, VarlenArgs{}, n_mode1);
}

// ------------------------------------------------------------------ host --

// [B,T,H,D] bf16 viewed as a 4-D tensor (D, H, T, B); box = one chunk of
// `rows` rows of one head.
template <int D>
bool make_map(CUtensorMap *m, const void *ptr, int B, int T, int H, int rows)
{
    return make_bthd_map(m, ptr, B, T, H, D, rows);
}

// Ring cache [B,Hkv,W,D] bf16 viewed as (D, W, Hkv, B); box = one chunk of
// BN consecutive slots of one kv head.
template <int D>
bool make_ring_map(CUtensorMap *m, const void *ptr, int B, int Hkv, int W)
{
    using C = Cfg<D>;
    EncodeTiledFn enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)W, (cuuint64_t)Hkv, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)W * D * 2, (cuuint64_t)Hkv * W * D * 2};
    cuuint32_t box[4] = {(cuuint32_t)C::E, (cuuint32_t)BN, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE,
                     C::RB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int D, bool RING>
cudaError_t launch_dr(int mode, const TcPrefillArgs &a, const RingArgs &ring, cudaStream_t s)
{
    using C = Cfg<D>;
    CUtensorMap mq, mk, mv, mo, mkr, mvr;
    if (!make_map<D>(&mq, a.q, a.B, a.T, a.Hq, BM) || !make_map<D>(&mk, a.k, a.B, a.T, a.Hkv, BN) ||
        !make_map<D>(&mv, a.v, a.B, a.T, a.Hkv, BN) || !make_map<D>(&mo, a.o, a.B, a.T, a.Hq, BM))
        return cudaErrorInvalidValue;
    if (RING) {
        if (!make_ring_map<D>(&mkr, ring.kc, a.B, a.Hkv, ring.W) || !make_ring_map<D>(&mvr, ring.vc, a.B, a.Hkv, ring.W))
            return cudaErrorInvalidValue;
    } else {
        mkr = mk; // unused without a ring
        mvr = mv;
    }
    // sinks: no global positions but g > 0 (causal window plus the first g
    // positions)
    const bool sinks = !RING && a.gidx == nullptr && a.g > 0;
    static DeviceOnce once[2];
    cudaError_t e = once[sinks].get(
        [&](int) {
            return RING    ? cudaFuncSetAttribute(swa_prefill_ring_kernel<D>,
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES)
                   : sinks ? cudaFuncSetAttribute(swa_prefill_sinks_kernel<D>,
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES)
                           : cudaFuncSetAttribute(swa_prefill_tc_kernel<D>,
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        },
        nullptr);
    if (e != cudaSuccess) return e;
    const int G = a.Hq / a.Hkv;
    const bool pair_heads = (G % 2) == 0;
    const int nqt = (a.T + BM - 1) / BM;
    const int ngt = (a.g + BM - 1) / BM;
    const bool globals = a.gidx != nullptr && a.g > 0;
    // CTAs: pairs of heads (even group size) or pairs of row tiles / global
    // row groups of one head
    const int units_q = pair_heads ? (a.Hq / 2) * nqt : a.Hq * ((nqt + 1) / 2);
    const int units_g = pair_heads ? (a.Hq / 2) * ngt : a.Hq * ((ngt + 1) / 2);
    int n_mode1 = 0, n_mode0 = 0;
    if (mode == 0) {
        n_mode0 = a.B * units_q;
        if (globals) n_mode1 = a.B * units_g;
    } else {
        n_mode1 = a.B * units_g;
    }
    const int grid = n_mode0 + n_mode1;
    if (grid == 0) return cudaSuccess;
    {
        const void *kfn = RING ? (const void *)swa_prefill_ring_kernel<D>
                          : sinks ? (const void *)swa_prefill_sinks_kernel<D> : (const void *)swa_prefill_tc_kernel<D>;
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, kfn) != cudaSuccess ||
            fa.numRegs * NTHREADS < 256 * TC_REG_SOFTMAX + 128 * TC_REG_OTHER)
            return cudaErrorInvalidConfiguration;
    }
    if (RING)
        swa_prefill_ring_kernel<D><<<grid, NTHREADS, C::SMEM_BYTES, s>>>(mq, mk, mv, mo, mkr, mvr, a, ring, n_mode1);
    else if (sinks)
        swa_prefill_sinks_kernel<D><<<grid, NTHREADS, C::SMEM_BYTES, s>>>(mq, mk, mv, mo, a, n_mode1);
    else
        swa_prefill_tc_kernel<D><<<grid, NTHREADS, C::SMEM_BYTES, s>>>(mq, mk, mv, mo, a, n_mode1);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_varlen_d(const TcPrefillArgs &a, const VarlenArgs &vl, cudaStream_t s)
{
    using C = Cfg<D>;
    // the packed tensors as one sequence of `total` rows
    CUtensorMap mq, mk, mv, mo;
    if (!make_map<D>(&mq, a.q, 1, a.T, a.Hq, BM) || !make_map<D>(&mk, a.k, 1, a.T, a.Hkv, BN) ||
        !make_map<D>(&mv, a.v, 1, a.T, a.Hkv, BN) || !make_map<D>(&mo, a.o, 1, a.T, a.Hq, BM))
        return cudaErrorInvalidValue;
    static DeviceOnce once;
    cudaError_t e = once.get(
        [&](int) {
            return cudaFuncSetAttribute(swa_prefill_varlen_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        C::SMEM_BYTES);
        },
        nullptr);
    if (e != cudaSuccess) return e;
    const int G = a.Hq / a.Hkv;
    const bool pair_heads = (G % 2) == 0;
    const int nqt = (vl.max_len + BM - 1) / BM;
    // units over (sequence, query tile [pair], head [pair]); those past a
    // sequence's end return at once
    const long long units = (long long)a.B * (pair_heads ? (a.Hq / 2) * nqt : a.Hq * ((nqt + 1) / 2));
    if (units == 0) return cudaSuccess;
    if (units > 0x7fffffffLL) return cudaErrorInvalidValue;
    {
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, (const void *)swa_prefill_varlen_kernel<D>) != cudaSuccess ||
            fa.numRegs * NTHREADS < 256 * TC_REG_SOFTMAX + 128 * TC_REG_OTHER)
            return cudaErrorInvalidConfiguration;
    }
    swa_prefill_varlen_kernel<D><<<(int)units, NTHREADS, C::SMEM_BYTES, s>>>(mq, mk, mv, mo, a, vl, 0);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(int mode, const TcPrefillArgs &a, const RingArgs &ring, cudaStream_t s)
{
    return ring.pos ? launch_dr<D, true>(mode, a, ring, s) : launch_dr<D, false>(mode, a, ring, s);
}

}  // namespace

cudaError_t launch_prefill_varlen(int d, const TcPrefillArgs &a, const VarlenArgs &vl, cudaStream_t s)
{
    if (prefill_pp_varlen_applies(d, a, vl)) return launch_prefill_pp_varlen(d, a, vl, s);
    switch (d) {
    case 32: return launch_varlen_d<32>(a, vl, s);
    case 64: return launch_varlen_d<64>(a, vl, s);
    case 128: return launch_varlen_d<128>(a, vl, s);
    default: return cudaErrorInvalidValue;
    }
}

// mode 0: band tiles (+ dense global-row CTAs first in the same grid when
// global tokens are present), or the narrow-window kernel; mode 1: dense
// global rows only.
cudaError_t launch_prefill_tc(int d, int mode, const TcPrefillArgs &a, const RingArgs &ring, cudaStream_t s)
{
    // a causal window of at most 64 keys: the single-pass kernel; windows of
    // 256 keys or more without global keys (a chunk over a ring included):
    // the 128-key kernel
    if (mode == 0 && ring.pos == nullptr && prefill_narrow_applies(d, a)) return launch_prefill_narrow(d, a, s);
    if (mode == 0 && prefill_pp_applies(d, a)) return launch_prefill_pp(d, a, ring, s);

    switch (d) {
    case 32: return launch_d<32>(mode, a, ring, s);
    case 64: return launch_d<64>(mode, a, ring, s);
    case 128: return launch_d<128>(mode, a, ring, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace swa
