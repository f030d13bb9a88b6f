// Sliding-window prefill on tcgen05 tensor cores (sm_100a).
//
// What it computes (the pages' definition): for query row i, softmax over the
// keys of its window of scale*q.k, logits outside the window being -inf, then
// the weighted sum of value rows ("Sliding Window Attention", robocikowo.com,
// opening definition).  The [T,T] score matrix never exists: each CTA owns
// one 128-row query tile and streams only the 128-key tiles that intersect
// the tile's window, skipping every tile that lies fully outside it (the
// fused-kernel point of the same page and of the Ultralytics glossary's
// FlashAttention entry).  Work per query tile is O(W*d), total O(T*W*d).
//
// CTA anatomy (192 threads):
//   warps 0-3  softmax + epilogue: thread r owns query row r of the tile,
//              which is TMEM lane r (warp w may only touch lanes 32w..32w+31)
//   warp 4     producer: TMA tile loads of Q, K, V (no multicast), or plain
//              gathers for global keys / global query rows
//   warp 5     TMEM allocator; lane 0 issues every tcgen05.mma
// Per key tile t:
//   S[t&1] = Q K_t^T          (TMEM, fp32, 128 x 128), double buffered so the
//                             MMA of tile t+1 overlaps the softmax of tile t
//   softmax: S -> registers (tcgen05.ld), mask (edge tiles only), running
//            row max in log2 units, P = 2^(S*scale*log2e - m) -> bf16 -> SMEM
//            (128B-swizzled, K-major, the UMMA A-operand layout)
//   O += P V_t                (TMEM, fp32, 128 x d)
// The running max is only raised when a tile's max exceeds it by more than
// 2^8; P then stays <= 256 and O, l share one reference, so the final O/l is
// exact; raising it rescales l and the O row in TMEM.
//
// Every mbarrier wait is bounded (wait_bounded): on expiry the CTA records
// SWA_STATUS_TIMEOUT, drains its own in-flight copies and MMAs with a second
// bound, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math_constants.h>

#include "ptx.cuh"
#include "swa_internal.h"

namespace swa {
namespace {

constexpr int BM = 128;              // query rows per tile (= TMEM lanes)
constexpr int BN = 128;              // keys per key tile
constexpr int NSTAGE = 2;            // K/V pipeline depth
constexpr int NTHREADS = 192;
constexpr float RESCALE_LOG2 = 8.0f; // raise the running max only beyond 2^8

template <int D>
struct Cfg {
    static constexpr int RB = (D * 2 >= 128) ? 128 : D * 2; // bytes per swizzled row
    static constexpr int E = RB / 2;                         // elements per chunk row
    static constexpr int NCH = D / E;                        // chunks per head row
    static constexpr int CH_BYTES = 128 * RB;                // one chunk of a 128-row tile
    static constexpr int TILE = 128 * D * 2;                 // a 128-row tile of Q, K, V or O
    static constexpr uint32_t LAYOUT = (RB == 128) ? UMMA_SW128 : UMMA_SW64;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + TILE;
    static constexpr int OFF_V = OFF_K + NSTAGE * TILE;
    static constexpr int OFF_P = OFF_V + NSTAGE * TILE;
    static constexpr int OFF_BAR = OFF_P + BM * BN * 2;
    // + room to align the base to 1 KiB; at least 120 KiB so that a second CTA
    // never shares the SM (each CTA takes all 512 TMEM columns)
    static constexpr int SMEM_NEED = OFF_BAR + 256 + 1024;
    static constexpr int SMEM_BYTES = SMEM_NEED > 120 * 1024 ? SMEM_NEED : 120 * 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_S = 0;                     // S buffers at columns 0 and 128
    static constexpr uint32_t COL_O = 256;                   // O accumulator, D columns
    static_assert(D == 32 || D == 64 || D == 128, "head dim");
    static_assert(SMEM_NEED <= 227 * 1024, "shared memory");
};

// Byte offset of element e of row r inside a swizzled [128 rows][D] tile
// (the layout a TMA SWIZZLE_128B / SWIZZLE_64B load produces).
template <int D>
__device__ __forceinline__ uint32_t tile_offset(int r, int e)
{
    using C = Cfg<D>;
    const int ch = e / C::E;
    const int u = (e % C::E) / 8;
    const int phys = (C::RB == 128) ? (u ^ (r & 7)) : (u ^ ((r >> 1) & 3));
    return ch * C::CH_BYTES + r * C::RB + phys * 16;
}

struct Bars {
    uint64_t q_full;
    uint64_t k_full[NSTAGE];
    uint64_t v_full[NSTAGE];
    uint64_t k_empty[NSTAGE];
    uint64_t v_empty[NSTAGE];
    uint64_t s_full[2];
    uint64_t p_full;
    uint64_t pv_done;
    uint64_t drain;
    uint64_t epi;
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

// The per-CTA work description every role derives identically.
struct Work {
    int mode;      // 0 band tile, 1 dense global rows
    int b, h, hk;
    int m0;        // first query row (mode 0)
    int gt;        // global-row group (mode 1)
    int nrows;     // real rows in the tile (mode 1)
    int j_lo;      // first key tile
    int n_band;    // key tiles streamed by TMA
    int n_glob;    // gathered tiles of global keys (mode 0 with globals)
    int n_tiles;
};

__device__ __forceinline__ Work make_work(const TcPrefillArgs &a, int n_mode1)
{
    Work w;
    const int nqt = (a.T + BM - 1) / BM;
    const int nkt = (a.T + BN - 1) / BN;
    int bid = blockIdx.x;
    if (bid < n_mode1) {
        const int ngt = (a.g + BM - 1) / BM;
        w.mode = 1;
        w.h = bid % a.Hq;
        w.gt = (bid / a.Hq) % ngt;
        w.b = bid / (a.Hq * ngt);
        w.m0 = 0;
        w.nrows = min(BM, a.g - w.gt * BM);
        w.j_lo = 0;
        w.n_band = nkt;
        w.n_glob = 0;
    } else {
        bid -= n_mode1;
        w.mode = 0;
        w.h = bid % a.Hq;
        const int qt = (bid / a.Hq) % nqt;
        w.b = bid / (a.Hq * nqt);
        w.m0 = qt * BM;
        w.gt = 0;
        w.nrows = min(BM, a.T - w.m0);
        const int lo_key = max(0, w.m0 - a.left);
        const int hi_key = min(a.T - 1, w.m0 + BM - 1 + a.right);
        w.j_lo = lo_key / BN;
        w.n_band = hi_key / BN - w.j_lo + 1;
        w.n_glob = (a.gidx != nullptr && a.g > 0) ? (a.g + BN - 1) / BN : 0;
    }
    w.hk = w.h / (a.Hq / a.Hkv);
    w.n_tiles = w.n_band + w.n_glob;
    return w;
}

// Producer-warp gather of up to 128 rows (positions from `rows_idx`) of one
// head into a swizzled tile; rows past `nrows` are zero.  All 32 lanes.
template <int D>
__device__ __forceinline__ void gather_tile(uint8_t *dst, const __nv_bfloat16 *base, const int32_t *rows_idx,
                                            int nrows, int b, int T, int H, int head, int lane)
{
    constexpr int GR = D / 8; // 16-byte granules per row
    for (int idx = lane; idx < 128 * GR; idx += 32) {
        const int r = idx / GR, u = idx % GR;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (r < nrows) {
            const long long pos = rows_idx[r];
            const __nv_bfloat16 *src = base + (((long long)b * T + pos) * H + head) * D + u * 8;
            val = __ldg(reinterpret_cast<const uint4 *>(src));
        }
        *reinterpret_cast<uint4 *>(dst + tile_offset<D>(r, u * 8)) = val;
    }
}

template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    swa_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                          const TcPrefillArgs a, const int n_mode1)
{
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + C::OFF_Q;
    uint8_t *sK = smem + C::OFF_K;
    uint8_t *sV = smem + C::OFF_V;
    uint8_t *sP = smem + C::OFF_P;
    Bars *bars = reinterpret_cast<Bars *>(smem + C::OFF_BAR);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const Work w = make_work(a, n_mode1);
    WaitCtl ctl{&bars->abort, a.ctl.status, a.ctl.limit_ns};

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
            mbar_init(&bars->v_empty[s], 1);
        }
        mbar_init(&bars->s_full[0], 1);
        mbar_init(&bars->s_full[1], 1);
        mbar_init(&bars->p_full, BM / 32);
        mbar_init(&bars->pv_done, 1);
        mbar_init(&bars->drain, 1);
        mbar_init(&bars->epi, BM / 32);
        bars->abort = 0;
        fence_mbar_init();
    }
    if (warp == 4 && lane == 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        prefetch_tensormap(&tmO);
    }
    if (warp == 5) tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    const int32_t *gb = a.gidx ? a.gidx + (long long)w.b * a.g : nullptr;

    if (warp == 4) {
        // ------------------------------------------------------ producer --
        int issued[NSTAGE] = {0, 0}, vissued[NSTAGE] = {0, 0};
        bool ok = true;
        if (w.mode == 0) {
            if (lane == 0) {
                mbar_expect_tx(&bars->q_full, C::TILE);
                for (int ch = 0; ch < C::NCH; ++ch)
                    tma_load_4d(sQ + ch * C::CH_BYTES, &tmQ, &bars->q_full, ch * C::E, w.h, w.m0, w.b);
            }
        } else {
            gather_tile<D>(sQ, static_cast<const __nv_bfloat16 *>(a.q), gb + w.gt * BM, w.nrows, w.b, a.T, a.Hq,
                           w.h, lane);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->q_full);
        }
        for (int t = 0; t < w.n_tiles && ok; ++t) {
            const int st = t % NSTAGE;
            const uint32_t ph = (t / NSTAGE) & 1;
            ok = warp_wait_bounded(&bars->k_empty[st], ph ^ 1, ctl);
            if (!ok) break;
            if (t < w.n_band) {
                const int key0 = (w.j_lo + t) * BN;
                if (lane == 0) {
                    mbar_expect_tx(&bars->k_full[st], C::TILE);
                    for (int ch = 0; ch < C::NCH; ++ch)
                        tma_load_4d(sK + st * C::TILE + ch * C::CH_BYTES, &tmK, &bars->k_full[st], ch * C::E, w.hk,
                                    key0, w.b);
                }
                issued[st]++;
                ok = warp_wait_bounded(&bars->v_empty[st], ph ^ 1, ctl);
                if (!ok) break;
                if (lane == 0) {
                    mbar_expect_tx(&bars->v_full[st], C::TILE);
                    for (int ch = 0; ch < C::NCH; ++ch)
                        tma_load_4d(sV + st * C::TILE + ch * C::CH_BYTES, &tmV, &bars->v_full[st], ch * C::E, w.hk,
                                    key0, w.b);
                }
            } else {
                const int gt = t - w.n_band;
                const int nr = min(BN, a.g - gt * BN);
                ok = warp_wait_bounded(&bars->v_empty[st], ph ^ 1, ctl);
                if (!ok) break;
                issued[st]++;
                gather_tile<D>(sK + st * C::TILE, static_cast<const __nv_bfloat16 *>(a.k), gb + gt * BN, nr, w.b,
                               a.T, a.Hkv, w.hk, lane);
                gather_tile<D>(sV + st * C::TILE, static_cast<const __nv_bfloat16 *>(a.v), gb + gt * BN, nr, w.b,
                               a.T, a.Hkv, w.hk, lane);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&bars->k_full[st]);
                    mbar_arrive(&bars->v_full[st]);
                }
            }
            vissued[st]++;
        }
        if (!ok && lane == 0) {
            // let our own copies land before the CTA's shared memory goes away
            for (int s = 0; s < NSTAGE; ++s)
            {
                if (issued[s] > 0) drain_wait(&bars->k_full[s], (issued[s] - 1) & 1, a.ctl.limit_ns);
                if (vissued[s] > 0) drain_wait(&bars->v_full[s], (vissued[s] - 1) & 1, a.ctl.limit_ns);
            }
        }
    } else if (warp == 5) {
        // ----------------------------------------------------------- MMA --
        if (lane == 0) {
            constexpr uint32_t idesc_qk = umma_idesc_bf16(BM, BN, 0, 0);
            constexpr uint32_t idesc_pv = umma_idesc_bf16(BM, D, 0, 1);
            const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK), v_base = smem_u32(sV);
            const uint32_t p_base = smem_u32(sP);
            bool ok = wait_bounded(&bars->q_full, 0, ctl);
            tc_fence_after();
            auto issue_pv = [&](int u) -> bool {
                const int st = u % NSTAGE;
                if (!wait_bounded(&bars->v_full[st], (u / NSTAGE) & 1, ctl)) return false;
                if (!wait_bounded(&bars->p_full, u & 1, ctl)) return false;
                tc_fence_after();
                const uint32_t vb = v_base + st * C::TILE;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint64_t da = umma_smem_desc(p_base + (kk / 4) * (BM * 128) + (kk % 4) * 32, 16, 1024,
                                                       UMMA_SW128);
                    const uint64_t db = umma_smem_desc(vb + kk * 16 * C::RB, C::CH_BYTES, 8 * C::RB, C::LAYOUT);
                    mma_bf16_ss(tmem + C::COL_O, da, db, idesc_pv, (u > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&bars->v_empty[st]);
                mma_commit(&bars->pv_done);
                return true;
            };
            for (int t = 0; t < w.n_tiles && ok; ++t) {
                const int st = t % NSTAGE;
                ok = wait_bounded(&bars->k_full[st], (t / NSTAGE) & 1, ctl);
                if (!ok) break;
                tc_fence_after();
                const uint32_t kb = k_base + st * C::TILE;
                const uint32_t d_s = tmem + C::COL_S + (t & 1) * BN;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int byte = kk * 32;
                    const uint32_t off = (byte / C::RB) * C::CH_BYTES + (byte % C::RB);
                    const uint64_t da = umma_smem_desc(q_base + off, 16, 8 * C::RB, C::LAYOUT);
                    const uint64_t db = umma_smem_desc(kb + off, 16, 8 * C::RB, C::LAYOUT);
                    mma_bf16_ss(d_s, da, db, idesc_qk, kk > 0 ? 1u : 0u);
                }
                mma_commit(&bars->s_full[t & 1]);
                mma_commit(&bars->k_empty[st]);
                if (t >= 1) ok = issue_pv(t - 1);
            }
            if (ok && w.n_tiles > 0) ok = issue_pv(w.n_tiles - 1);
            // all MMAs this thread issued are complete before TMEM is freed
            mma_commit(&bars->drain);
            drain_wait(&bars->drain, 0, a.ctl.limit_ns);
        }
        __syncwarp();
    } else {
        // ------------------------------------------- softmax + epilogue --
        const int r = threadIdx.x;              // row in tile = TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        long long i_row;                        // absolute query position
        if (w.mode == 0) i_row = w.m0 + r;
        else i_row = (r < w.nrows) ? gb[w.gt * BM + r] : 0;
        const bool row_real = r < w.nrows;
        float m = -CUDART_INF_F, l = 0.f;
        bool ok = true;
        float s[BN];
        for (int t = 0; t < w.n_tiles; ++t) {
            ok = warp_wait_bounded(&bars->s_full[t & 1], (t / 2) & 1, ctl);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) tmem_ld32(lane_base + C::COL_S + (t & 1) * BN + c * 32, s + c * 32);
            tmem_ld_wait();

            // ---- mask (edge tiles only) ----
            if (w.mode == 1) {
                const int key0 = t * BN;
                if (key0 + BN > a.T) {
#pragma unroll
                    for (int c = 0; c < BN; ++c)
                        if (key0 + c >= a.T) s[c] = -CUDART_INF_F;
                }
            } else if (t < w.n_band) {
                const int key0 = (w.j_lo + t) * BN;
                const bool interior = (key0 + BN - 1 < a.T) && band_contains(w.m0 + BM - 1, key0, a.left, a.right) &&
                                      band_contains(w.m0, key0 + BN - 1, a.left, a.right);
                if (!interior) {
#pragma unroll
                    for (int c = 0; c < BN; ++c) {
                        const long long key = key0 + c;
                        if (!(key < a.T && band_contains(i_row, key, a.left, a.right))) s[c] = -CUDART_INF_F;
                    }
                }
            } else {
                // gathered global keys: only those outside this row's band
                const int c0 = (t - w.n_band) * BN;
#pragma unroll
                for (int c = 0; c < BN; ++c) {
                    const int gc = c0 + c;
                    bool keep = false;
                    if (gc < a.g) keep = !band_contains(i_row, __ldg(gb + gc), a.left, a.right);
                    if (!keep) s[c] = -CUDART_INF_F;
                }
            }

            // ---- online softmax (log2 domain, lazy rescale) ----
            // row max: 8 independent 3-input max chains, then a short tree
            float mx8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) mx8[j] = fmax3(s[j], s[8 + j], s[16 + j]);
#pragma unroll
            for (int c = 24; c + 16 <= BN; c += 16)
#pragma unroll
                for (int j = 0; j < 8; ++j) mx8[j] = fmax3(mx8[j], s[c + j], s[c + 8 + j]);
#pragma unroll
            for (int c = 24 + ((BN - 24) / 16) * 16; c < BN; c += 8)
#pragma unroll
                for (int j = 0; j < 8; ++j) mx8[j] = fmaxf(mx8[j], s[c + j]);
            const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                                   fmaxf(mx8[6], mx8[7]));
            const float mt = mx * a.scale_log2;
            bool rescale_o = false;
            float alpha = 1.f;
            if (mt > m + RESCALE_LOG2) {
                alpha = ex2_approx(m - mt);     // 0 when m was -inf
                l *= alpha;
                rescale_o = (t > 0);
                m = mt;
            }
            const float m_use = (m == -CUDART_INF_F) ? 0.f : m;
            // exponent arguments two at a time (fma.f32x2), four partial sums
            const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
            const float2 nm2 = make_float2(-m_use, -m_use);
            float2 rs2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                             make_float2(0.f, 0.f)};
#pragma unroll
            for (int c = 0; c < BN; c += 2) {
                float2 x = fma2(make_float2(s[c], s[c + 1]), sc2, nm2);
                s[c] = ex2_approx(x.x);
                s[c + 1] = ex2_approx(x.y);
                rs2[(c / 2) & 3] = add2(rs2[(c / 2) & 3], make_float2(s[c], s[c + 1]));
            }
            const float2 r01 = add2(rs2[0], rs2[1]), r23 = add2(rs2[2], rs2[3]);
            const float2 rsum = add2(r01, r23);
            l += rsum.x + rsum.y;

            // PV of the previous tile must be done: it reads the P buffer and
            // writes O, which a rescale touches
            if (t > 0) {
                ok = warp_wait_bounded(&bars->pv_done, (t - 1) & 1, ctl);
                if (!ok) break;
                tc_fence_after();
            }
            if (__any_sync(0xffffffffu, rescale_o)) {
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    float ov[32];
                    tmem_ld32(lane_base + C::COL_O + c * 32, ov);
                    tmem_ld_wait();
                    const float f = rescale_o ? alpha : 1.f;
#pragma unroll
                    for (int e = 0; e < 32; ++e) ov[e] *= f;
                    tmem_st32(lane_base + C::COL_O + c * 32, ov);
                }
                tmem_st_wait();
            }
            // P (bf16) into the swizzled K-major A-operand tile
#pragma unroll
            for (int u = 0; u < BN / 8; ++u) {
                uint4 pk;
                pk.x = pack_bf16x2(s[u * 8 + 0], s[u * 8 + 1]);
                pk.y = pack_bf16x2(s[u * 8 + 2], s[u * 8 + 3]);
                pk.z = pack_bf16x2(s[u * 8 + 4], s[u * 8 + 5]);
                pk.w = pack_bf16x2(s[u * 8 + 6], s[u * 8 + 7]);
                const int kc = u / 8, g16 = u % 8;
                *reinterpret_cast<uint4 *>(sP + kc * (BM * 128) + r * 128 + ((g16 ^ (r & 7)) << 4)) = pk;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->p_full);
        }

        // ---- epilogue ----
        if (ok && w.n_tiles > 0) ok = warp_wait_bounded(&bars->pv_done, (w.n_tiles - 1) & 1, ctl);
        if (ok) {
            tc_fence_after();
            const float inv = (l > 0.f) ? 1.f / l : 0.f;
            const bool direct = (w.mode == 1) || (a.gidx != nullptr && a.g > 0);
            __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(a.o);
            bool skip_row = !row_real;
            if (w.mode == 0 && direct && row_real) {
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
            for (int c = 0; c < D / 32; ++c) {
                float ov[32];
                tmem_ld32(lane_base + C::COL_O + c * 32, ov);
                tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    uint4 pk;
                    pk.x = pack_bf16x2(ov[u * 8 + 0] * inv, ov[u * 8 + 1] * inv);
                    pk.y = pack_bf16x2(ov[u * 8 + 2] * inv, ov[u * 8 + 3] * inv);
                    pk.z = pack_bf16x2(ov[u * 8 + 4] * inv, ov[u * 8 + 5] * inv);
                    pk.w = pack_bf16x2(ov[u * 8 + 6] * inv, ov[u * 8 + 7] * inv);
                    const int e = c * 32 + u * 8;
                    if (direct) {
                        if (!skip_row) {
                            __nv_bfloat16 *dst = o + (((long long)w.b * a.T + i_row) * a.Hq + w.h) * D + e;
                            *reinterpret_cast<uint4 *>(dst) = pk;
                        }
                    } else {
                        *reinterpret_cast<uint4 *>(sQ + tile_offset<D>(r, e)) = pk;
                    }
                }
            }
            if (a.lse && row_real && !skip_row)
                a.lse[((long long)w.b * a.Hq + w.h) * a.T + i_row] =
                    (l > 0.f) ? (m + __log2f(l)) * 0.69314718055994530942f : -CUDART_INF_F;
        }
        // staging tile complete -> one thread stores it (bounded; an abort
        // anywhere in the CTA skips the store)
        const bool direct_store = (w.mode == 1) || (a.gidx != nullptr && a.g > 0);
        if (!direct_store) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->epi);
            if (r == 0 && wait_bounded(&bars->epi, 0, ctl) && !bars->abort) {
                for (int ch = 0; ch < C::NCH; ++ch)
                    tma_store_4d(&tmO, sQ + ch * C::CH_BYTES, ch * C::E, w.h, w.m0, w.b);
                tma_store_commit();
                tma_store_wait_all();
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ host --

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode()
{
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

// [B,T,H,D] bf16 viewed as a 4-D tensor (D, H, T, B); box = one chunk of 128
// rows of one head.
template <int D>
bool make_map(CUtensorMap *m, const void *ptr, int B, int T, int H)
{
    using C = Cfg<D>;
    EncodeTiledFn enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)T * H * D * 2};
    cuuint32_t box[4] = {(cuuint32_t)C::E, 1, 128, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE,
                     C::RB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_d(int mode, const TcPrefillArgs &a, cudaStream_t s)
{
    using C = Cfg<D>;
    CUtensorMap mq, mk, mv, mo;
    if (!make_map<D>(&mq, a.q, a.B, a.T, a.Hq) || !make_map<D>(&mk, a.k, a.B, a.T, a.Hkv) ||
        !make_map<D>(&mv, a.v, a.B, a.T, a.Hkv) || !make_map<D>(&mo, a.o, a.B, a.T, a.Hq))
        return cudaErrorInvalidValue;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(swa_prefill_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    const int nqt = (a.T + BM - 1) / BM;
    const bool globals = a.gidx != nullptr && a.g > 0;
    int n_mode1 = 0, n_mode0 = 0;
    if (mode == 0) {
        n_mode0 = a.B * a.Hq * nqt;
        if (globals) n_mode1 = a.B * a.Hq * ((a.g + BM - 1) / BM);
    } else {
        n_mode1 = a.B * a.Hq * ((a.g + BM - 1) / BM);
    }
    const int grid = n_mode0 + n_mode1;
    if (grid == 0) return cudaSuccess;
    swa_prefill_tc_kernel<D><<<grid, NTHREADS, C::SMEM_BYTES, s>>>(mq, mk, mv, mo, a, n_mode1);
    return cudaGetLastError();
}

}  // namespace

// mode 0: band tiles (+ dense global-row CTAs first in the same grid when
// global tokens are present); mode 1: dense global rows only.
cudaError_t launch_prefill_tc(int d, int mode, const TcPrefillArgs &a, cudaStream_t s)
{
    switch (d) {
    case 32: return launch_d<32>(mode, a, s);
    case 64: return launch_d<64>(mode, a, s);
    case 128: return launch_d<128>(mode, a, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace swa
