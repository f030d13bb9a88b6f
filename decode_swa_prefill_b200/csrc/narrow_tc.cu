// Causal sliding-window prefill for narrow windows (W <= 64) on tcgen05.
//
// Same operation as the band kernel (for query row i, softmax over keys
// i-W+1 .. i of scale*q.k, then the weighted sum of value rows: "Sliding
// Window Attention", robocikowo.com, opening definition), organised for the
// case where a 128-row query tile sees so few keys that the band kernel's
// per-tile pipeline fill and drain dominate.  A tile at rows q0 .. q0+127
// sees keys q0-PAD .. q0+127 at most (PAD = 32 for W <= 32, 64 for W <= 64),
// so one S = Q K^T of N = 128+PAD columns holds every score of the tile and
// the softmax is a single pass: one row maximum, no rescaling of O, and O
// divided by the row sum in the epilogue once the PV product is done.
//
// Persistent CTAs, one per SM (two TMEM buffers take all 512 columns), walk
// units of (batch, kv head, query tile[, slice of the query heads]) with a
// stride of the grid size; the query heads of a unit share its K/V tile and
// are its jobs.  Job j uses TMEM buffer j & 1:
//   O[b]  columns 256b .. 256b+d-1       fp32 output of the job
//   S[b]  columns 256b+64 .. +128+PAD-1  fp32 scores; P (bf16 pairs) over
//                                        its first (128+PAD)/2 columns
// CTA anatomy (320 threads):
//   warps 0-3  softmax + epilogue of the even jobs (thread r = row r = TMEM
//              lane r), warps 4-7 the same for the odd jobs
//   warp 8     producer: TMA loads of K, V (128+PAD rows) per unit and of Q
//              (128 rows) per job (per pair of jobs with paired head rows)
//              into rings of 3-4 and 4-8 stages
//   warp 9     TMEM allocator and MMA issuer (lane 0): QK^T of job j, then
//              PV of job j-1, so a QK^T runs while the previous job's
//              softmax works.  S[b] is rewritten once the PV that read P[b]
//              has completed, O[b] once the epilogue two jobs back has read
//              it: the epilogue is off the MMA's critical path.
// A warp only computes the 32-key chunks its rows can see (two for PAD 32,
// three for PAD 64) and writes zeros to the rest of its P columns; every
// exponential runs on the MUFU.
//
// Every mbarrier wait is bounded: on expiry the CTA records
// SWA_STATUS_TIMEOUT, drains its in-flight copies and MMAs with a second
// bound, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math_constants.h>

#include "ptx.cuh"
#include "swa_internal.h"
#include "tma_map.h"

namespace swa {
namespace {

constexpr int NB_BM = 128;          // query rows per tile (= TMEM lanes)
constexpr int NB_QST_MAX = 8;      // Q stages (at most)
constexpr int NB_KVST_MAX = 4;     // K/V stages (at most)
constexpr int NB_THREADS = 320;

// HP heads side by side per tile row: HP = 2 for d = 32 loads two adjacent
// heads as one 128-byte row (one TMA row request instead of two; rows of 64
// bytes halve what a load moves per request), and the MMAs of head x of the
// pair start 64 bytes into the row.
template <int D, int PAD, int HP>
struct NCfg {
    static constexpr int KEYS = NB_BM + PAD;                 // key rows of a unit
    static constexpr int RD = HP * D;                        // elements per tile row
    static constexpr int RB = (RD * 2 >= 128) ? 128 : RD * 2; // bytes per swizzled row
    static constexpr int QTILE = NB_BM * RD * 2;             // HP jobs' Q
    static constexpr int KVTILE = KEYS * RD * 2;             // HP kv heads' K (or V)
    static constexpr uint32_t LAYOUT = (RB == 128) ? UMMA_SW128 : UMMA_SW64;
    static constexpr int NCHK = PAD / 32 + 1;                // live 32-key chunks per warp
    // prefetch depth: a load takes a few microseconds, several units' worth
    // of jobs, so as many stages as shared memory holds
    static constexpr int QST = RD == 32 ? 8 : 4;
    static constexpr int KVST = RD == 32 ? 4 : 3;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + QST * QTILE;
    static constexpr int OFF_V = OFF_K + KVST * KVTILE;
    static constexpr int OFF_BAR = OFF_V + KVST * KVTILE;
    // + room to align the base to 1 KiB; more than half the SM's shared
    // memory, so that a second CTA (which would wait for TMEM) never shares
    // the SM
    static constexpr int SMEM_NEED = OFF_BAR + 256 + 1024;
    static constexpr int SMEM_BYTES = SMEM_NEED > 120 * 1024 ? SMEM_NEED : 120 * 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(RD == 32 || RD == 64, "one swizzle chunk per tile row");
    static_assert(HP == 1 || HP == 2, "heads per row");
    static_assert(PAD == 32 || PAD == 64, "pad");
    static_assert(64 + KEYS <= 256 && D <= 64, "one TMEM buffer = 256 columns");
    static_assert(QTILE % 1024 == 0 && KVTILE % 1024 == 0, "1 KiB aligned stages");
    static_assert(SMEM_BYTES <= 227 * 1024, "fits one SM");
    static_assert(2 * (SMEM_BYTES + 1024) > 228 * 1024, "never two CTAs per SM");
    static_assert(QST <= NB_QST_MAX && KVST <= NB_KVST_MAX, "barrier arrays");
};

__host__ __device__ constexpr uint32_t nb_col_o(int b) { return 256u * b; }
__host__ __device__ constexpr uint32_t nb_col_s(int b) { return 256u * b + 64u; }

struct NBars {
    uint64_t q_full[NB_QST_MAX];
    uint64_t q_empty[NB_QST_MAX];
    uint64_t kv_full[NB_KVST_MAX];
    uint64_t kv_empty[NB_KVST_MAX];
    uint64_t s_full[2];
    uint64_t p_full[2];     // one arrival per softmax warp
    uint64_t o_full[2];
    uint64_t tmem_free[2];  // one arrival per epilogue warp
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ void nb_drain_wait(uint64_t *bar, uint32_t parity, unsigned long long limit)
{
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > limit) return;
    }
}

// Unit u -> (batch, group of HP kv heads, query tile, slice of the group's
// query heads); consecutive units share K/V rows (the slices of one tile,
// then the next tile), so neighbouring CTAs find them in L2.
struct NUnit {
    int b, kp, q0, h0; // kp: kv head group (tile row index); h0: first query head
};
__device__ __forceinline__ NUnit nb_unit(int u, int n_kp, int nqt, int n_slice, int gs)
{
    NUnit x;
    x.h0 = (u % n_slice) * gs;
    u /= n_slice;
    x.q0 = (u % nqt) * NB_BM;
    const int r = u / nqt;
    x.kp = r % n_kp;
    x.b = r / n_kp;
    x.h0 += x.kp * gs * n_slice;
    return x;
}

template <int D, int PAD, int HP>
__global__ void __launch_bounds__(NB_THREADS, 1)
    swa_prefill_narrow_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                              const __grid_constant__ CUtensorMap tmV, const TcPrefillArgs a, const int n_units,
                              const int n_slice)
{
    using C = NCfg<D, PAD, HP>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + C::OFF_Q;
    uint8_t *sK = smem + C::OFF_K;
    uint8_t *sV = smem + C::OFF_V;
    NBars *bars = reinterpret_cast<NBars *>(smem + C::OFF_BAR);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int Gq = a.Hq / a.Hkv;             // query heads per kv head
    const int G = HP * Gq / n_slice;         // jobs (query heads) per unit, a multiple of HP
    const int n_kp = a.Hkv / HP;
    const int nqt = (a.T + NB_BM - 1) / NB_BM;
    WaitCtl ctl{&bars->abort, a.ctl.status, a.ctl.limit_ns};

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::QST; ++s) {
            mbar_init(&bars->q_full[s], 1);
            mbar_init(&bars->q_empty[s], 1);
        }
        for (int s = 0; s < C::KVST; ++s) {
            mbar_init(&bars->kv_full[s], 1);
            mbar_init(&bars->kv_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->s_full[b], 1);
            mbar_init(&bars->p_full[b], 4);
            mbar_init(&bars->o_full[b], 1);
            mbar_init(&bars->tmem_free[b], 4);
        }
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        fence_mbar_init();
    }
    if (warp == 8 && lane == 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    if (warp == 9) tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 8) {
        // ------------------------------------------------------ producer --
        int qiss[C::QST] = {}, kviss[C::KVST] = {};
        bool ok = true;
        int jq = 0, it = 0;
        for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++it) {
            const NUnit x = nb_unit(u, n_kp, nqt, n_slice, G);
            SWA_DCHECK(x.q0 >= 0 && x.q0 < a.T && x.kp < n_kp && x.h0 + G <= a.Hq, a.ctl.status);
            const int ks = it % C::KVST;
            ok = warp_wait_bounded(&bars->kv_empty[ks], ((it / C::KVST) & 1) ^ 1, ctl);
            if (!ok) break;
            if (lane == 0) {
                // rows q0-PAD .. q0+127; rows before 0 or past T read zeros
                mbar_expect_tx(&bars->kv_full[ks], 2 * C::KVTILE);
                tma_load_4d(sK + ks * C::KVTILE, &tmK, &bars->kv_full[ks], 0, x.kp, x.q0 - PAD, x.b);
                tma_load_4d(sV + ks * C::KVTILE, &tmV, &bars->kv_full[ks], 0, x.kp, x.q0 - PAD, x.b);
            }
            kviss[ks]++;
            // one Q tile per HP jobs (query heads h0+g .. h0+g+HP-1)
            for (int g = 0; g < G && ok; g += HP, ++jq) {
                const int qs = jq % C::QST;
                ok = warp_wait_bounded(&bars->q_empty[qs], ((jq / C::QST) & 1) ^ 1, ctl);
                if (!ok) break;
                if (lane == 0) {
                    mbar_expect_tx(&bars->q_full[qs], C::QTILE);
                    tma_load_4d(sQ + qs * C::QTILE, &tmQ, &bars->q_full[qs], 0, (x.h0 + g) / HP, x.q0, x.b);
                }
                qiss[qs]++;
            }
        }
        if (!ok && lane == 0) {
            // let our own copies land before the CTA's shared memory goes away
            for (int s = 0; s < C::QST; ++s)
                if (qiss[s] > 0) nb_drain_wait(&bars->q_full[s], (qiss[s] - 1) & 1, a.ctl.limit_ns);
            for (int s = 0; s < C::KVST; ++s)
                if (kviss[s] > 0) nb_drain_wait(&bars->kv_full[s], (kviss[s] - 1) & 1, a.ctl.limit_ns);
        }
    } else if (warp == 9) {
        // ----------------------------------------------------------- MMA --
        // The whole warp runs the schedule; lane 0 issues MMAs and commits.
        constexpr uint32_t idesc_qk = umma_idesc_bf16(NB_BM, C::KEYS, 0, 0);
        constexpr uint32_t idesc_pv = umma_idesc_bf16(NB_BM, D, 0, 1);
        const uint64_t dq0 = umma_smem_desc(smem_u32(sQ), 16, 8 * C::RB, C::LAYOUT);
        const uint64_t dk0 = umma_smem_desc(smem_u32(sK), 16, 8 * C::RB, C::LAYOUT);
        const uint64_t dv0 = umma_smem_desc(smem_u32(sV), C::KEYS * C::RB, 8 * C::RB, C::LAYOUT);
        const bool leader = lane == 0;
        bool ok = true;
        // the job whose PV is still to issue
        int pj = -1, pks = 0, pkvo = 0;
        bool plast = false;
        auto pv_step = [&]() -> bool {
            const int b = pj & 1;
            if (!warp_wait_bounded(&bars->p_full[b], (pj >> 1) & 1, ctl)) return false;
            // O[b] is free once job pj-2's epilogue has read it
            if (pj >= 2 && !warp_wait_bounded(&bars->tmem_free[b], ((pj >> 1) - 1) & 1, ctl)) return false;
            tc_fence_after();
            if (leader) {
                const uint64_t dv = dv0 + (uint64_t)((pks * C::KVTILE + pkvo) >> 4);
#pragma unroll
                for (int kk = 0; kk < C::KEYS / 16; ++kk)
                    mma_bf16_ts(tmem + nb_col_o(b), tmem + nb_col_s(b) + kk * 8,
                                dv + (uint64_t)((kk * 16 * C::RB) >> 4), idesc_pv, kk > 0 ? 1u : 0u);
                mma_commit(&bars->o_full[b]);
                if (plast) mma_commit(&bars->kv_empty[pks]);
            }
            __syncwarp();
            pj = -1;
            return true;
        };
        int j = 0, it = 0;
        for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++it) {
            const NUnit un = nb_unit(u, n_kp, nqt, n_slice, G);
            const int ks = it % C::KVST;
            // the previous unit's last PV does not wait for this unit's K/V
            if (pj >= 0) ok = pv_step();
            if (!ok) break;
            ok = warp_wait_bounded(&bars->kv_full[ks], (it / C::KVST) & 1, ctl);
            for (int g = 0; g < G && ok; ++g, ++j) {
                // Q tile of job pair j / HP; byte offsets of this job's head
                // in the Q row and of its kv head in the K/V row
                const int jp = j / HP, qs = jp % C::QST, b = j & 1;
                const int h = un.h0 + g;
                const int qo = (h % HP) * D * 2, kvo = ((h / Gq) % HP) * D * 2;
                ok = warp_wait_bounded(&bars->q_full[qs], (jp / C::QST) & 1, ctl);
                // S[b] (P of job j-2) is free once that job's PV has completed
                if (ok && j >= 2) ok = warp_wait_bounded(&bars->o_full[b], ((j >> 1) - 1) & 1, ctl);
                if (!ok) break;
                tc_fence_after();
                if (leader) {
                    const uint64_t dq = dq0 + (uint64_t)((qs * C::QTILE + qo) >> 4);
                    const uint64_t dk = dk0 + (uint64_t)((ks * C::KVTILE + kvo) >> 4);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_bf16_ss(tmem + nb_col_s(b), dq + 2 * kk, dk + 2 * kk, idesc_qk, kk > 0 ? 1u : 0u);
                    mma_commit(&bars->s_full[b]);
                    if (g % HP == HP - 1) mma_commit(&bars->q_empty[qs]);
                }
                __syncwarp();
                if (pj >= 0) ok = pv_step();
                pj = j;
                pks = ks;
                pkvo = kvo;
                plast = (g == G - 1);
            }
        }
        if (ok && pj >= 0) ok = pv_step();
        // all MMAs lane 0 issued are complete before TMEM is freed
        if (leader) {
            mma_commit(&bars->drain);
            nb_drain_wait(&bars->drain, 0, a.ctl.limit_ns);
        }
        __syncwarp();
    } else {
        // ------------------------------------------- softmax + epilogue --
        const int x = warp / 4;            // jobs with j & 1 == x
        const int quarter = warp % 4;
        const int r = quarter * 32 + lane; // row in tile = TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t s_base = tmem + lane_off + nb_col_s(x);
        const uint32_t o_base = tmem + lane_off + nb_col_o(x);
        const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
        __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(a.o);
        bool ok = true;
        int j = 0;
        for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
            const NUnit un = nb_unit(u, n_kp, nqt, n_slice, G);
            const int i = un.q0 + r;          // query position of this thread's row
            const bool row_real = i < a.T;
            // visible key columns of this row: key position q0-PAD+c for
            // column c, from max(i-left, 0) to i; as offsets e from the
            // warp's first live column 32*quarter: e_lo <= e <= lane + PAD
            // (rows past T compute garbage that is never stored)
            const int e_lo = max(r + PAD - a.left, PAD - un.q0) - quarter * 32;
            const int e_hi = lane + PAD;
            for (int g = 0; g < G; ++g, ++j) {
                if ((j & 1) != x) continue;
                ok = warp_wait_bounded(&bars->s_full[x], (j >> 1) & 1, ctl);
                if (!ok) break;
                tc_fence_after();
                float sr[C::NCHK * 32];
#pragma unroll
                for (int cc = 0; cc < C::NCHK; ++cc) tmem_ld32(s_base + (quarter + cc) * 32, sr + cc * 32);
                tmem_ld_wait_dep(sr);
#pragma unroll
                for (int cc = 1; cc < C::NCHK; ++cc) reg_fence32(sr + cc * 32);
                // -inf outside the window: only the last chunk can pass e_hi
                // (e_hi >= PAD), every chunk e_lo
#pragma unroll
                for (int e = 0; e < C::NCHK * 32; ++e) {
                    bool keep = e >= e_lo;
                    if (e > PAD) keep = keep && e <= e_hi;
                    sr[e] = keep ? sr[e] : -CUDART_INF_F;
                }
                float mx4[4];
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) mx4[k4] = fmax3(sr[k4], sr[4 + k4], sr[8 + k4]);
#pragma unroll
                for (int e = 12; e + 8 <= C::NCHK * 32; e += 8)
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) mx4[k4] = fmax3(mx4[k4], sr[e + k4], sr[e + 4 + k4]);
#pragma unroll
                for (int e = 12 + ((C::NCHK * 32 - 12) / 8) * 8; e < C::NCHK * 32; e += 4)
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) mx4[k4] = fmaxf(mx4[k4], sr[e + k4]);
                const float mx = fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
                const float m = mx * a.scale_log2;
                const float ref = (mx == -CUDART_INF_F) ? 0.f : m;
                const float2 nr2 = make_float2(-ref, -ref);
                float2 acc2 = make_float2(0.f, 0.f), acc2b = make_float2(0.f, 0.f);
                // P = 2^(s*scale*log2e - m) as bf16 pairs over the first
                // KEYS/2 columns of S (O is divided by the row sum in the
                // epilogue); columns of chunks this warp cannot see are zero
                uint32_t pk[C::NCHK * 16];
#pragma unroll
                for (int e = 0; e < C::NCHK * 32; e += 2) {
                    float2 y = fma2(make_float2(sr[e], sr[e + 1]), sc2, nr2);
                    y.x = ex2_approx(y.x);
                    y.y = ex2_approx(y.y);
                    if (e & 2) acc2b = add2(acc2b, y);
                    else acc2 = add2(acc2, y);
                    pk[e / 2] = pack_bf16x2(y.x, y.y);
                }
                const float2 tot = add2(acc2, acc2b);
                const float l = tot.x + tot.y;
                const float inv = (l > 0.f) ? 1.f / l : 0.f;
                uint32_t zero[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) zero[e] = 0u;
#pragma unroll
                for (int cu = 0; cu < C::KEYS / 32; ++cu) {
                    const int cc = cu - quarter;
                    if (cc >= 0 && cc < C::NCHK) continue;
                    tmem_st16u(s_base + cu * 16, zero);
                }
#pragma unroll
                for (int cc = 0; cc < C::NCHK; ++cc) tmem_st16u(s_base + (quarter + cc) * 16, pk + cc * 16);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->p_full[x]);

                // ---- epilogue: O is final once this job's PV completes ----
                const int h = un.h0 + g;
                if (a.lse && row_real)
                    a.lse[((long long)un.b * a.Hq + h) * a.T + i] =
                        (l > 0.f) ? (m + __log2f(l)) * 0.69314718055994530942f : -CUDART_INF_F;
                ok = warp_wait_bounded(&bars->o_full[x], (j >> 1) & 1, ctl);
                if (!ok) break;
                tc_fence_after();
                __nv_bfloat16 *dst = out + (((long long)un.b * a.T + i) * a.Hq + h) * D;
#pragma unroll
                for (int cc = 0; cc < D / 16; ++cc) {
                    float ov[16];
                    tmem_ld16(o_base + cc * 16, ov);
                    tmem_ld_wait_dep16(ov);
                    uint4 pk0, pk1;
                    pk0.x = pack_bf16x2(ov[0] * inv, ov[1] * inv);
                    pk0.y = pack_bf16x2(ov[2] * inv, ov[3] * inv);
                    pk0.z = pack_bf16x2(ov[4] * inv, ov[5] * inv);
                    pk0.w = pack_bf16x2(ov[6] * inv, ov[7] * inv);
                    pk1.x = pack_bf16x2(ov[8] * inv, ov[9] * inv);
                    pk1.y = pack_bf16x2(ov[10] * inv, ov[11] * inv);
                    pk1.z = pack_bf16x2(ov[12] * inv, ov[13] * inv);
                    pk1.w = pack_bf16x2(ov[14] * inv, ov[15] * inv);
                    if (row_real) {
                        reinterpret_cast<uint4 *>(dst + cc * 16)[0] = pk0;
                        reinterpret_cast<uint4 *>(dst + cc * 16)[1] = pk1;
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->tmem_free[x]);
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

template <int D, int PAD, int HP>
cudaError_t launch_narrow_dp(const TcPrefillArgs &a, cudaStream_t s)
{
    using C = NCfg<D, PAD, HP>;
    // HP adjacent heads as one row of HP*D elements
    CUtensorMap mq, mk, mv;
    if (!make_bthd_map(&mq, a.q, a.B, a.T, a.Hq / HP, C::RD, NB_BM) ||
        !make_bthd_map(&mk, a.k, a.B, a.T, a.Hkv / HP, C::RD, C::KEYS) ||
        !make_bthd_map(&mv, a.v, a.B, a.T, a.Hkv / HP, C::RD, C::KEYS))
        return cudaErrorInvalidValue;
    static DeviceOnce once;
    int n_sm = 0;
    cudaError_t e = once.get(
        [&](int) {
            return cudaFuncSetAttribute(swa_prefill_narrow_kernel<D, PAD, HP>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        },
        &n_sm);
    if (e != cudaSuccess) return e;
    // a unit takes all G query heads of its tile (one K/V load) unless that
    // leaves fewer than ~6 units per SM: then the heads are split in halves
    // (quarters, ...), trading an L2 re-read of K/V for a shorter tail
    const int G = HP * (a.Hq / a.Hkv);
    long long units = (long long)a.B * (a.Hkv / HP) * ((a.T + NB_BM - 1) / NB_BM);
    int n_slice = 1;
    if (HP == 1)
        while (G % (2 * n_slice) == 0 && units * n_slice < 6LL * n_sm) n_slice *= 2;
    units *= n_slice;
    if (units == 0) return cudaSuccess;
    if (units > 0x7fffffffLL) return cudaErrorInvalidValue;
    const int grid = (int)(units < n_sm ? units : n_sm);
    swa_prefill_narrow_kernel<D, PAD, HP><<<grid, NB_THREADS, C::SMEM_BYTES, s>>>(mq, mk, mv, a, (int)units, n_slice);
    return cudaGetLastError();
}

}  // namespace

bool prefill_narrow_applies(int d, const TcPrefillArgs &a)
{
    return (d == 32 || d == 64) && a.right == 0 && a.left >= 0 && a.left <= 63 && a.gidx == nullptr && a.g == 0;
}

cudaError_t launch_prefill_narrow(int d, const TcPrefillArgs &a, cudaStream_t s)
{
    if (!prefill_narrow_applies(d, a)) return cudaErrorInvalidValue;
    if (d == 32) {
        // one query head per kv head and an even head count: two adjacent
        // heads per tile row, so a unit has two jobs and its loads half the
        // rows (with larger groups a unit already has several jobs, and
        // single-head rows with sliced units measured faster)
        if (a.Hkv % 2 == 0 && a.Hq == a.Hkv)
            return a.left <= 31 ? launch_narrow_dp<32, 32, 2>(a, s) : launch_narrow_dp<32, 64, 2>(a, s);
        return a.left <= 31 ? launch_narrow_dp<32, 32, 1>(a, s) : launch_narrow_dp<32, 64, 1>(a, s);
    }
    return a.left <= 31 ? launch_narrow_dp<64, 32, 1>(a, s) : launch_narrow_dp<64, 64, 1>(a, s);
}

}  // namespace swa
