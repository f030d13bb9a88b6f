// Backward pass of the sliding-window prefill on tcgen05 tensor cores
// (sm_100a): dq, dk, dv for an upstream gradient dout.
//
// The pages define only the forward computation (for query row i, softmax
// over the keys of its window of scale*q.k, then the weighted sum of value
// rows: "Sliding Window Attention", robocikowo.com, opening definition).  This
// file computes that definition's gradient by the chain rule, recomputing the
// probabilities from the forward pass's log-sum-exp instead of storing them:
//   p_ij  = exp(scale q_i.k_j - lse_i)          (j in the window of i)
//   dp_ij = dout_i . v_j,   D_i = dout_i . o_i  (= sum_j p_ij dp_ij)
//   ds_ij = p_ij (dp_ij - D_i)
//   dq_i  = scale sum_j ds_ij k_j
//   dk_j  = scale sum_i ds_ij q_i,   dv_j = sum_i p_ij dout_i
// Only the 128 x 128 tiles that meet the window are visited, so the work is
// O(T W d) like the forward pass.
//
// Three launches:
//   bwd_delta_kernel   D_i = dout_i . o_i (fp32), 16-byte loads, D/8 lanes per row
//   bwd_dq_kernel      one CTA per (batch, query head, 128-row query tile):
//                      per 128-key tile, in two halves of 64 keys, S = Q K^T
//                      and dP = dO V^T into TMEM, the elementwise warps turn
//                      them into dS (bf16, over the S columns), then dQ +=
//                      dS K accumulates in TMEM; one half's elementwise pass
//                      runs while the tensor core works on the other half
//   bwd_dkdv_kernel    one CTA per (batch, kv head, 128-key tile): per
//                      (query head of the group, 128-row query tile)
//                      S^T = K Q^T and dP^T = V dO^T, then P^T and dS^T
//                      (bf16, over their own columns), dV += P^T dO and
//                      dK += dS^T Q in TMEM; the query heads of a group add
//                      into the same accumulators, so no atomics are needed
// CTA anatomy of the two tcgen05 kernels (192 threads): warps 0-3 elementwise
// and epilogue (thread r owns TMEM lane r), warp 4 TMA producer (two stages,
// no multicast), warp 5 TMEM allocator and MMA issuer (lane 0).  An MMA
// that reads bf16 dS (or P) from TMEM is followed in issue order by the next
// tile's S, dP MMAs that overwrite those columns; the tensor core runs one
// thread's MMAs in order, so no wait separates them.
//
// Every mbarrier wait is bounded: on expiry the CTA records
// SWA_STATUS_TIMEOUT, drains its own copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math_constants.h>

#include "ptx.cuh"
#include "swa_internal.h"
#include "tma_map.h"

namespace swa {
namespace {

constexpr int BW_T = 128;          // rows of a query tile and of a key tile
constexpr int BW_THREADS = 192;

template <int D>
struct BCfg {
    static constexpr int NCH = D / 64;             // 64-element (128-byte) chunks per row
    static constexpr int CH = BW_T * 128;          // one chunk of a 128-row tile
    static constexpr int TILE = BW_T * D * 2;
    static_assert(D == 64 || D == 128, "head dim");
};

struct BwdBars {
    uint64_t fixed_full;      // the CTA's own tiles (Q and dO, or K and V)
    uint64_t full[2];         // streamed tiles of a step
    uint64_t empty[2];
    uint64_t s_full[2];       // S and dP (or their transposes) complete [half of the key tile; dK/dV: [0]]
    uint64_t p_full[2];       // dS (and P) written, one arrival per warp [likewise]
    uint64_t done;            // the last accumulating MMA complete
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ void bw_drain_wait(uint64_t *bar, uint32_t parity, unsigned long long limit)
{
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > limit) return;
    }
}

// Two K-major operands from shared memory into 128 TMEM columns:
// d_tmem = A B^T over the head dimension (8 or 4 MMAs of K = 16).
template <int D>
__device__ __forceinline__ void bw_mma_rows(uint32_t d_tmem, uint64_t da, uint64_t db)
{
    using C = BCfg<D>;
    constexpr uint32_t idesc = umma_idesc_bf16(BW_T, BW_T, 0, 0);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const int byte = kk * 32;
        const uint64_t off = (uint64_t)(((byte / 128) * C::CH + (byte % 128)) >> 4);
        mma_bf16_ss(d_tmem, da + off, db + off, idesc, kk > 0 ? 1u : 0u);
    }
}

// d_tmem (D columns) += A B over 128 rows of the contraction: A (bf16,
// 128 rows x 128) from TMEM at a_tmem, B a [128 rows][D] tile read as an
// MN-major operand (the rows are the contraction).
template <int D>
__device__ __forceinline__ void bw_mma_acc(uint32_t d_tmem, uint32_t a_tmem, uint64_t db_mn, bool acc_first)
{
    constexpr uint32_t idesc = umma_idesc_bf16(BW_T, D, 0, 1);
#pragma unroll
    for (int kk = 0; kk < BW_T / 16; ++kk)
        mma_bf16_ts(d_tmem, a_tmem + kk * 8, db_mn + (uint64_t)((kk * 16 * 128) >> 4), idesc,
                    (acc_first || kk > 0) ? 1u : 0u);
}

// The same two products for one half of the key tile: d_tmem (64 columns) =
// A B^T with B the 64 rows of the tile from row 64h (8-row swizzle atoms, so
// the start moves by whole 1 KB blocks).
template <int D>
__device__ __forceinline__ void bw_mma_rows_half(uint32_t d_tmem, uint64_t da, uint64_t db, int h)
{
    using C = BCfg<D>;
    constexpr uint32_t idesc = umma_idesc_bf16(BW_T, BW_T / 2, 0, 0);
    const uint64_t dbh = db + (uint64_t)((h * (BW_T / 2) * 128) >> 4);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const int byte = kk * 32;
        const uint64_t off = (uint64_t)(((byte / 128) * C::CH + (byte % 128)) >> 4);
        mma_bf16_ss(d_tmem, da + off, dbh + off, idesc, kk > 0 ? 1u : 0u);
    }
}

// d_tmem += A B over the 64 contraction rows of half h: A (bf16, 128 rows x
// 64) from TMEM at a_tmem, B rows 64h .. 64h+63 of a [128 rows][D] tile
// read MN-major.
template <int D>
__device__ __forceinline__ void bw_mma_acc_half(uint32_t d_tmem, uint32_t a_tmem, uint64_t db_mn, int h,
                                                bool acc_first)
{
    constexpr uint32_t idesc = umma_idesc_bf16(BW_T, D, 0, 1);
    const uint64_t dbh = db_mn + (uint64_t)((h * (BW_T / 2) * 128) >> 4);
#pragma unroll
    for (int kk = 0; kk < BW_T / 32; ++kk)
        mma_bf16_ts(d_tmem, a_tmem + kk * 8, dbh + (uint64_t)((kk * 16 * 128) >> 4), idesc,
                    (acc_first || kk > 0) ? 1u : 0u);
}

__device__ __forceinline__ bool bw_allowed(int i, int j, int T, int left, int right)
{
    return i < T && j < T && j >= i - left && j <= i + right;
}

// ------------------------------------------------------------ D_i = dO.O --
// D/8 lanes per row, 16 bytes each; a warp takes BW_DPASS groups of 32/(D/8)
// consecutive rows, all loads issued before the first product.
constexpr int BW_DPASS = 4;

template <int D>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const __nv_bfloat16 *dout, const __nv_bfloat16 *o,
                                                         float *delta, int B, int T, int Hq)
{
    constexpr int LPR = D / 8;        // lanes per row
    constexpr int RPW = 32 / LPR;     // rows per warp and pass
    const long long rows = (long long)B * T * Hq;   // row = (b*T + i)*Hq + h
    const int lane = threadIdx.x % 32;
    const long long r0 = ((long long)blockIdx.x * 8 + threadIdx.x / 32) * RPW * BW_DPASS + lane / LPR;
    const int e0 = (lane % LPR) * 8;
    uint4 g[BW_DPASS], x[BW_DPASS];
#pragma unroll
    for (int p = 0; p < BW_DPASS; ++p) {
        const long long row = r0 + (long long)p * RPW;
        g[p] = make_uint4(0, 0, 0, 0);
        x[p] = make_uint4(0, 0, 0, 0);
        if (row < rows) {
            g[p] = __ldg(reinterpret_cast<const uint4 *>(dout + row * D + e0));
            x[p] = __ldg(reinterpret_cast<const uint4 *>(o + row * D + e0));
        }
    }
#pragma unroll
    for (int p = 0; p < BW_DPASS; ++p) {
        const uint32_t gu[4] = {g[p].x, g[p].y, g[p].z, g[p].w}, xu[4] = {x[p].x, x[p].y, x[p].z, x[p].w};
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            acc += __uint_as_float(gu[k] << 16) * __uint_as_float(xu[k] << 16);
            acc += __uint_as_float(gu[k] & 0xffff0000u) * __uint_as_float(xu[k] & 0xffff0000u);
        }
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        const long long row = r0 + (long long)p * RPW;
        if (lane % LPR == 0 && row < rows) {
            const long long h = row % Hq, bi = row / Hq, i = bi % T, b = bi / T;
            delta[(b * Hq + h) * T + i] = acc;
        }
    }
}

// ------------------------------------------------------------------- dQ --
template <int D>
__global__ void __launch_bounds__(BW_THREADS, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const BwdArgs a)
{
    using C = BCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;                       // Q tile, then dO tile
    uint8_t *sDO = smem + C::TILE;
    uint8_t *sKV = smem + 2 * C::TILE;        // stage st: K at sKV + 2st TILE, V after it
    BwdBars *bars = reinterpret_cast<BwdBars *>(smem + 6 * C::TILE);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int m0 = qt * BW_T;
    const int hk = h / (a.Hq / a.Hkv);
    const int lo = max(0, m0 - a.left), hi = min(a.T - 1, m0 + BW_T - 1 + a.right);
    const int t0 = lo / BW_T, n = hi / BW_T - t0 + 1;
    WaitCtl ctl{&bars->abort, a.ctl.status, a.ctl.limit_ns};

    if (threadIdx.x == 0) {
        mbar_init(&bars->fixed_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int h = 0; h < 2; ++h) {
            mbar_init(&bars->s_full[h], 1);
            mbar_init(&bars->p_full[h], 4);
        }
        mbar_init(&bars->done, 1);
        bars->abort = 0;
        fence_mbar_init();
    }
    if (warp == 4 && lane == 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        prefetch_tensormap(&tmDO);
    }
    if (warp == 5) tmem_alloc(&bars->tmem_base, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 4) {
        // ------------------------------------------------------ producer --
        int iss[2] = {0, 0};
        bool ok = true;
        if (lane == 0) {
            mbar_expect_tx(&bars->fixed_full, 2 * C::TILE);
            for (int ch = 0; ch < C::NCH; ++ch) {
                tma_load_4d(sQ + ch * C::CH, &tmQ, &bars->fixed_full, ch * 64, h, m0, b);
                tma_load_4d(sDO + ch * C::CH, &tmDO, &bars->fixed_full, ch * 64, h, m0, b);
            }
        }
        for (int t = 0; t < n && ok; ++t) {
            const int st = t & 1;
            ok = warp_wait_bounded(&bars->empty[st], ((t >> 1) & 1) ^ 1, ctl);
            if (!ok) break;
            const int key0 = (t0 + t) * BW_T;
            SWA_DCHECK(key0 >= 0 && key0 < a.T, a.ctl.status);
            if (lane == 0) {
                uint8_t *dk = sKV + 2 * st * C::TILE;
                mbar_expect_tx(&bars->full[st], 2 * C::TILE);
                for (int ch = 0; ch < C::NCH; ++ch) {
                    tma_load_4d(dk + ch * C::CH, &tmK, &bars->full[st], ch * 64, hk, key0, b);
                    tma_load_4d(dk + C::TILE + ch * C::CH, &tmV, &bars->full[st], ch * 64, hk, key0, b);
                }
            }
            iss[st]++;
        }
        if (!ok && lane == 0)
            for (int s = 0; s < 2; ++s)
                if (iss[s] > 0) bw_drain_wait(&bars->full[s], (iss[s] - 1) & 1, a.ctl.limit_ns);
    } else if (warp == 5) {
        // ----------------------------------------------------------- MMA --
        const bool leader = lane == 0;
        const uint64_t dq = umma_smem_desc(smem_u32(sQ), 16, 8 * 128, UMMA_SW128);
        const uint64_t ddo = umma_smem_desc(smem_u32(sDO), 16, 8 * 128, UMMA_SW128);
        // Key tiles in two halves of 64 keys: S_h, dP_h into columns 64h and
        // 128 + 64h, dS_h (bf16) over the first 32 of S_h's.  The next
        // tile's half h is issued as soon as this tile's dQ += dS_h K_h is,
        // so one half's elementwise pass runs while the tensor core works on
        // the other half; the tensor core runs these MMAs in issue order, so
        // no wait separates a dS read from the S write that follows it.
        auto s_dp = [&](int st, int h) {
            const uint32_t ks = smem_u32(sKV + 2 * st * C::TILE), vs = ks + C::TILE;
            bw_mma_rows_half<D>(tmem + 64 * h, dq, umma_smem_desc(ks, 16, 8 * 128, UMMA_SW128), h);        // S_h
            bw_mma_rows_half<D>(tmem + 128 + 64 * h, ddo, umma_smem_desc(vs, 16, 8 * 128, UMMA_SW128), h); // dP_h
            mma_commit(&bars->s_full[h]);
        };
        bool ok = warp_wait_bounded(&bars->fixed_full, 0, ctl);
        if (ok && n > 0) ok = warp_wait_bounded(&bars->full[0], 0, ctl);
        if (ok && n > 0) {
            tc_fence_after();
            if (leader) {
                s_dp(0, 0);
                s_dp(0, 1);
            }
            __syncwarp();
        }
        for (int t = 0; t < n && ok; ++t) {
            const int st = t & 1;
            const bool more = t + 1 < n;
            const uint32_t ks = smem_u32(sKV + 2 * st * C::TILE);
            const uint64_t dk_mn = umma_smem_desc(ks, C::CH, 8 * 128, UMMA_SW128);
            // half 0: dQ += dS_0 K_0, then the next tile's S_0, dP_0
            ok = warp_wait_bounded(&bars->p_full[0], t & 1, ctl);
            if (ok && more) ok = warp_wait_bounded(&bars->full[st ^ 1], ((t + 1) >> 1) & 1, ctl);
            if (!ok) break;
            tc_fence_after();
            if (leader) {
                bw_mma_acc_half<D>(tmem + 256, tmem, dk_mn, 0, t > 0);
                if (more) s_dp(st ^ 1, 0);
            }
            __syncwarp();
            // half 1: dQ += dS_1 K_1; the stage is free; the next tile's S_1, dP_1
            ok = warp_wait_bounded(&bars->p_full[1], t & 1, ctl);
            if (!ok) break;
            tc_fence_after();
            if (leader) {
                bw_mma_acc_half<D>(tmem + 256, tmem + 64, dk_mn, 1, true);
                mma_commit(&bars->empty[st]);
                if (more) s_dp(st ^ 1, 1);
            }
            __syncwarp();
        }
        if (leader) {
            mma_commit(&bars->done);
            if (!ok) bw_drain_wait(&bars->done, 0, a.ctl.limit_ns);
        }
        __syncwarp();
    } else {
        // ------------------------------------------- elementwise + epilogue --
        const int r = warp * 32 + lane;
        const int i = m0 + r;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const long long rowid = ((long long)b * a.Hq + h) * a.T + i;
        const float lse2 = i < a.T ? a.lse[rowid] * 1.4426950408889634f : CUDART_INF_F;
        const float dl = i < a.T ? a.delta[rowid] : 0.f;
        bool ok = true;
        for (int t = 0; t < n && ok; ++t) {
            const int key0 = (t0 + t) * BW_T;
            for (int h = 0; h < 2; ++h) {
                ok = warp_wait_bounded(&bars->s_full[h], t & 1, ctl);
                if (!ok) break;
                tc_fence_after();
#pragma unroll 1
                for (int c2 = 0; c2 < 2; ++c2) {
                    const int cc = 2 * h + c2;   // 32-key chunk of the tile
                    float s[32], dp[32];
                    tmem_ld32(tmem + lane_off + cc * 32, s);
                    tmem_ld32(tmem + lane_off + 128 + cc * 32, dp);
                    tmem_ld_wait_dep(s);
                    reg_fence32(dp);
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const int j = key0 + cc * 32 + e;
                        const float p0 =
                            bw_allowed(i, j, a.T, a.left, a.right) ? ex2_approx(s[e] * a.scale_log2 - lse2) : 0.f;
                        const float p1 = bw_allowed(i, j + 1, a.T, a.left, a.right)
                                             ? ex2_approx(s[e + 1] * a.scale_log2 - lse2)
                                             : 0.f;
                        pk[e / 2] = pack_bf16x2(p0 * (dp[e] - dl), p1 * (dp[e + 1] - dl));
                    }
                    // dS of this half: bf16 pairs from column 64h on
                    tmem_st16u(tmem + lane_off + 64 * h + c2 * 16, pk);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->p_full[h]);
            }
        }
        // ---- epilogue: dQ * scale -> bf16 ----
        // (the TMEM loads are warp-wide: every lane takes part, rows past T
        // only skip their stores)
        if (ok) ok = warp_wait_bounded(&bars->done, 0, ctl);
        __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(a.dq) + (((long long)b * a.T + i) * a.Hq + h) * D;
        if (ok) {
            tc_fence_after();
#pragma unroll 1
            for (int cc = 0; cc < D / 16; ++cc) {
                float v[16];
                tmem_ld16(tmem + lane_off + 256 + cc * 16, v);
                tmem_ld_wait_dep16(v);
                if (i < a.T) {
                    uint4 u0, u1;
                    u0.x = pack_bf16x2(v[0] * a.scale, v[1] * a.scale);
                    u0.y = pack_bf16x2(v[2] * a.scale, v[3] * a.scale);
                    u0.z = pack_bf16x2(v[4] * a.scale, v[5] * a.scale);
                    u0.w = pack_bf16x2(v[6] * a.scale, v[7] * a.scale);
                    u1.x = pack_bf16x2(v[8] * a.scale, v[9] * a.scale);
                    u1.y = pack_bf16x2(v[10] * a.scale, v[11] * a.scale);
                    u1.z = pack_bf16x2(v[12] * a.scale, v[13] * a.scale);
                    u1.w = pack_bf16x2(v[14] * a.scale, v[15] * a.scale);
                    reinterpret_cast<uint4 *>(dst + cc * 16)[0] = u0;
                    reinterpret_cast<uint4 *>(dst + cc * 16)[1] = u1;
                }
                __syncwarp();
            }
        } else if (i < a.T) {
            // leave no stale rows behind on an aborted CTA
            for (int e = 0; e < D; e += 8) *reinterpret_cast<uint4 *>(dst + e) = make_uint4(0, 0, 0, 0);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- dK, dV --
template <int D>
__global__ void __launch_bounds__(BW_THREADS, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const BwdArgs a)
{
    using C = BCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sK = smem, *sV = smem + C::TILE;
    uint8_t *sQD = smem + 2 * C::TILE;                                   // stage st: Q, then dO
    float *vec = reinterpret_cast<float *>(smem + 6 * C::TILE);          // stage st: lse2[128], delta[128]
    BwdBars *bars = reinterpret_cast<BwdBars *>(smem + 6 * C::TILE + 2048);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int kt = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const int j0 = kt * BW_T;
    const int G = a.Hq / a.Hkv;
    // query rows whose window holds a key of this tile
    const int ilo = max(0, j0 - a.right), ihi = min(a.T - 1, j0 + BW_T - 1 + a.left);
    const int u0 = ilo / BW_T, nu = ihi / BW_T - u0 + 1;
    const int nsteps = G * nu;
    WaitCtl ctl{&bars->abort, a.ctl.status, a.ctl.limit_ns};

    if (threadIdx.x == 0) {
        mbar_init(&bars->fixed_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        mbar_init(&bars->s_full[0], 1);
        mbar_init(&bars->p_full[0], 4);
        mbar_init(&bars->done, 1);
        bars->abort = 0;
        fence_mbar_init();
    }
    if (warp == 4 && lane == 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        prefetch_tensormap(&tmDO);
    }
    if (warp == 5) tmem_alloc(&bars->tmem_base, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 4) {
        // ------------------------------------------------------ producer --
        int iss[2] = {0, 0};
        bool ok = true;
        if (lane == 0) {
            mbar_expect_tx(&bars->fixed_full, 2 * C::TILE);
            for (int ch = 0; ch < C::NCH; ++ch) {
                tma_load_4d(sK + ch * C::CH, &tmK, &bars->fixed_full, ch * 64, hk, j0, b);
                tma_load_4d(sV + ch * C::CH, &tmV, &bars->fixed_full, ch * 64, hk, j0, b);
            }
        }
        for (int s = 0; s < nsteps && ok; ++s) {
            const int st = s & 1;
            ok = warp_wait_bounded(&bars->empty[st], ((s >> 1) & 1) ^ 1, ctl);
            if (!ok) break;
            const int h = hk * G + s / nu, m0 = (u0 + s % nu) * BW_T;
            SWA_DCHECK(m0 >= 0 && m0 < a.T && h < a.Hq, a.ctl.status);
            // the step's log-sum-exp (log2 units) and D of its 128 query rows;
            // rows past T get a probability of 0
            float *lv = vec + st * 256;
            for (int rr = lane; rr < BW_T; rr += 32) {
                const int i = m0 + rr;
                const long long id = ((long long)b * a.Hq + h) * a.T + i;
                lv[rr] = i < a.T ? a.lse[id] * 1.4426950408889634f : CUDART_INF_F;
                lv[BW_T + rr] = i < a.T ? a.delta[id] : 0.f;
            }
            __syncwarp();
            if (lane == 0) {
                uint8_t *dq = sQD + 2 * st * C::TILE;
                mbar_expect_tx(&bars->full[st], 2 * C::TILE);
                for (int ch = 0; ch < C::NCH; ++ch) {
                    tma_load_4d(dq + ch * C::CH, &tmQ, &bars->full[st], ch * 64, h, m0, b);
                    tma_load_4d(dq + C::TILE + ch * C::CH, &tmDO, &bars->full[st], ch * 64, h, m0, b);
                }
            }
            iss[st]++;
        }
        if (!ok && lane == 0)
            for (int s = 0; s < 2; ++s)
                if (iss[s] > 0) bw_drain_wait(&bars->full[s], (iss[s] - 1) & 1, a.ctl.limit_ns);
    } else if (warp == 5) {
        // ----------------------------------------------------------- MMA --
        const bool leader = lane == 0;
        const uint64_t dk = umma_smem_desc(smem_u32(sK), 16, 8 * 128, UMMA_SW128);
        const uint64_t dv = umma_smem_desc(smem_u32(sV), 16, 8 * 128, UMMA_SW128);
        bool ok = warp_wait_bounded(&bars->fixed_full, 0, ctl);
        for (int s = 0; s < nsteps && ok; ++s) {
            const int st = s & 1;
            ok = warp_wait_bounded(&bars->full[st], (s >> 1) & 1, ctl);
            if (!ok) break;
            tc_fence_after();
            const uint32_t qs = smem_u32(sQD + 2 * st * C::TILE), gs = qs + C::TILE;
            if (leader) {
                bw_mma_rows<D>(tmem, dk, umma_smem_desc(qs, 16, 8 * 128, UMMA_SW128));        // S^T  = K Q^T
                bw_mma_rows<D>(tmem + 128, dv, umma_smem_desc(gs, 16, 8 * 128, UMMA_SW128));  // dP^T = V dO^T
                mma_commit(&bars->s_full[0]);
            }
            __syncwarp();
            ok = warp_wait_bounded(&bars->p_full[0], s & 1, ctl);
            if (!ok) break;
            tc_fence_after();
            if (leader) {
                // dV += P^T dO and dK += dS^T Q (P^T, dS^T: bf16 over their columns)
                bw_mma_acc<D>(tmem + 256, tmem, umma_smem_desc(gs, C::CH, 8 * 128, UMMA_SW128), s > 0);
                bw_mma_acc<D>(tmem + 256 + D, tmem + 128, umma_smem_desc(qs, C::CH, 8 * 128, UMMA_SW128), s > 0);
                mma_commit(&bars->empty[st]);
            }
            __syncwarp();
        }
        if (leader) {
            mma_commit(&bars->done);
            if (!ok) bw_drain_wait(&bars->done, 0, a.ctl.limit_ns);
        }
        __syncwarp();
    } else {
        // ------------------------------------------- elementwise + epilogue --
        const int r = warp * 32 + lane;
        const int j = j0 + r;                   // key position of this TMEM lane
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        bool ok = true;
        for (int s = 0; s < nsteps; ++s) {
            ok = warp_wait_bounded(&bars->s_full[0], s & 1, ctl);
            if (!ok) break;
            tc_fence_after();
            const int m0 = (u0 + s % nu) * BW_T;
            const float *lv = vec + (s & 1) * 256;
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                float sv[32], dp[32];
                tmem_ld32(tmem + lane_off + cc * 32, sv);
                tmem_ld32(tmem + lane_off + 128 + cc * 32, dp);
                tmem_ld_wait_dep(sv);
                reg_fence32(dp);
                uint32_t pk[16], dk16[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const int q0 = cc * 32 + e;
                    const int i = m0 + q0;
                    const float p0 =
                        bw_allowed(i, j, a.T, a.left, a.right) ? ex2_approx(sv[e] * a.scale_log2 - lv[q0]) : 0.f;
                    const float p1 = bw_allowed(i + 1, j, a.T, a.left, a.right)
                                         ? ex2_approx(sv[e + 1] * a.scale_log2 - lv[q0 + 1])
                                         : 0.f;
                    pk[e / 2] = pack_bf16x2(p0, p1);
                    dk16[e / 2] = pack_bf16x2(p0 * (dp[e] - lv[BW_T + q0]), p1 * (dp[e + 1] - lv[BW_T + q0 + 1]));
                }
                tmem_st16u(tmem + lane_off + cc * 16, pk);
                tmem_st16u(tmem + lane_off + 128 + cc * 16, dk16);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->p_full[0]);
        }
        // ---- epilogue: dK * scale, dV -> bf16 ----
        // (the TMEM loads are warp-wide: every lane takes part, keys past T
        // only skip their stores)
        if (ok) ok = warp_wait_bounded(&bars->done, 0, ctl);
        {
            const long long row = ((long long)b * a.T + j) * a.Hkv + hk;
            __nv_bfloat16 *dkr = static_cast<__nv_bfloat16 *>(a.dk) + row * D;
            __nv_bfloat16 *dvr = static_cast<__nv_bfloat16 *>(a.dv) + row * D;
            if (ok && nsteps > 0) {
                tc_fence_after();
#pragma unroll 1
                for (int x = 0; x < 2; ++x) {
                    __nv_bfloat16 *dst = x ? dkr : dvr;
                    const float f = x ? a.scale : 1.f;
#pragma unroll 1
                    for (int cc = 0; cc < D / 16; ++cc) {
                        float v[16];
                        tmem_ld16(tmem + lane_off + 256 + x * D + cc * 16, v);
                        tmem_ld_wait_dep16(v);
                        if (j < a.T) {
                            uint4 u0, u1;
                            u0.x = pack_bf16x2(v[0] * f, v[1] * f);
                            u0.y = pack_bf16x2(v[2] * f, v[3] * f);
                            u0.z = pack_bf16x2(v[4] * f, v[5] * f);
                            u0.w = pack_bf16x2(v[6] * f, v[7] * f);
                            u1.x = pack_bf16x2(v[8] * f, v[9] * f);
                            u1.y = pack_bf16x2(v[10] * f, v[11] * f);
                            u1.z = pack_bf16x2(v[12] * f, v[13] * f);
                            u1.w = pack_bf16x2(v[14] * f, v[15] * f);
                            reinterpret_cast<uint4 *>(dst + cc * 16)[0] = u0;
                            reinterpret_cast<uint4 *>(dst + cc * 16)[1] = u1;
                        }
                        __syncwarp();
                    }
                }
            } else if (j < a.T) {
                // no query row sees this key, or the CTA aborted
                for (int e = 0; e < D; e += 8) {
                    *reinterpret_cast<uint4 *>(dkr + e) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4 *>(dvr + e) = make_uint4(0, 0, 0, 0);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D>
cudaError_t launch_bwd_d(const BwdArgs &a, cudaStream_t s)
{
    using C = BCfg<D>;
    // more than half the SM's shared memory, so that a second CTA (which
    // would wait for the 512 TMEM columns this one holds) never shares the SM
    constexpr int SMEM_DQ = (6 * C::TILE + 256 + 1024) > 120 * 1024 ? (6 * C::TILE + 256 + 1024) : 120 * 1024;
    constexpr int SMEM_KV =
        (6 * C::TILE + 2048 + 256 + 1024) > 120 * 1024 ? (6 * C::TILE + 2048 + 256 + 1024) : 120 * 1024;
    static_assert(SMEM_KV <= 227 * 1024, "fits one CTA's shared memory");
    static_assert(2 * (SMEM_DQ + 1024) > 228 * 1024 && 2 * (SMEM_KV + 1024) > 228 * 1024, "one CTA per SM");
    CUtensorMap mq, mk, mv, mdo;
    if (!make_bthd_map(&mq, a.q, a.B, a.T, a.Hq, D, BW_T) || !make_bthd_map(&mk, a.k, a.B, a.T, a.Hkv, D, BW_T) ||
        !make_bthd_map(&mv, a.v, a.B, a.T, a.Hkv, D, BW_T) || !make_bthd_map(&mdo, a.dout, a.B, a.T, a.Hq, D, BW_T))
        return cudaErrorInvalidValue;
    static DeviceOnce once;
    cudaError_t e = once.get(
        [&](int) {
            cudaError_t r = cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_DQ);
            if (r != cudaSuccess) return r;
            return cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_KV);
        },
        nullptr);
    if (e != cudaSuccess) return e;
    const long long rows = (long long)a.B * a.T * a.Hq;
    const long long rows_per_block = 8LL * (32 / (D / 8)) * BW_DPASS;
    bwd_delta_kernel<D><<<(unsigned)((rows + rows_per_block - 1) / rows_per_block), 256, 0, s>>>(
                                                                   static_cast<const __nv_bfloat16 *>(a.dout),
                                                                   static_cast<const __nv_bfloat16 *>(a.o), a.delta,
                                                                   a.B, a.T, a.Hq);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int nt = (a.T + BW_T - 1) / BW_T;
    bwd_dq_kernel<D><<<dim3(nt, a.Hq, a.B), BW_THREADS, SMEM_DQ, s>>>(mq, mk, mv, mdo, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    bwd_dkdv_kernel<D><<<dim3(nt, a.Hkv, a.B), BW_THREADS, SMEM_KV, s>>>(mq, mk, mv, mdo, a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_backward(int d, const BwdArgs &a, cudaStream_t s)
{
    if (d == 128) return launch_bwd_d<128>(a, s);
    if (d == 64) return launch_bwd_d<64>(a, s);
    return cudaErrorInvalidValue;
}

}  // namespace swa
