// Dilated window as a plain window on strided sub-sequences.
//
// A dilated window with dilation dil (aivaro.ru "How sliding window attention
// works in Mistral and Longformer", section 4.2: every dil-th token instead of
// all neighbours) only ever pairs positions with the same residue modulo dil,
// and within the residue class r the sub-sequence r, r+dil, r+2dil, ... sees
// exactly a plain window of the same width.  So the call permutes q, k and v
// into residue-major sub-sequences, runs the plain prefill kernels on them as
// a batch, and permutes o and lse back.  Residues below T mod dil have one
// row more than the others, so the sub-sequences form two groups of equal
// length each, launched separately (no padding rows, which a symmetric window
// would otherwise see).
#include <cuda_runtime.h>
#include <stdint.h>

#include "swa_internal.h"

namespace swa {
namespace {

// Rows of [B,T,H,row16 x 16 bytes] <-> group rows [B*n,L,H,...] where group
// sequence b*n + rr holds original positions r0 + rr + t*dil, t < L.
__global__ void dilate_rows_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst, DilateGroup g,
                                   int to_group)
{
    const long long units = (long long)g.B * g.n * g.L * g.H * g.row16;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < units;
         idx += (long long)gridDim.x * blockDim.x) {
        const int u = (int)(idx % g.row16);
        long long rest = idx / g.row16;
        const int h = (int)(rest % g.H);
        rest /= g.H;
        const int t = (int)(rest % g.L);
        rest /= g.L;
        const int rr = (int)(rest % g.n);
        const long long b = rest / g.n;
        const long long pos = g.r0 + rr + (long long)t * g.dil;
        const long long gi = idx;
        const long long oi = ((b * g.T + pos) * g.H + h) * g.row16 + u;
        if (to_group) dst[gi] = src[oi];
        else dst[oi] = src[gi];
    }
}

// lse: group [B*n,H,L] -> original [B,H,T]
__global__ void dilate_lse_kernel(const float *__restrict__ src, float *__restrict__ dst, DilateGroup g)
{
    const long long units = (long long)g.B * g.n * g.H * g.L;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < units;
         idx += (long long)gridDim.x * blockDim.x) {
        const int t = (int)(idx % g.L);
        long long rest = idx / g.L;
        const int h = (int)(rest % g.H);
        rest /= g.H;
        const int rr = (int)(rest % g.n);
        const long long b = rest / g.n;
        dst[(b * g.H + h) * g.T + g.r0 + rr + (long long)t * g.dil] = src[idx];
    }
}

int blocks_for(long long units)
{
    long long b = (units + 255) / 256;
    if (b < 1) b = 1;
    if (b > 148 * 32) b = 148 * 32;
    return (int)b;
}

}  // namespace

cudaError_t launch_dilate_rows(const void *src, void *dst, const DilateGroup &g, int to_group, cudaStream_t s)
{
    const long long units = (long long)g.B * g.n * g.L * g.H * g.row16;
    if (units == 0) return cudaSuccess;
    dilate_rows_kernel<<<blocks_for(units), 256, 0, s>>>(static_cast<const uint4 *>(src), static_cast<uint4 *>(dst),
                                                         g, to_group);
    return cudaGetLastError();
}

cudaError_t launch_dilate_lse(const float *src, float *dst, const DilateGroup &g, cudaStream_t s)
{
    const long long units = (long long)g.B * g.n * g.H * g.L;
    if (units == 0) return cudaSuccess;
    dilate_lse_kernel<<<blocks_for(units), 256, 0, s>>>(src, dst, g);
    return cudaGetLastError();
}

}  // namespace swa
