// dispatch.cu -- grouping of the (token, slot) pairs by expert.
//
//  * ranks_kernel: per 128-token tile, the expert histogram and stable ranks
//    of an idx[T,k] array given by the caller, and the expert offsets (the
//    routing kernel does the same inside its epilogue).
//  * scatter_kernel: x_perm[tilebase[tile,e] + rank[t,j]] = x[t], written as
//    16-byte vectors by one warp per token, plus row_of_slot[t,j].
//
// Method: "MoE" (theaiera.top, LLMs-from-scratch ch.10) sec. 10.4 gathers,
// per expert, the tokens that selected it (mask / nonzero / index_select);
// here every expert's tokens become one contiguous, token-ordered segment.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

struct RanksParams {
    int T, E, k;
    const int32_t *idx;
    uint32_t *err;
    DispatchOut dout;
};

__global__ void __launch_bounds__(kTileTokens) ranks_kernel(const RanksParams p)
{
    __shared__ DispatchSmem ds;
    const int row = threadIdx.x;
    const int tile = blockIdx.x;
    const int t = tile * kTileTokens + row;
    for (int j = 0; j < kMaxK; ++j) {
        int e = -1;
        if (t < p.T && j < p.k) {
            e = p.idx[static_cast<size_t>(t) * p.k + j];
            if (e < 0 || e >= p.E) {
                atomicOr(p.err, kErrIndex);
                e = -1;
            }
        }
        ds.sel[row][j] = e;
    }
    dispatch_tile(ds, row, tile, p.T, p.E, p.k, p.dout, 1);
}

struct ScatterParams {
    int T, d, E, k;
    const uint4 *x;
    const int32_t *idx, *rank, *tilebase;
    uint4 *x_perm;
    int32_t *row_of_slot;
    uint32_t *err;
    int S;
};

constexpr int kScatterWarps = 8;

__global__ void __launch_bounds__(32 * kScatterWarps) scatter_kernel(const ScatterParams p)
{
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * kScatterWarps + (threadIdx.x >> 5);
    if (t >= p.T) return;
    int my_row = -1;
    if (lane < p.k) {
        const size_t s = static_cast<size_t>(t) * p.k + lane;
        const int e = p.idx[s];
        const int r = p.rank[s];
        if (e >= 0 && e < p.E && r >= 0) {
            const int row = p.tilebase[static_cast<size_t>(t / kTileTokens) * p.E + e] + r;
            if (row >= 0 && row < p.S) my_row = row;
        }
        if (my_row < 0) atomicOr(p.err, kErrIndex);
        p.row_of_slot[s] = my_row;
    }
    int rows[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) rows[j] = __shfl_sync(0xffffffffu, my_row, j);
    const int nv = p.d >> 3;  // 16-byte vectors per row
    const uint4 *src = p.x + static_cast<size_t>(t) * nv;
    for (int v = lane; v < nv; v += 32) {
        const uint4 val = __ldg(src + v);
#pragma unroll
        for (int j = 0; j < kMaxK; ++j)
            if (j < p.k && rows[j] >= 0) p.x_perm[static_cast<size_t>(rows[j]) * nv + v] = val;
    }
}

}  // namespace

cudaError_t launch_ranks(const RanksLaunch &a, cudaStream_t s)
{
    RanksParams p;
    p.T = a.T;
    p.E = a.E;
    p.k = a.k;
    p.idx = a.idx;
    p.err = a.err;
    p.dout.tilecnt = a.tilecnt;
    p.dout.tilebase = a.tilebase;
    p.dout.rank = a.rank;
    p.dout.offsets = a.offsets;
    p.dout.counts = nullptr;
    p.dout.done = a.done;
    p.dout.ntiles = (a.T + kTileTokens - 1) / kTileTokens;
    ranks_kernel<<<p.dout.ntiles, kTileTokens, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_scatter(const ScatterLaunch &a, cudaStream_t s)
{
    ScatterParams p;
    p.T = a.T;
    p.d = a.d;
    p.E = a.E;
    p.k = a.k;
    p.x = reinterpret_cast<const uint4 *>(a.x);
    p.idx = a.idx;
    p.rank = a.rank;
    p.tilebase = a.tilebase;
    p.x_perm = reinterpret_cast<uint4 *>(a.x_perm);
    p.row_of_slot = a.row_of_slot;
    p.err = a.err;
    p.S = a.T * a.k;
    const int blocks = (a.T + kScatterWarps - 1) / kScatterWarps;
    scatter_kernel<<<blocks, 32 * kScatterWarps, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace moe
