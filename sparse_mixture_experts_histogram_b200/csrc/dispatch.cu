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
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

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
            bool bad = (e < 0 || e >= p.E);
            for (int jj = 0; jj < j; ++jj) bad |= (ds.sel[row][jj] == e);  // repeated expert
            if (bad) {
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
    int cap;             // per-expert capacity, or -1 (dropless)
    const int32_t *offsets;  // [E+1] segment starts (read when cap >= 0)
    const uint4 *x;
    const int32_t *idx, *rank, *tilebase;
    uint4 *x_perm;
    int32_t *row_of_slot;
    int32_t *slot_of_row;  // or nullptr
    float4 *out_zero;      // or nullptr
    uint32_t *err;
    int S;
    int allow_empty;  // expert -1 marks an unused slot (no row, no error)
    int to_f16;  // convert the rows to fp16 on the way
    int chunks;  // 16-byte-vector chunks of kScatterVec*32 per row
};

constexpr int kScatterWarps = 8;
constexpr int kScatterVec = 4;  // 16-byte vectors per lane per chunk

// One warp per (token, chunk of 32*kScatterVec 16-byte vectors): the rows of
// the token's k slots are computed by lanes 0..k-1 and broadcast, then each
// lane loads its kScatterVec vectors of x (independent loads in flight) and
// stores them to the k rows.
__global__ void __launch_bounds__(32 * kScatterWarps) scatter_kernel(const ScatterParams p)
{
    ptx::grid_dep_launch();
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * kScatterWarps + (threadIdx.x >> 5);
    const int t = gw / p.chunks;
    const int c = gw - t * p.chunks;
    if (t >= p.T) return;
    ptx::grid_dep_wait();
    int my_row = -1;
    if (lane < p.k) {
        const size_t s = static_cast<size_t>(t) * p.k + lane;
        const int e = p.idx[s];
        const int r = p.rank[s];
        bool dropped = p.allow_empty && e == -1;
        if (e >= 0 && e < p.E && r >= 0) {
            const int row = p.tilebase[static_cast<size_t>(t / kTileTokens) * p.E + e] + r;
            // With a capacity, a pair ranked at or beyond it in its expert's
            // token order is dropped: no row, nothing added for this slot.
            if (p.cap >= 0 && row - p.offsets[e] >= p.cap) dropped = true;
            else if (row >= 0 && row < p.S) my_row = row;
        }
        if (c == 0) {
            if (my_row < 0 && !dropped) atomicOr(p.err, kErrIndex);
            p.row_of_slot[s] = my_row;
            if (p.slot_of_row != nullptr && my_row >= 0) p.slot_of_row[my_row] = static_cast<int>(s);
        }
    }
    int rows[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) rows[j] = __shfl_sync(0xffffffffu, my_row, j);
    const int nv = p.d >> 3;  // 16-byte vectors per row
    const uint4 *src = p.x + static_cast<size_t>(t) * nv;
    uint4 val[kScatterVec];
#pragma unroll
    for (int u = 0; u < kScatterVec; ++u) {
        const int v = (c * kScatterVec + u) * 32 + lane;
        if (v < nv) val[u] = __ldg(src + v);
    }
    if (p.to_f16) {
#pragma unroll
        for (int u = 0; u < kScatterVec; ++u) {
            uint32_t *w = reinterpret_cast<uint32_t *>(&val[u]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float lo = __uint_as_float(w[i] << 16);
                const float hi = __uint_as_float(w[i] & 0xffff0000u);
                const __half2 h = __floats2half2_rn(lo, hi);
                w[i] = *reinterpret_cast<const uint32_t *>(&h);
            }
        }
    }
    if (p.out_zero != nullptr) {
        // The same columns of out (fp32: two 16-byte vectors per bf16 one).
        float4 *o = p.out_zero + static_cast<size_t>(t) * (2 * nv);
#pragma unroll
        for (int u = 0; u < kScatterVec; ++u) {
            const int v = (c * kScatterVec + u) * 32 + lane;
            if (v < nv) {
                o[2 * v] = make_float4(0.f, 0.f, 0.f, 0.f);
                o[2 * v + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
        if (j < p.k && rows[j] >= 0) {
            uint4 *dst = p.x_perm + static_cast<size_t>(rows[j]) * nv;
#pragma unroll
            for (int u = 0; u < kScatterVec; ++u) {
                const int v = (c * kScatterVec + u) * 32 + lane;
                if (v < nv) dst[v] = val[u];
            }
        }
    }
}

}  // namespace

cudaError_t launch_ranks(const RanksLaunch &a, cudaStream_t s)
{
    RanksParams p{};
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
    p.dout.cap = -1;
    ranks_kernel<<<p.dout.ntiles, kTileTokens, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_scatter(const ScatterLaunch &a, cudaStream_t s)
{
    ScatterParams p{};
    p.T = a.T;
    p.d = a.d;
    p.E = a.E;
    p.k = a.k;
    p.cap = a.cap;
    p.offsets = a.offsets;
    p.x = reinterpret_cast<const uint4 *>(a.x);
    p.idx = a.idx;
    p.rank = a.rank;
    p.tilebase = a.tilebase;
    p.x_perm = reinterpret_cast<uint4 *>(a.x_perm);
    p.row_of_slot = a.row_of_slot;
    p.slot_of_row = a.slot_of_row;
    p.out_zero = reinterpret_cast<float4 *>(a.out_zero);
    p.err = a.err;
    p.S = a.T * a.k;
    p.allow_empty = a.allow_empty ? 1 : 0;
    p.to_f16 = a.to_f16 ? 1 : 0;
    const int nv = a.d / 8;
    p.chunks = (nv + 32 * kScatterVec - 1) / (32 * kScatterVec);
    const long long warps = static_cast<long long>(a.T) * p.chunks;
    const int blocks = static_cast<int>((warps + kScatterWarps - 1) / kScatterWarps);
    return launch_pdl(scatter_kernel, dim3(blocks), dim3(32 * kScatterWarps), 0, s, a.pdl, p);
}

}  // namespace moe
