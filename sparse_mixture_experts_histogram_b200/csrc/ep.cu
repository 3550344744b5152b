// ep.cu -- expert parallelism: the E experts are split in contiguous blocks
// of E/R over R ranks (one GPU each); every (token, slot) row travels to the
// rank that owns its expert, and the expert's output row travels back.
//
//  * ep_ranks_plan_kernel: the stable ranks of this rank's (token, slot)
//    pairs per expert (as the single-GPU dispatch), then, in the CTA that
//    completes the expert offsets, the plan: from every rank's per-expert
//    pair counts (all-gathered by the caller into counts_all[R, E]) the first
//    receive row of each (expert, this source rank) block in its owner's
//    buffer, and this rank's own receive segments (its experts' offsets).
//  * ep_dispatch_kernel: x[t] is stored straight into the owner's receive
//    buffer (peer memory over NVLink when the owner is another GPU) at the
//    block's first row + the pair's rank in token order.  The scatter of the
//    single-GPU layer and the all-to-all of rows are one pass over x.
//  * ep_combine_kernel: each slot's expert output row is loaded from its
//    owner's output buffer (peer memory; bf16 rows where the owner's expert
//    kernel wrote complete sums, which halves what crosses NVLink on the way
//    back) and the k rows are summed, gate-weighted, in slot order.
//
// Receive layout on owner q: its experts in index order; inside an expert,
// the rows sent by rank 0, then rank 1, ...; inside one sender, token order.
// Every row's place follows from the routing alone, so the result does not
// depend on timing or on which rank finishes first.
//
// Method: the placement of experts on several GPUs ("Mistral 8x7B SMoE
// architecture", jsqmd.com, problem 4 of the deployment section: experts
// assigned to GPUs by hand to even out memory and load); the per-expert
// gathering and weighted index_add of "MoE" (theaiera.top, LLMs-from-scratch
// ch.10) sec. 10.4, done across ranks.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace moe {

namespace {

constexpr int kMaxRanks = 8;          // ranks of one expert-parallel group
constexpr uint32_t kErrEpCounts = 0x40u;  // MOE_DEVERR_EP_COUNTS

struct RanksPlanParams {
    int T, E, k, R, rank, El;
    int recv_rows;               // rows of every rank's receive buffer
    const int32_t *idx;          // [T, k] this rank's routing
    const int32_t *counts_all;   // [R, E]
    DispatchOut dout;            // per-tile ranks and this rank's expert offsets
    int32_t *base;               // [E] out: first receive row of (expert e, this rank)
    int32_t *recv_offsets;       // [El+1] out: this rank's receive segments
    uint32_t *ok;                // out: 1 when the counts are consistent
    uint32_t *err;
};

// The receive plan, run by the CTA that finished the expert offsets (all
// kTileTokens threads; E <= kMaxE).  For every expert e (owner q = e / El):
//   colsum[e] = sum_r counts_all[r, e]          (rows the owner gets for e)
//   seg[e]    = sum of colsum over q's experts before e (e's segment start)
//   base[e]   = seg[e] + sum_{r < rank} counts_all[r, e]
// and this rank's own segment starts.  Checks: this rank's row of
// counts_all equals the counts of its own idx (offs), no count is negative,
// and no owner receives more than recv_rows rows.
__device__ void ep_plan(const RanksPlanParams &p, const int32_t *offs, int32_t *colsum,
                        int32_t *excl, int *bad)
{
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    if (tid == 0) *bad = 0;
    __syncthreads();
    for (int e = tid; e < p.E; e += kTileTokens) {
        int c = 0;
        bool b = false;
        for (int r = 0; r < p.R; ++r) {
            const int v = p.counts_all[static_cast<size_t>(r) * p.E + e];
            b |= v < 0;
            c += v;
        }
        b |= p.counts_all[static_cast<size_t>(p.rank) * p.E + e] != offs[e + 1] - offs[e];
        colsum[e] = c;
        if (b) atomicOr(bad, 1);
    }
    __syncthreads();
    // Exclusive scan of colsum by the first warp (per-lane runs of experts).
    if (tid < 32) {
        const int per = (p.E + 31) >> 5;
        const int first = lane * per;
        int local = 0;
        for (int i = 0; i < per; ++i)
            if (first + i < p.E) local += colsum[first + i];
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        int run = incl - local;
        for (int i = 0; i < per; ++i) {
            if (first + i < p.E) {
                excl[first + i] = run;
                run += colsum[first + i];
            }
        }
        if (lane == 31) excl[p.E] = incl;
    }
    __syncthreads();
    for (int e = tid; e < p.E; e += kTileTokens) {
        int below = 0;
        for (int r = 0; r < p.rank; ++r) below += p.counts_all[static_cast<size_t>(r) * p.E + e];
        p.base[e] = excl[e] - excl[(e / p.El) * p.El] + below;
    }
    for (int q = tid; q < p.R; q += kTileTokens)
        if (excl[(q + 1) * p.El] - excl[q * p.El] > p.recv_rows) atomicOr(bad, 1);
    const int q0 = p.rank * p.El;
    for (int i = tid; i <= p.El; i += kTileTokens) p.recv_offsets[i] = excl[q0 + i] - excl[q0];
    __syncthreads();
    if (tid == 0) {
        *p.ok = *bad ? 0u : 1u;
        if (*bad) atomicOr(p.err, kErrEpCounts);
    }
}

// Per 128-token tile: the expert histogram and stable ranks of idx (as the
// single-GPU dispatch), and, in the CTA that completes the expert offsets,
// the receive plan.
__global__ void __launch_bounds__(kTileTokens) ep_ranks_plan_kernel(
    const __grid_constant__ RanksPlanParams p)
{
    __shared__ DispatchSmem ds;
    __shared__ int32_t colsum[kMaxE];
    __shared__ int32_t excl[kMaxE + 1];
    __shared__ int bad;
    ptx::grid_dep_launch();
    const int row = threadIdx.x;
    const int tile = blockIdx.x;
    const int t = tile * kTileTokens + row;
    for (int j = 0; j < kMaxK; ++j) {
        int e = -1;
        if (t < p.T && j < p.k) {
            e = p.idx[static_cast<size_t>(t) * p.k + j];
            bool b = (e < 0 || e >= p.E);
            for (int jj = 0; jj < j; ++jj) b |= (ds.sel[row][jj] == e);  // repeated expert
            if (b) {
                atomicOr(p.err, kErrIndex);
                e = -1;
            }
        }
        ds.sel[row][j] = e;
    }
    dispatch_tile(ds, row, tile, p.T, p.E, p.k, p.dout, 1);
    // Only the CTA that wrote the offsets goes on (the only one when there
    // is a single tile).
    if (p.dout.ntiles > 1 && !ds.is_last) return;
    __syncthreads();
    __threadfence();
    ep_plan(p, p.dout.offsets, colsum, excl, &bad);
}

struct EpDispatchParams {
    int T, d, E, k, El, R;
    int recv_rows;
    const uint4 *x;
    const int32_t *idx, *rank, *tilebase, *offsets, *base;
    const uint32_t *ok;
    uint4 *recv[kMaxRanks];  // every rank's receive buffer [recv_rows, d] bf16
    int32_t *pos_of_slot;    // [T, k] out
    uint32_t *err;
    int chunks;              // 16-byte-vector chunks of kEpVec*32 per row
};

constexpr int kEpWarps = 8;
constexpr int kEpVec = 4;  // 16-byte vectors per lane per chunk

// The receive buffer of owner q, picked with constant indices so that the
// pointer table stays in the parameter space.
template <typename P>
__device__ __forceinline__ P pick_rank(P const (&tab)[kMaxRanks], int q)
{
    P r = tab[0];
#pragma unroll
    for (int i = 1; i < kMaxRanks; ++i)
        if (q == i) r = tab[i];
    return r;
}

// One warp per (token, chunk of 32*kEpVec 16-byte vectors), as the
// single-GPU scatter: lanes 0..k-1 find the destination (owner, row) of the
// token's slots, every lane loads its vectors of x once and stores them to
// the k destinations.
__global__ void __launch_bounds__(32 * kEpWarps) ep_dispatch_kernel(const __grid_constant__ EpDispatchParams p)
{
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * kEpWarps + (threadIdx.x >> 5);
    const int t = gw / p.chunks;
    const int c = gw - t * p.chunks;
    if (t >= p.T) return;
    // x and idx were written before the plan kernel started, so they are
    // read while it finishes; everything it writes is read after the wait.
    const int nv = p.d >> 3;
    const uint4 *src = p.x + static_cast<size_t>(t) * nv;
    uint4 val[kEpVec];
#pragma unroll
    for (int u = 0; u < kEpVec; ++u) {
        const int v = (c * kEpVec + u) * 32 + lane;
        if (v < nv) val[u] = __ldg(src + v);
    }
    const size_t s = static_cast<size_t>(t) * p.k + lane;
    const int e = lane < p.k ? p.idx[s] : -1;
    ptx::grid_dep_wait();  // the ranks and the plan of ep_ranks_plan_kernel
    const bool ok = *p.ok != 0u;  // inconsistent counts: nothing is sent
    int my_pos = -1, my_q = 0;
    if (lane < p.k && ok) {
        const int r = p.rank[s];
        if (e >= 0 && e < p.E && r >= 0) {
            const int row = p.tilebase[static_cast<size_t>(t / kTileTokens) * p.E + e] + r;
            const int pos = p.base[e] + (row - p.offsets[e]);
            if (pos >= 0 && pos < p.recv_rows) {
                my_pos = pos;
                my_q = e / p.El;
            }
        }
        if (c == 0) {
            if (my_pos < 0) atomicOr(p.err, kErrIndex);
            p.pos_of_slot[s] = my_pos;
        }
    } else if (lane < p.k && c == 0) {
        p.pos_of_slot[s] = -1;
    }
    if (!ok) return;
    bool stored = false;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
        const int pos = __shfl_sync(0xffffffffu, my_pos, j);
        const int q = __shfl_sync(0xffffffffu, my_q, j);
        if (j < p.k && pos >= 0) {
            uint4 *dst = pick_rank(p.recv, q) + static_cast<size_t>(pos) * nv;
#pragma unroll
            for (int u = 0; u < kEpVec; ++u) {
                const int v = (c * kEpVec + u) * 32 + lane;
                if (v < nv) dst[v] = val[u];
            }
            stored = true;
        }
    }
    // Stores to another GPU's memory are made visible system-wide before the
    // kernel ends; the caller's collective that follows orders them before
    // the owner's expert kernel.
    if (stored) __threadfence_system();
}

struct EpCombineParams {
    int T, d, E, k, El;
    int ksplit;              // partial outputs per receive row, summed in order
    size_t part_stride;      // 4-element vectors between partial outputs (recv_rows * d / 4)
    int recv_rows;
    const int32_t *idx, *pos_of_slot;
    const float *w;
    const void *y[kMaxRanks];    // every rank's output buffer [ksplit, recv_rows, d], fp32
                                 // or bf16 (kernel template; ksplit 1)
    const float4 *shared_y;      // [T, d] or nullptr
    float4 *out;
    int chunks;              // chunks of 32*kEpOutVec float4 per row
};

constexpr int kEpOutVec = 2;
constexpr int kEpBatch = 4;  // (slot, partial) rows whose loads are in flight together

// Four consecutive elements (group i of 4) of an fp32 or a bf16 array.
template <bool BF>
__device__ __forceinline__ float4 load_y4(const void *base, size_t i)
{
    if constexpr (BF) {
        const uint2 u = __ldg(reinterpret_cast<const uint2 *>(base) + i);
        return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                           __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
    } else {
        return __ldg(reinterpret_cast<const float4 *>(base) + i);
    }
}

// One warp per (token, chunk): y_j = sum of the K-split partials of slot j's
// row (in order), out = sum_j w_j * y_j in slot order (+ shared_y).  The
// (slot, partial) pairs are visited slot-major in batches of kEpBatch whose
// loads are all issued before any is used; the order of every addition is
// fixed.
template <bool BF>
__global__ void __launch_bounds__(32 * kEpWarps) ep_combine_kernel(const __grid_constant__ EpCombineParams p)
{
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * kEpWarps + (threadIdx.x >> 5);
    const int t = gw / p.chunks;
    const int c = gw - t * p.chunks;
    if (t >= p.T) return;
    int my_pos = -1, my_q = 0;
    float my_w = 0.0f;
    if (lane < p.k) {
        const size_t s = static_cast<size_t>(t) * p.k + lane;
        const int e = p.idx[s];
        const int pos = p.pos_of_slot[s];
        if (e >= 0 && e < p.E && pos >= 0 && pos < p.recv_rows) {
            my_pos = pos;
            my_q = e / p.El;
        }
        my_w = p.w[s];
    }
    const int nv = p.d >> 2;
    const int npairs = p.k * p.ksplit;
    float4 acc[kEpOutVec], yj[kEpOutVec];
#pragma unroll
    for (int u = 0; u < kEpOutVec; ++u) {
        acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        yj[u] = acc[u];
    }
    // (j0, sp0): slot and partial of the batch's first pair, advanced
    // without divisions.
    int j0 = 0, sp0 = 0;
    for (int p0 = 0; p0 < npairs; p0 += kEpBatch) {
        float4 val[kEpBatch][kEpOutVec];
        int jj[kEpBatch], ss[kEpBatch];
        {
            int j = j0, sp = sp0;
#pragma unroll
            for (int i = 0; i < kEpBatch; ++i) {
                jj[i] = j;
                ss[i] = sp;
                if (++sp == p.ksplit) {
                    sp = 0;
                    ++j;
                }
            }
            j0 = j;
            sp0 = sp;
        }
#pragma unroll
        for (int i = 0; i < kEpBatch; ++i) {
            const int pi = p0 + i;
            const int pos = __shfl_sync(0xffffffffu, my_pos, jj[i] & 31);
            const int q = __shfl_sync(0xffffffffu, my_q, jj[i] & 31);
            const bool ok = pi < npairs && pos >= 0;
            const void *yq = pick_rank(p.y, q);
            const size_t row = ss[i] * p.part_stride + static_cast<size_t>(ok ? pos : 0) * nv;
#pragma unroll
            for (int u = 0; u < kEpOutVec; ++u) {
                const int v = (c * kEpOutVec + u) * 32 + lane;
                val[i][u] = (ok && v < nv) ? load_y4<BF>(yq, row + v) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int i = 0; i < kEpBatch; ++i) {
            const int pi = p0 + i;
            if (pi < npairs) {
                const int j = jj[i];
                const int sp = ss[i];
#pragma unroll
                for (int u = 0; u < kEpOutVec; ++u) {
                    if (sp == 0) {
                        yj[u] = val[i][u];
                    } else {
                        yj[u].x += val[i][u].x;
                        yj[u].y += val[i][u].y;
                        yj[u].z += val[i][u].z;
                        yj[u].w += val[i][u].w;
                    }
                }
                if (sp == p.ksplit - 1) {
                    const float wj = __shfl_sync(0xffffffffu, my_w, j & 31);
#pragma unroll
                    for (int u = 0; u < kEpOutVec; ++u) {
                        acc[u].x = fmaf(wj, yj[u].x, acc[u].x);
                        acc[u].y = fmaf(wj, yj[u].y, acc[u].y);
                        acc[u].z = fmaf(wj, yj[u].z, acc[u].z);
                        acc[u].w = fmaf(wj, yj[u].w, acc[u].w);
                    }
                }
            }
        }
    }
#pragma unroll
    for (int u = 0; u < kEpOutVec; ++u) {
        const int v = (c * kEpOutVec + u) * 32 + lane;
        if (v < nv) {
            if (p.shared_y != nullptr) {
                const float4 b = p.shared_y[static_cast<size_t>(t) * nv + v];
                acc[u].x += b.x;
                acc[u].y += b.y;
                acc[u].z += b.z;
                acc[u].w += b.w;
            }
            p.out[static_cast<size_t>(t) * nv + v] = acc[u];
        }
    }
}

}  // namespace

cudaError_t launch_ep_dispatch(const EpDispatchLaunch &a, cudaStream_t s)
{
    if (a.R < 1 || a.R > kMaxRanks || a.E % a.R != 0 || a.E > kMaxE) return cudaErrorInvalidValue;
    RanksPlanParams pp{};
    pp.T = a.T;
    pp.E = a.E;
    pp.k = a.k;
    pp.R = a.R;
    pp.rank = a.rank;
    pp.El = a.E / a.R;
    pp.recv_rows = a.recv_rows;
    pp.idx = a.idx;
    pp.counts_all = a.counts_all;
    pp.dout.tilecnt = a.tilecnt;
    pp.dout.tilebase = a.tilebase;
    pp.dout.rank = a.rank_of_pair;
    pp.dout.offsets = a.offsets;
    pp.dout.counts = nullptr;
    pp.dout.done = a.done;
    // T = 0: one CTA with no tokens still computes the plan (zero counts of
    // its own, the receive segments it owns).
    pp.dout.ntiles = a.T > 0 ? (a.T + kTileTokens - 1) / kTileTokens : 1;
    pp.dout.cap = -1;
    pp.base = a.base;
    pp.recv_offsets = a.recv_offsets;
    pp.ok = a.ok;
    pp.err = a.err;
    ep_ranks_plan_kernel<<<pp.dout.ntiles, kTileTokens, 0, s>>>(pp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || a.T == 0) return e;

    EpDispatchParams p{};
    p.T = a.T;
    p.d = a.d;
    p.E = a.E;
    p.k = a.k;
    p.El = pp.El;
    p.R = a.R;
    p.recv_rows = a.recv_rows;
    p.x = reinterpret_cast<const uint4 *>(a.x);
    p.idx = a.idx;
    p.rank = a.rank_of_pair;
    p.tilebase = a.tilebase;
    p.offsets = a.offsets;
    p.base = a.base;
    p.ok = a.ok;
    for (int r = 0; r < kMaxRanks; ++r)
        p.recv[r] = reinterpret_cast<uint4 *>(r < a.R ? a.recv_x[r] : a.recv_x[0]);
    p.pos_of_slot = a.pos_of_slot;
    p.err = a.err;
    const int nv = a.d / 8;
    p.chunks = (nv + 32 * kEpVec - 1) / (32 * kEpVec);
    const long long warps = static_cast<long long>(a.T) * p.chunks;
    const int blocks = static_cast<int>((warps + kEpWarps - 1) / kEpWarps);
    return launch_pdl(ep_dispatch_kernel, dim3(blocks), dim3(32 * kEpWarps), 0, s, true, p);
}

cudaError_t launch_ep_combine(const EpCombineLaunch &a, cudaStream_t s)
{
    if (a.R < 1 || a.R > kMaxRanks || a.E % a.R != 0) return cudaErrorInvalidValue;
    EpCombineParams p{};
    p.T = a.T;
    p.d = a.d;
    p.E = a.E;
    p.k = a.k;
    p.El = a.E / a.R;
    p.ksplit = a.ksplit < 1 ? 1 : a.ksplit;
    if (a.y_bf16 && p.ksplit != 1) return cudaErrorInvalidValue;
    p.recv_rows = a.recv_rows;
    p.part_stride = static_cast<size_t>(a.recv_rows) * (a.d / 4);
    p.idx = a.idx;
    p.pos_of_slot = a.pos_of_slot;
    p.w = a.w;
    for (int r = 0; r < kMaxRanks; ++r)
        p.y[r] = r < a.R ? a.recv_y[r] : a.recv_y[0];
    p.shared_y = reinterpret_cast<const float4 *>(a.shared_y);
    p.out = reinterpret_cast<float4 *>(a.out);
    const int nv = a.d / 4;
    p.chunks = (nv + 32 * kEpOutVec - 1) / (32 * kEpOutVec);
    const long long warps = static_cast<long long>(a.T) * p.chunks;
    const int blocks = static_cast<int>((warps + kEpWarps - 1) / kEpWarps);
    if (a.y_bf16) ep_combine_kernel<true><<<blocks, 32 * kEpWarps, 0, s>>>(p);
    else ep_combine_kernel<false><<<blocks, 32 * kEpWarps, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace moe
