// combine.cu -- gate-weighted un-permute: out[t] = sum_j w[t,j] *
// y[row_of_slot[t,j]] (+ shared_y[t]), summed in slot order j = 0..k-1, one
// warp per token with 16-byte vectors.  Each output element is written
// exactly once, so the result does not depend on scheduling.
//
// Method: "MoE" (theaiera.top, LLMs-from-scratch ch.10) sec. 10.4, the
// weighted index_add of each expert's output back to its tokens, and
// sec. 10.5, the shared expert's output added with weight 1.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace moe {

namespace {

constexpr int kCombineWarps = 8;
constexpr int kCombineVec = 2;   // float4 per lane per chunk
constexpr int kCombineBatch = 8; // (slot, partial) pairs whose loads are in flight together

struct CombineParams {
    int T, d, k;
    int ksplit;          // partial outputs per row, summed in order before weighting
    const int *ksplit_dev; // if set, the count is read here (written by the previous kernel)
    size_t part_stride;  // float4 between consecutive partial outputs
    const float4 *y;
    const int32_t *row_of_slot;
    const int32_t *idx, *slot_pos, *offsets;  // used when row_of_slot is null
    const float *w;
    const float4 *shared_y;
    float4 *out;
    int chunks;          // chunks of 32*kCombineVec float4 per row
};

__device__ __forceinline__ void add4(float4 &a, const float4 &b)
{
    a.x += b.x;
    a.y += b.y;
    a.z += b.z;
    a.w += b.w;
}

// One warp per (token, chunk of 32*kCombineVec float4).  The (slot j,
// partial q) pairs are visited j-major: y_j = sum_q partial_q(row_j), then
// acc += w_j * y_j, so the order of every addition is fixed.  Loads of
// kCombineBatch pairs are issued before any of them is used.
__global__ void __launch_bounds__(32 * kCombineWarps) combine_kernel(const CombineParams p)
{
    ptx::grid_dep_launch();
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
    const int t = gw / p.chunks;
    const int c = gw - t * p.chunks;
    if (t >= p.T) return;
    ptx::grid_dep_wait();
    int my_row = -1;
    float my_w = 0.0f;
    if (lane < p.k) {
        const size_t sl = static_cast<size_t>(t) * p.k + lane;
        if (p.row_of_slot) {
            my_row = p.row_of_slot[sl];
        } else {
            const int e = p.idx[sl];
            const int q = p.slot_pos[sl];
            my_row = (e >= 0 && q >= 0) ? p.offsets[e] + q : -1;
        }
        my_w = p.w[sl];
        if (my_row >= p.T * p.k) my_row = -1;  // rows live in [0, T*k)
    }
    const int nv = p.d >> 2;
    const int ksplit = p.ksplit_dev ? *p.ksplit_dev : p.ksplit;
    const int npairs = p.k * ksplit;
    float4 acc[kCombineVec], yj[kCombineVec];
#pragma unroll
    for (int u = 0; u < kCombineVec; ++u) {
        acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        yj[u] = acc[u];
    }
    for (int p0 = 0; p0 < npairs; p0 += kCombineBatch) {
        float4 val[kCombineBatch][kCombineVec];
#pragma unroll
        for (int i = 0; i < kCombineBatch; ++i) {
            const int pi = p0 + i;
            const int j = pi / ksplit;
            const int q = pi - j * ksplit;
            const int row = __shfl_sync(0xffffffffu, my_row, j & 31);
            const bool ok = pi < npairs && row >= 0;
            const float4 *src = p.y + q * p.part_stride + static_cast<size_t>(ok ? row : 0) * nv;
#pragma unroll
            for (int u = 0; u < kCombineVec; ++u) {
                const int v = (c * kCombineVec + u) * 32 + lane;
                val[i][u] = (ok && v < nv) ? __ldg(src + v) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int i = 0; i < kCombineBatch; ++i) {
            const int pi = p0 + i;
            if (pi < npairs) {
                const int j = pi / ksplit;
                const int q = pi - j * ksplit;
#pragma unroll
                for (int u = 0; u < kCombineVec; ++u) {
                    if (q == 0) yj[u] = val[i][u];
                    else add4(yj[u], val[i][u]);
                }
                if (q == ksplit - 1) {
                    const float wj = __shfl_sync(0xffffffffu, my_w, j & 31);
#pragma unroll
                    for (int u = 0; u < kCombineVec; ++u) {
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
    for (int u = 0; u < kCombineVec; ++u) {
        const int v = (c * kCombineVec + u) * 32 + lane;
        if (v < nv) {
            if (p.shared_y != nullptr) add4(acc[u], __ldg(p.shared_y + static_cast<size_t>(t) * nv + v));
            p.out[static_cast<size_t>(t) * nv + v] = acc[u];
        }
    }
}

}  // namespace

cudaError_t launch_combine(const CombineLaunch &a, cudaStream_t s)
{
    CombineParams p{};
    p.T = a.T;
    p.d = a.d;
    p.k = a.k;
    p.y = reinterpret_cast<const float4 *>(a.y);
    p.row_of_slot = a.row_of_slot;
    p.idx = a.idx;
    p.slot_pos = a.slot_pos;
    p.offsets = a.offsets;
    p.w = a.w;
    p.shared_y = reinterpret_cast<const float4 *>(a.shared_y);
    p.out = reinterpret_cast<float4 *>(a.out);
    p.ksplit = a.ksplit < 1 ? 1 : a.ksplit;
    p.ksplit_dev = a.ksplit_dev;
    p.part_stride = static_cast<size_t>(a.T) * a.k * (a.d / 4);
    const int nv = a.d / 4;
    p.chunks = (nv + 32 * kCombineVec - 1) / (32 * kCombineVec);
    const long long warps = static_cast<long long>(a.T) * p.chunks;
    const int blocks = static_cast<int>((warps + kCombineWarps - 1) / kCombineWarps);
    return launch_pdl(combine_kernel, dim3(blocks), dim3(32 * kCombineWarps), 0, s, a.pdl, p);
}

}  // namespace moe
