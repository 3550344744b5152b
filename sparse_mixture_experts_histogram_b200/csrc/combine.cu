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

namespace moe {

namespace {

constexpr int kCombineWarps = 8;

struct CombineParams {
    int T, d, k;
    const float4 *y;
    const int32_t *row_of_slot;
    const float *w;
    const float4 *shared_y;
    float4 *out;
};

__global__ void __launch_bounds__(32 * kCombineWarps) combine_kernel(const CombineParams p)
{
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
    if (t >= p.T) return;
    int my_row = -1;
    float my_w = 0.0f;
    if (lane < p.k) {
        my_row = p.row_of_slot[static_cast<size_t>(t) * p.k + lane];
        my_w = p.w[static_cast<size_t>(t) * p.k + lane];
        if (my_row >= p.T * p.k) my_row = -1;  // rows live in [0, T*k)
    }
    int rows[kMaxK];
    float ws[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
        rows[j] = __shfl_sync(0xffffffffu, my_row, j);
        ws[j] = __shfl_sync(0xffffffffu, my_w, j);
    }
    const int nv = p.d >> 2;
    for (int v = lane; v < nv; v += 32) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
            if (j < p.k && rows[j] >= 0) {
                const float4 y = __ldg(p.y + static_cast<size_t>(rows[j]) * nv + v);
                acc.x = fmaf(ws[j], y.x, acc.x);
                acc.y = fmaf(ws[j], y.y, acc.y);
                acc.z = fmaf(ws[j], y.z, acc.z);
                acc.w = fmaf(ws[j], y.w, acc.w);
            }
        }
        if (p.shared_y != nullptr) {
            const float4 s = __ldg(p.shared_y + static_cast<size_t>(t) * nv + v);
            acc.x += s.x;
            acc.y += s.y;
            acc.z += s.z;
            acc.w += s.w;
        }
        p.out[static_cast<size_t>(t) * nv + v] = acc;
    }
}

}  // namespace

cudaError_t launch_combine(const CombineLaunch &a, cudaStream_t s)
{
    CombineParams p;
    p.T = a.T;
    p.d = a.d;
    p.k = a.k;
    p.y = reinterpret_cast<const float4 *>(a.y);
    p.row_of_slot = a.row_of_slot;
    p.w = a.w;
    p.shared_y = reinterpret_cast<const float4 *>(a.shared_y);
    p.out = reinterpret_cast<float4 *>(a.out);
    const int blocks = (a.T + kCombineWarps - 1) / kCombineWarps;
    combine_kernel<<<blocks, 32 * kCombineWarps, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace moe
