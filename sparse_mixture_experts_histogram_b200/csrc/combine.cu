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
    size_t part_stride;  // 4-element vectors between consecutive partial outputs
    const void *y;       // fp32 rows, or bf16 rows (kernel template)
    const int32_t *row_of_slot;
    const int32_t *idx, *slot_pos, *offsets;  // used when row_of_slot is null
    const float *w;
    const void *shared_y;  // fp32 or bf16 rows (kernel template), or nullptr
    float4 *out;
    int chunks;          // chunks of 32*kCombineVec float4 per row
};

// Four consecutive elements (vector i of 4) of an fp32 or a bf16 array.
template <bool BF16>
__device__ __forceinline__ float4 load4(const void *base, size_t i)
{
    if constexpr (BF16) {
        const uint2 u = __ldg(reinterpret_cast<const uint2 *>(base) + i);
        return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                           __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
    } else {
        return __ldg(reinterpret_cast<const float4 *>(base) + i);
    }
}

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
// kCombineBatch pairs are issued before any of them is used.  SB: shared_y
// holds bf16 rows (the CTA-pair expert kernel's output) instead of fp32 ones.
template <bool SB>
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
            const size_t src = q * p.part_stride + static_cast<size_t>(ok ? row : 0) * nv;
#pragma unroll
            for (int u = 0; u < kCombineVec; ++u) {
                const int v = (c * kCombineVec + u) * 32 + lane;
                val[i][u] = (ok && v < nv) ? load4<false>(p.y, src + v) : make_float4(0.f, 0.f, 0.f, 0.f);
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
            if (p.shared_y != nullptr) add4(acc[u], load4<SB>(p.shared_y, static_cast<size_t>(t) * nv + v));
            p.out[static_cast<size_t>(t) * nv + v] = acc[u];
        }
    }
}

// The same combine over bf16 rows of y (complete sums: no K split): one
// warp per (token, chunk of 32*kCombineVec 8-element vectors).  Each lane
// loads 16 bytes per slot and vector, kept packed until used, so a warp has
// as many bytes in flight as the fp32 kernel with half the warps.  The
// arithmetic is the fp32 kernel's: acc = fma(w_j, y_j, acc) in slot order,
// then + shared_y.
__device__ __forceinline__ void fma8(float (&acc)[8], float w, const uint4 &v)
{
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] = fmaf(w, __uint_as_float(u[i] << 16), acc[2 * i]);
        acc[2 * i + 1] = fmaf(w, __uint_as_float(u[i] & 0xffff0000u), acc[2 * i + 1]);
    }
}

template <bool SB>
__global__ void __launch_bounds__(32 * kCombineWarps) combine_bf16_kernel(const CombineParams p)
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
        my_row = p.row_of_slot[sl];
        my_w = p.w[sl];
        if (my_row >= p.T * p.k) my_row = -1;  // rows live in [0, T*k)
    }
    const int n8 = p.d >> 3;
    const uint4 *y = static_cast<const uint4 *>(p.y);
    float acc[kCombineVec][8];
#pragma unroll
    for (int u = 0; u < kCombineVec; ++u)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[u][e] = 0.0f;
    for (int j0 = 0; j0 < p.k; j0 += kCombineBatch) {
        uint4 val[kCombineBatch][kCombineVec];
#pragma unroll
        for (int i = 0; i < kCombineBatch; ++i) {
            const int j = j0 + i;
            const int row = __shfl_sync(0xffffffffu, my_row, j & 31);
            const bool ok = j < p.k && row >= 0;
            const uint4 *src = y + static_cast<size_t>(ok ? row : 0) * n8;
#pragma unroll
            for (int u = 0; u < kCombineVec; ++u) {
                const int v = (c * kCombineVec + u) * 32 + lane;
                val[i][u] = (ok && v < n8) ? __ldg(src + v) : make_uint4(0u, 0u, 0u, 0u);
            }
        }
#pragma unroll
        for (int i = 0; i < kCombineBatch; ++i) {
            const int j = j0 + i;
            if (j < p.k) {
                const float wj = __shfl_sync(0xffffffffu, my_w, j & 31);
#pragma unroll
                for (int u = 0; u < kCombineVec; ++u) fma8(acc[u], wj, val[i][u]);
            }
        }
    }
#pragma unroll
    for (int u = 0; u < kCombineVec; ++u) {
        const int v = (c * kCombineVec + u) * 32 + lane;
        if (v < n8) {
            float4 lo = make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
            float4 hi = make_float4(acc[u][4], acc[u][5], acc[u][6], acc[u][7]);
            if (p.shared_y != nullptr) {
                const size_t i4 = static_cast<size_t>(t) * (2 * n8) + 2 * v;
                add4(lo, load4<SB>(p.shared_y, i4));
                add4(hi, load4<SB>(p.shared_y, i4 + 1));
            }
            float4 *o = p.out + static_cast<size_t>(t) * (2 * n8) + 2 * v;
            o[0] = lo;
            o[1] = hi;
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
    p.y = a.y;
    p.row_of_slot = a.row_of_slot;
    p.idx = a.idx;
    p.slot_pos = a.slot_pos;
    p.offsets = a.offsets;
    p.w = a.w;
    p.shared_y = a.shared_y;
    p.out = reinterpret_cast<float4 *>(a.out);
    p.ksplit = a.ksplit < 1 ? 1 : a.ksplit;
    p.ksplit_dev = a.ksplit_dev;
    p.part_stride = static_cast<size_t>(a.T) * a.k * (a.d / 4);
    const int nv = a.d / 4;
    p.chunks = (nv + 32 * kCombineVec - 1) / (32 * kCombineVec);
    const long long warps = static_cast<long long>(a.T) * p.chunks;
    const int blocks = static_cast<int>((warps + kCombineWarps - 1) / kCombineWarps);
    const dim3 b(32 * kCombineWarps);
    if (a.y_bf16) {
        // bf16 rows are complete sums, indexed through row_of_slot
        if (p.ksplit != 1 || p.ksplit_dev != nullptr || p.row_of_slot == nullptr)
            return cudaErrorInvalidValue;
        const int n8 = a.d / 8;
        p.chunks = (n8 + 32 * kCombineVec - 1) / (32 * kCombineVec);
        const long long w8 = static_cast<long long>(a.T) * p.chunks;
        const dim3 g(static_cast<unsigned>((w8 + kCombineWarps - 1) / kCombineWarps));
        return a.shared_bf16 ? launch_pdl(combine_bf16_kernel<true>, g, b, 0, s, a.pdl, p)
                             : launch_pdl(combine_bf16_kernel<false>, g, b, 0, s, a.pdl, p);
    }
    const dim3 g(blocks);
    return a.shared_bf16 ? launch_pdl(combine_kernel<true>, g, b, 0, s, a.pdl, p)
                         : launch_pdl(combine_kernel<false>, g, b, 0, s, a.pdl, p);
}

}  // namespace moe
