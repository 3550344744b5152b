// internal.h -- host-side launchers of the kernels (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace moe {

struct RouteLaunch {
    int T, d, E, k;
    const uint16_t *x;   // [T,d] bf16
    const uint16_t *Wg;  // [E,d] bf16
    const float *bias;   // [E] or nullptr
    int32_t *idx;        // [T,k]
    float *w;            // [T,k]
    int32_t *counts;     // [E] or nullptr
    int32_t *offsets;    // [E+1]
    int32_t *tilecnt;    // [ntiles,E]
    int32_t *tilebase;   // [ntiles,E]
    int32_t *rank;       // [T,k]
    uint32_t *done;      // counter, zero before the launch
    uint32_t *tile_ctr;  // [ntiles] counters, zero before the launch
    uint32_t *err;       // device error word
};

struct RanksLaunch {
    int T, E, k;
    const int32_t *idx;
    int32_t *offsets, *tilecnt, *tilebase, *rank;
    uint32_t *done, *err;
};

struct ScatterLaunch {
    int T, d, E, k;
    const uint16_t *x;
    const int32_t *idx, *rank, *tilebase;
    uint16_t *x_perm;
    int32_t *row_of_slot;
    uint32_t *err;
    bool pdl;  // launched right after another kernel of this library
};

struct GemmLaunch {
    int up;               // 1: H = silu(W1 x) * (W3 x) (bf16 out); 0: Y = W2 H (fp32 out)
    int E;                // experts (segments)
    int M_rows;           // weight rows per expert: d_ff (up) or d (down)
    int K;                // reduction length: d (up) or d_ff (down)
    int S;                // rows of the activation operand
    int max_rows;         // upper bound of rows in one segment (weights streamed once if <= tile)
    int ksplit;           // down only: K split into this many ranges, partial outputs
                          // [ksplit, S, M_rows] summed by the caller (the combine)
    const int32_t *offsets;   // [E+1] device, or nullptr for one segment [0, S)
    const uint16_t *A0, *A1;  // W1, W3 (up) or W2 (down, A1 unused)
    const uint16_t *B;        // x_perm (up) or H (down)
    void *out;                // H [S, M_rows] bf16 or Y [S, M_rows] fp32
    uint32_t *err;
    bool pdl;                 // launched right after another kernel of this library
};

struct CombineLaunch {
    int T, d, k;
    int ksplit;            // partial outputs per row of y, summed in order before weighting
    const float *y;        // [ksplit, T*k, d]
    const int32_t *row_of_slot;
    const float *w;
    const float *shared_y;
    float *out;
    bool pdl;                 // launched right after another kernel of this library
};

cudaError_t launch_route(const RouteLaunch &a, cudaStream_t s);
cudaError_t launch_ranks(const RanksLaunch &a, cudaStream_t s);
cudaError_t launch_scatter(const ScatterLaunch &a, cudaStream_t s);
cudaError_t launch_gemm(const GemmLaunch &a, cudaStream_t s);
int gemm_token_tile(int up, int S, int E_seg);
int down_ksplit(int S, int E_seg, int d, int d_ff);
cudaError_t launch_combine(const CombineLaunch &a, cudaStream_t s);

// Tensor maps (tensormap.cpp side, implemented in api.cu).
// 2-D bf16 row-major matrix [rows, cols] read in boxes of 64 columns (128 B,
// 128-byte swizzle) by box_rows rows.
cudaError_t make_tmap_bf16(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                           uint32_t box_rows);

int device_sm_count();

}  // namespace moe
