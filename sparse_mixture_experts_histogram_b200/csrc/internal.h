// internal.h -- host-side launchers of the kernels (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace moe {

struct RouteLaunch {
    int T, d, E, k;
    int wmode;           // gate weights: 0 softmax over the selected, 1 softmax over all, 2 sigmoid,
                         // 3 tempered softmax over all with entropy-controlled k (slot K-1 may be -1)
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
    // Slot mode (slot_pos set): instead of the token-ordered tile histogram,
    // positions from atomics (common.cuh assign_slots), the token list of
    // every expert and the per-expert totals in gcnt; offsets, counts,
    // tilecnt, tilebase, rank, done and tile_ctr are not written.
    int32_t *slot_pos;   // [T,k]
    int32_t *perm;       // [E, perm_stride]
    int32_t *gcnt;       // [E] zero before the launch (left zero)
    int perm_stride;
    int cap;             // per-expert capacity of the token-ordered dispatch, or -1
};

struct RanksLaunch {
    int T, E, k;
    const int32_t *idx;
    int32_t *offsets, *tilecnt, *tilebase, *rank;
    uint32_t *done, *err;
};

struct ScatterLaunch {
    int T, d, E, k;
    int cap;                  // per-expert capacity, or -1 (dropless)
    const int32_t *offsets;   // [E+1] segment starts, needed when cap >= 0
    const uint16_t *x;
    const int32_t *idx, *rank, *tilebase;
    uint16_t *x_perm;
    int32_t *row_of_slot;
    uint32_t *err;
    bool pdl;  // launched right after another kernel of this library
    bool to_f16;  // write x_perm as fp16 (the FP8 expert path) instead of bf16
    bool allow_empty;  // idx -1 marks an unused slot (entropy-controlled k), not an error
    // For the expert kernel's weighted output (FfnLaunch::out), when set:
    // slot_of_row[row] = t*k + j for every row that got a slot, and out[T, d]
    // set to zero.
    int32_t *slot_of_row;
    float *out_zero;
};

struct FfnLaunch {
    int E;                    // segments (ignored when offsets is null: one segment [0, S))
    int d, d_ff;
    int S;                    // rows of x / H / Y
    int S_hint;               // rows expected (0: S); picks the token tile when S is only
                              // a capacity and the segments are filled on the device
    int max_rows;             // upper bound of rows in one segment (weights streamed once if <= tile)
    int ksplit;               // K ranges of the down projection: partial outputs
                              // [ksplit, S, d] summed by the caller (the combine)
    const int32_t *offsets;   // [E+1] device, or nullptr
    const uint16_t *W1, *W3;  // [E, d_ff, d]
    const uint16_t *W2;       // [E, d, d_ff]
    const uint16_t *x;        // [S, d]
    uint16_t *H;              // [S, d_ff] intermediate
    float *Y;                 // [ksplit, S, d]
    uint32_t *h_ready;        // ffn_ready_counters(S, E, d_ff) counters, zero before the launch
    uint32_t *sched;          // work counter, zero before the launch; when set, large
                              // batches run the CTA-pair kernel (launch_ffn_pair)
    uint32_t *err;
    bool pdl;                 // launched right after another kernel of this library
    int act;                  // expert activation: 0 silu(W1 x) * W3 x (SwiGLU),
                              // 1 sigmoid(W1 x) * W3 x
    // Narrow kernel only: when set, the rows of segment e are gathered from x
    // ([x_rows, d]) through the token list perm[e * perm_stride + position]
    // instead of being read from a permuted copy.
    const int32_t *perm;
    int perm_stride;
    int x_rows;
    const int32_t *counts;    // [E] rows per segment (the router's totals); offsets are
    int32_t *offsets_out;     // their exclusive prefix, written here [E+1]
    // CTA-pair kernel only: when out is set, the down units add their rows,
    // weighted, into out[T, d] (zero before the launch) instead of writing Y:
    // out[s / k] += gate_w[s] * y_row with s = slot_of_row[row].  For k <= 2
    // and no K split, where two terms added onto zero give the same sum in
    // either order.
    float *out;
    const int32_t *slot_of_row;
    const float *gate_w;
    int k;
    // CTA-pair kernel only: Y holds bf16 rows [S, d] instead of fp32 (its
    // rows are complete sums: that kernel never splits K).
    bool y_bf16;
};

struct CombineLaunch {
    int T, d, k;
    int ksplit;            // partial outputs per row of y, summed in order before weighting
    const int *ksplit_dev; // or read from device memory (written by the expert kernel), if set
    const float *y;        // [ksplit, T*k, d]
    const int32_t *row_of_slot;
    // or, when row_of_slot is null: row of (t, j) = offsets[idx[t,j]] + slot_pos[t,j]
    const int32_t *idx, *slot_pos, *offsets;
    const float *w;
    const float *shared_y;
    float *out;
    bool pdl;                 // launched right after another kernel of this library
    bool y_bf16;              // y holds bf16 rows [T*k, d] (ksplit 1), not fp32
    bool shared_bf16;         // shared_y holds bf16 rows [T, d]
};

// Expert parallelism (ep.cu): rank `rank` of R owns experts
// [rank*E/R, (rank+1)*E/R), R <= 8.  recv_x / recv_y hold every rank's
// receive and output buffer, as addresses this GPU can use (its own, or a
// peer's mapped here).
struct EpDispatchLaunch {
    int T, d, E, k, R, rank;
    int recv_rows;               // rows of each receive buffer
    const uint16_t *x;           // [T, d] bf16
    const int32_t *idx;          // [T, k]
    const int32_t *counts_all;   // [R, E]
    int32_t *offsets;            // [E+1] scratch: this rank's expert segments
    int32_t *tilecnt, *tilebase; // [ntiles, E] scratch
    int32_t *rank_of_pair;       // [T, k] scratch
    uint32_t *done;              // tile counter, zero before the first launch (left zero)
    int32_t *base;               // [E] scratch
    uint32_t *ok;                // scratch word
    uint16_t *const *recv_x;     // [R] host array of device addresses
    int32_t *pos_of_slot;        // [T, k] out
    int32_t *recv_offsets;       // [E/R + 1] out
    uint32_t *err;
};

struct EpCombineLaunch {
    int T, d, E, k, R;
    int recv_rows;
    int ksplit;                  // partial outputs per receive row
    const int32_t *idx, *pos_of_slot;
    const float *w;
    const void *const *recv_y;   // [R] host array of device addresses
    bool y_bf16;                 // the output buffers hold bf16 rows (ksplit 1), not fp32
    const float *shared_y;       // [T, d] or nullptr
    float *out;
};

cudaError_t launch_ep_dispatch(const EpDispatchLaunch &a, cudaStream_t s);
cudaError_t launch_ep_combine(const EpCombineLaunch &a, cudaStream_t s);

// Failure-detection self-test (selftest.cu): a bounded wait that runs out.
cudaError_t launch_wait_timeout(uint32_t *err, cudaStream_t s);

cudaError_t launch_route(const RouteLaunch &a, cudaStream_t s);
cudaError_t launch_ranks(const RanksLaunch &a, cudaStream_t s);
cudaError_t launch_scatter(const ScatterLaunch &a, cudaStream_t s);
cudaError_t launch_ffn(const FfnLaunch &a, cudaStream_t s);
// The same computation by CTA pairs sharing 256-row MMAs, for segments of
// about 128 rows or more and no K split (called by launch_ffn).
bool ffn_pair_eligible(int S, int E_seg, int ksplit);
cudaError_t launch_ffn_pair(const FfnLaunch &a, uint32_t *sched, cudaStream_t s);
// Narrow layers (d <= 1024): every CTA runs whole hidden chunks (up, H in
// shared memory, down) and writes `nsplit` partial outputs [nsplit, S, d].
cudaError_t launch_ffn_small(const FfnLaunch &a, int nsplit_max, int *nsplit_out,
                             cudaStream_t s);
bool ffn_small_supported(int d);
int ffn_small_splits(int S, int E, int d, int d_ff);
int ffn_token_tile(int S, int E_seg);
size_t ffn_ready_counters(int S, int E_seg, int d_ff);
int down_ksplit(int S, int E_seg, int d, int d_ff);
cudaError_t launch_combine(const CombineLaunch &a, cudaStream_t s);

// Expert FFN with FP8 weights (gemm_fp8.cu): e4m3 codes and per-row fp32
// scales; f.x (the permuted token rows) and f.H are fp16 in this path.
struct FfnFp8Launch {
    FfnLaunch f;
    const uint8_t *q1, *q3;   // [E, d_ff, d] e4m3
    const uint8_t *q2;        // [E, d, d_ff] e4m3
    const float *s1, *s3;     // [E, d_ff]
    const float *s2;          // [E, d]
};
cudaError_t launch_ffn_fp8(const FfnFp8Launch &a, cudaStream_t s);

// A bf16 matrix [rows, cols] viewed as (64-column atoms) so that one box
// brings `atoms` consecutive 64-column tiles of box_rows rows (128-byte
// swizzle), each tile at the next multiple of box_rows * 128 bytes.
cudaError_t make_tmap_bf16_atoms(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                                 uint32_t box_rows, uint32_t atoms);

// 2-D e4m3 (byte) matrix read in boxes of 128 columns (128-byte swizzle) by
// 128 rows; fp16 matrices read like make_tmap_bf16 / make_tmap_bf16_atoms.
cudaError_t make_tmap_e4m3(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols);
cudaError_t make_tmap_f16(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                          uint32_t box_rows);
cudaError_t make_tmap_f16_atoms(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                                uint32_t box_rows, uint32_t atoms);

// Tensor maps (tensormap.cpp side, implemented in api.cu).
// 2-D bf16 row-major matrix [rows, cols] read in boxes of 64 columns (128 B,
// 128-byte swizzle) by box_rows rows.
cudaError_t make_tmap_bf16(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                           uint32_t box_rows);

int device_sm_count();

}  // namespace moe
