// gemm_fp8.cu -- the experts' feed-forward with FP8 weights: e4m3 codes with
// one fp32 scale per weight row, W = scale[row] * e4m3(code).  One
// persistent kernel on the 5th-generation tensor cores.
//
// The unit structure is that of the bf16 expert kernel (gemm.cu): up units
// (expert, 128 W1 and W3 rows, token tile) then down units (expert, two
// 128-row W2 blocks, token tile, K range), weights on the MMA's M side and
// the segment's rows on N.  What differs is the operand path:
//   * TMA brings each 128 x 128 weight tile (a 128-column K step) as e4m3
//     bytes (16 KB, 128-byte swizzle) -- half the bytes of bf16, the point of
//     FP8 where the layer streams its weights from HBM (decode);
//   * eight converter warps widen the tiles to fp16 with the hardware
//     conversion of two e4m3 codes to two fp16 values (exact: every e4m3
//     value is an fp16 value), then release the raw stage and mark the
//     operand stage full.
//     With token tiles of up to 64 rows (decode) the widened weights go to
//     tensor memory, one weight row per lane, and the MMA reads its A operand
//     from there: the shared-memory traffic per weight code is then the TMA
//     write and one converter read.  With 128-row token tiles the
//     accumulators fill tensor memory, and the operands go to shared memory
//     in the 128-byte-swizzled K-major layout;
//   * the MMA is kind::f16 with fp16 A and B (the token rows x_perm and the
//     hidden activations H are fp16 in this path) and fp32 accumulators;
//   * the epilogue multiplies each accumulator row by its weight row's scale
//     before the activation (up units) or before the fp32 output (down units).
//
// Pipelines: a deep ring of input stages (the two e4m3 weight tiles of a K
// step, the step's fp16 token rows) keeps enough bytes in flight to stream
// HBM; the converters fill a ring of operand stages (64-column halves of a K
// step: six or four in tensor memory, two in shared memory) from it.  An
// input stage is free once the converters have read its tiles and the MMAs
// its token rows.  With tensor-memory operands the MMA thread waits for both
// halves of a step and issues its 16 MMAs together: each wait stalls the
// MMA issue for a few hundred cycles, which these short (N <= 64) MMAs do
// not hide.

// Roles: warp 0 TMA, warps 1 and 14 MMA (one weight tile each: a thread
// issuing 128 x N x 16 MMAs with N <= 64 is itself the limit, at about 50
// cycles per MMA, and two issuing warps double the rate), warps 2..5
// epilogue, warps 6..13 converters (one weight row of one tile per thread).
//
// Method: the SwiGLU expert w2(silu(w1 x) * w3 x) ("Mistral 8x7B SMoE
// architecture" (jsqmd.com) sec. 3.1 FeedForward) with quantised expert
// weights and the router kept in higher precision (the same page's
// deployment section on quantisation).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace moe {

namespace {

constexpr int kF8Threads = 480;   // warp 0 TMA, 1 and 14 MMA, 2..5 epilogue, 6..13 converters
constexpr int kF8MmaWarp1 = 14;   // issues the second weight tile's MMAs
constexpr int kF8ConvWarps = 8;
constexpr int kF8MaxStages = 8;
constexpr int kF8MaxOps = 6;     // operand ring depth, tensor-memory operands
constexpr int kF8OpStages = 2;   // operand ring depth, shared-memory operands
constexpr uint32_t kRawTile = 128 * 128;  // 128 weight rows x 128 e4m3 codes (16 KB)
constexpr uint32_t kW16Tile = 128 * 128;  // 128 weight rows x 64 fp16 (16 KB)
constexpr size_t kF8Fixed = 1024 /* alignment slack */ +
                            (2 * kF8MaxStages + 2 * kF8MaxOps + 5) * 8 + 16 +
                            4 * (kMaxE + 1) * sizeof(int32_t) + 64;

// Two rings: a deep one of input stages (the e4m3 weight tiles of a K step
// and its token rows, fp16), which keeps enough bytes in flight to stream
// HBM, and one of converted fp16 weight operands.
template <int BN>
struct F8Cfg {
    // Operands in tensor memory when the double-buffered accumulators
    // (2 x 2 x BN columns) leave room for at least four operand stages.
    static constexpr bool kTA = BN <= 64;
    // One input stage covers a 128-column K step: two e4m3 weight tiles and
    // the step's token rows as two 64-column fp16 atoms; an operand stage is
    // one 64-column half of the step, widened: 2 x 16 KB of shared memory, or
    // 2 x 32 tensor-memory columns (two fp16 of K per 32-bit column).
    static constexpr uint32_t kInStage = 2 * kRawTile + 2 * BN * 128u;
    static constexpr int kAccCols = 2 * BN;
    static constexpr int OPS = kTA ? (512 - 2 * kAccCols) / 64 : kF8OpStages;
    static constexpr uint32_t kOpStage = kTA ? 0u : 2 * kW16Tile;  // shared memory
    static constexpr uint32_t kOpCol0 = 2u * kAccCols;            // tensor memory
    static constexpr int kFit = static_cast<int>(
        (227 * 1024 - kF8Fixed - OPS * kOpStage) / kInStage);
    static constexpr int ST = kFit < kF8MaxStages ? kFit : kF8MaxStages;
    static constexpr uint32_t kTmemCols = kTA ? 512u : 2u * kAccCols;
    static constexpr size_t kSmem =
        kF8Fixed + static_cast<size_t>(ST) * kInStage + OPS * kOpStage;
    static_assert(OPS >= 2 && OPS <= kF8MaxOps, "operand ring");
    static_assert(!kTA || OPS % 2 == 0, "operand stages taken in pairs");
    static_assert(!kTA || kOpCol0 + 64u * OPS <= kTmemCols, "tensor-memory operands");
    static_assert(ST >= 2, "pipeline depth");
    static_assert(kTmemCols >= 32 && kTmemCols <= 512, "tensor memory");
    static_assert(kSmem <= 227 * 1024, "shared memory");
    static_assert(kSmem > 227 * 1024 / 2, "one CTA per SM");
};

struct F8Params {
    int E, d, d_ff, S, ksplit;
    size_t part_stride;
    const int32_t *offsets;
    const float *s1, *s3, *s2;  // row scales [E, d_ff], [E, d_ff], [E, d]
    __half *H;                  // [S, d_ff]
    float *Y;                   // [ksplit, S, d]
    uint32_t *h_ready;
    uint32_t *err;
    int act;
};

struct F8Unit {
    bool up;
    int e, blk, r0, valid, tile, k_beg, k_end, ks;
};

template <int BN>
__device__ __forceinline__ F8Unit decode_f8(int u, int u_up, const int32_t *s_off,
                                            const int32_t *s_pu, const int32_t *s_pd,
                                            const int32_t *s_tb, int E, int ksplit, int ksu, int ksd)
{
    F8Unit w;
    w.up = u < u_up;
    const int32_t *pre = w.up ? s_pu : s_pd;
    const int x = w.up ? u : u - u_up;
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pre[mid] <= x) lo = mid;
        else hi = mid - 1;
    }
    w.e = lo;
    int local = x - pre[lo];
    const int cnt = s_off[lo + 1] - s_off[lo];
    const int ntb = (cnt + BN - 1) / BN;
    if (w.up) {
        w.ks = 0;
        w.k_beg = 0;
        w.k_end = ksu;
    } else {
        w.ks = local % ksplit;
        local /= ksplit;
        w.k_beg = w.ks * ksd / ksplit;
        w.k_end = (w.ks + 1) * ksd / ksplit;
    }
    w.blk = local / ntb;
    const int tb = local - w.blk * ntb;
    w.r0 = s_off[lo] + tb * BN;
    const int rem = cnt - tb * BN;
    w.valid = rem < BN ? rem : BN;
    w.tile = s_tb[lo] + tb;
    return w;
}

__device__ __forceinline__ void f8_drain_wait(uint64_t *bar, uint32_t parity)
{
    const uint64_t t0 = ptx::globaltimer();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::globaltimer() - t0 > 100000000ull) break;  // 100 ms
    }
}

__device__ __forceinline__ uint32_t f8_ld_acquire(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void f8_fence_proxy_async_global()
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void f8_fence_proxy_async_shared()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ bool f8_wait_counter(const uint32_t *ctr, uint32_t target,
                                                volatile uint32_t *abort_flag, uint32_t *gerr)
{
    if (f8_ld_acquire(ctr) >= target) return true;
    const uint64_t t0 = ptx::globaltimer();
    for (uint32_t it = 1;; ++it) {
        __nanosleep(64);
        if (f8_ld_acquire(ctr) >= target) return true;
        if (*abort_flag) return false;
        if ((it & 15u) == 0 && ptx::globaltimer() - t0 > kWaitTimeoutNs) {
            *abort_flag = 1u;
            if (gerr) atomicOr(gerr, kErrTimeoutEpi);
            return false;
        }
    }
}

__device__ __forceinline__ int f8_scan(int v, int lane)
{
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += n;
    }
    return v;
}

// Four e4m3 codes (low byte first) to four fp16 values, two per word, with
// the hardware conversion of an e4m3 pair (exact: every e4m3 value, the
// subnormals included, is an fp16 value).  Measured against widening by
// integer bit moves at decode: the converters were the limit, with the
// integer pipe 65% busy, and the expert kernel went from 219 to 189 us per
// launch at T = 8.
__device__ __forceinline__ void e4m3x4_to_f16x4(uint32_t v, uint32_t &lo, uint32_t &hi)
{
    const __half2_raw a =
        __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(v & 0xffffu), __NV_E4M3);
    const __half2_raw b =
        __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(v >> 16), __NV_E4M3);
    lo = *reinterpret_cast<const uint32_t *>(&a);  // codes 0, 1
    hi = *reinterpret_cast<const uint32_t *>(&b);  // codes 2, 3
}

// Instruction descriptor of kind::f16 with fp16 A/B, fp32 D, both K-major.
__device__ __forceinline__ uint32_t idesc_f16_f32(int M, int N)
{
    return (1u << 4)                                 // D format fp32
           | (static_cast<uint32_t>(N >> 3) << 17)   // N / 8   (A, B format fp16 = 0)
           | (static_cast<uint32_t>(M >> 4) << 24);  // M / 16
}

template <int BN>
__global__ void __launch_bounds__(kF8Threads, 1)
    ffn_fp8_kernel(const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmW3,
                   const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmX,
                   const __grid_constant__ CUtensorMap tmH, const F8Params p)
{
    using C = F8Cfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    constexpr int ST = C::ST;
    constexpr int OPS = C::OPS;
    uint8_t *ops = smem;                                       // [OPS] fp16 weight operands
    uint8_t *ins = smem + OPS * C::kOpStage;                   // [ST] e4m3 tiles + token rows
    uint64_t *in_full = reinterpret_cast<uint64_t *>(ins + ST * C::kInStage);
    uint64_t *in_empty = in_full + kF8MaxStages;
    uint64_t *op_full = in_empty + kF8MaxStages;
    uint64_t *op_empty = op_full + kF8MaxOps;
    uint64_t *tfull = op_empty + kF8MaxOps;  // [2]
    uint64_t *tempty = tfull + 2;             // [2]
    uint64_t *drain = tempty + 2;             // [1]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile uint32_t *abort_flag = tmem_slot + 1;
    int32_t *s_off = reinterpret_cast<int32_t *>(tmem_slot + 4);
    int32_t *s_pu = s_off + (kMaxE + 1);
    int32_t *s_pd = s_pu + (kMaxE + 1);
    int32_t *s_tb = s_pd + (kMaxE + 1);

    const int E = p.offsets ? p.E : 1;
    const int MBU = p.d_ff / 128;
    const int MBD = (p.d + 255) / 256;
    const int KSU = p.d / 128;       // 128-column K steps
    const int KSD = p.d_ff / 128;
    const int KSPLIT = p.ksplit;

    if (threadIdx.x == 0) {
        for (int s = 0; s < ST; ++s) {
            ptx::mbar_init(&in_full[s], 1);
            ptx::mbar_init(&in_empty[s], kF8ConvWarps + 2);  // converters (e4m3 read) + 2 MMA warps (rows read)
        }
        for (int s = 0; s < OPS; ++s) {
            ptx::mbar_init(&op_full[s], kF8ConvWarps);
            ptx::mbar_init(&op_empty[s], 2);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&tfull[b], 2);
            ptx::mbar_init(&tempty[b], 4);
        }
        ptx::mbar_init(drain, 2);
        *abort_flag = 0u;
        ptx::fence_barrier_init();
    }
    if (threadIdx.x == 32) {
        ptx::prefetch_tensormap(&tmW1);
        ptx::prefetch_tensormap(&tmW3);
        ptx::prefetch_tensormap(&tmW2);
        ptx::prefetch_tensormap(&tmX);
        ptx::prefetch_tensormap(&tmH);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, C::kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::grid_dep_wait();
    if (warp == 2) {
        const int per = (E + 31) >> 5;
        const int base = lane * per;
        bool bad = false;
        int nu = 0, nd = 0, nt = 0;
        for (int i = 0; i < per; ++i) {
            const int e = base + i;
            if (e < E) {
                const int o0 = p.offsets ? p.offsets[e] : 0;
                const int o1 = p.offsets ? p.offsets[e + 1] : p.S;
                s_off[e] = o0;
                if (e == E - 1) s_off[E] = o1;
                const int c = o1 - o0;
                if (o0 < 0 || c < 0 || o1 > p.S) {
                    bad = true;
                } else {
                    const int ntb = (c + BN - 1) / BN;
                    nt += ntb;
                    nu += ntb * MBU;
                    nd += ntb * MBD * KSPLIT;
                }
            }
        }
        __syncwarp();
        bad = __any_sync(0xffffffffu, bad);
        if (bad) {
            nu = nd = nt = 0;
            if (lane == 0) atomicOr(p.err, kErrOffsets);
        }
        const int iu = f8_scan(nu, lane);
        const int id = f8_scan(nd, lane);
        const int it = f8_scan(nt, lane);
        int ru = iu - nu, rd = id - nd, rt = it - nt;
        for (int i = 0; i < per; ++i) {
            const int e = base + i;
            if (e < E) {
                s_pu[e] = ru;
                s_pd[e] = rd;
                s_tb[e] = rt;
                if (!bad) {
                    const int ntb = (s_off[e + 1] - s_off[e] + BN - 1) / BN;
                    ru += ntb * MBU;
                    rd += ntb * MBD * KSPLIT;
                    rt += ntb;
                }
            }
        }
        if (lane == 31) {
            s_pu[E] = iu;
            s_pd[E] = id;
            s_tb[E] = it;
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int u_up = s_pu[E];
    const int total = u_up + s_pd[E];

    if (warp == 0) {
        if (lane == 0) {
            uint32_t stage = 0, phase = 0, issued = 0;
            uint32_t last_parity[kF8MaxStages];
#pragma unroll
            for (int s = 0; s < kF8MaxStages; ++s) last_parity[s] = 0;
            const uint64_t pol_w = ptx::policy_evict_first();
            bool stop = false;
            for (int u = blockIdx.x; u < total && !stop; u += gridDim.x) {
                const F8Unit w = decode_f8<BN>(u, u_up, s_off, s_pu, s_pd, s_tb, E, KSPLIT, KSU, KSD);
                const CUtensorMap *ta0 = w.up ? &tmW1 : &tmW2;
                const CUtensorMap *ta1 = w.up ? &tmW3 : &tmW2;
                const CUtensorMap *tb = w.up ? &tmX : &tmH;
                const int arow0 = w.up ? w.e * p.d_ff + w.blk * 128 : w.e * p.d + w.blk * 256;
                const int arow1 = w.up ? arow0 : arow0 + 128;
                for (int ks = w.k_beg; ks < w.k_end; ++ks) {
                    if (!bounded_wait(&in_empty[stage], phase ^ 1u, abort_flag, p.err,
                                      kErrTimeoutEpi)) {
                        stop = true;
                        break;
                    }
                    uint8_t *in = ins + stage * C::kInStage;
                    ptx::mbar_arrive_expect_tx(&in_full[stage], C::kInStage);
                    ptx::tma_load_2d_hint(in, ta0, &in_full[stage], ks * 128, arow0, pol_w);
                    ptx::tma_load_2d_hint(in + kRawTile, ta1, &in_full[stage], ks * 128, arow1,
                                          pol_w);
                    issued |= 1u << stage;
                    last_parity[stage] = phase;
                    if (!w.up) {
                        // The step's 128 columns of H are block ks.
                        if (!f8_wait_counter(&p.h_ready[w.tile * MBU + ks], 4u, abort_flag,
                                             p.err)) {
                            stop = true;
                            break;
                        }
                        f8_fence_proxy_async_global();
                    }
                    ptx::tma_load_3d(in + 2 * kRawTile, tb, &in_full[stage], 0, w.r0, ks * 2);
                    if (++stage == static_cast<uint32_t>(ST)) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            for (int s = 0; s < ST; ++s)
                if (issued & (1u << s)) f8_drain_wait(&in_full[s], last_parity[s]);
        }
    } else if (warp == 1 || warp == kF8MmaWarp1) {
        if (lane == 0) {
            // This warp's weight tile: 0 (W1 rows, or W2 rows 0..127 of the
            // down block) into accumulator d0, 1 (W3, or W2 rows 128..255)
            // into d0 + BN.  Both warps wait for the same stages, and every
            // barrier they release counts one commit from each.
            const int t = warp == 1 ? 0 : 1;
            uint32_t stage = 0, phase = 0;    // input ring
            uint32_t ost = 0, ophase = 0;     // operand ring
            int i = 0;
            bool stop = false;
            for (int u = blockIdx.x; u < total && !stop; u += gridDim.x, ++i) {
                const F8Unit w = decode_f8<BN>(u, u_up, s_off, s_pu, s_pd, s_tb, E, KSPLIT, KSU, KSD);
                const int n = ((w.valid + 15) >> 4) << 4;
                const uint32_t idesc = idesc_f16_f32(128, n);
                const int buf = i & 1;
                const uint32_t use = static_cast<uint32_t>(i >> 1);
                if (!bounded_wait(&tempty[buf], (use & 1u) ^ 1u, abort_flag, p.err,
                                  kErrTimeoutEpi))
                    break;
                ptx::tc_fence_after();
                const uint32_t d0 = tmem + static_cast<uint32_t>(buf * C::kAccCols + t * BN);
                for (int ks = w.k_beg; ks < w.k_end && !stop; ++ks) {
                    // The token rows came with the input stage; the weights
                    // were converted, one 64-column half at a time, into the
                    // operand stages.
                    if (!bounded_wait(&in_full[stage], phase, abort_flag, p.err, kErrTimeoutTma)) {
                        stop = true;
                        break;
                    }
                    if constexpr (C::kTA) {
                        // Both halves' operands (stages ost, ost + 1: OPS is
                        // even, so a pair never wraps), then this tile's 8
                        // MMAs of the step.  Each wait stalls the MMA issue
                        // for a few hundred cycles, which MMAs this short
                        // (N <= 64) do not hide: one wait per step.
                        if (!bounded_wait(&op_full[ost], ophase, abort_flag, p.err,
                                          kErrTimeoutTma) ||
                            !bounded_wait(&op_full[ost + 1], ophase, abort_flag, p.err,
                                          kErrTimeoutTma)) {
                            stop = true;
                            break;
                        }
                        ptx::tc_fence_after();
#pragma unroll
                        for (int hf = 0; hf < 2; ++hf) {
                            const uint32_t sb = ptx::smem_addr(ins + stage * C::kInStage +
                                                               2 * kRawTile + hf * BN * 128);
                            // A: tile t of stage ost + hf at columns
                            // kOpCol0 + 64 (ost + hf) + 32 t, 16 K elements per 8 columns.
                            const uint32_t ta = tmem + C::kOpCol0 + 64u * (ost + hf) + 32u * t;
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint64_t bdesc = ptx::sw128_kmajor_desc(sb + kk * 32);
                                const uint32_t acc = ((ks - w.k_beg) | hf | kk) ? 1u : 0u;
                                ptx::tc_mma_f16_ts(d0, ta + 8u * kk, bdesc, idesc, acc);
                            }
                        }
                        ptx::tc_commit(&op_empty[ost]);
                        ptx::tc_commit(&op_empty[ost + 1]);
                        ost += 2;
                        if (ost == static_cast<uint32_t>(OPS)) {
                            ost = 0;
                            ophase ^= 1u;
                        }
                    } else {
                        // Shared-memory operands, two stages: one 64-column
                        // half at a time, so the converters refill the first
                        // stage while the MMAs read the second.
                        for (int hf = 0; hf < 2; ++hf) {
                            if (!bounded_wait(&op_full[ost], ophase, abort_flag, p.err,
                                              kErrTimeoutTma)) {
                                stop = true;
                                break;
                            }
                            ptx::tc_fence_after();
                            const uint32_t sb = ptx::smem_addr(ins + stage * C::kInStage +
                                                               2 * kRawTile + hf * BN * 128);
                            const uint32_t sa = ptx::smem_addr(ops + ost * C::kOpStage + t * kW16Tile);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint64_t bdesc = ptx::sw128_kmajor_desc(sb + kk * 32);
                                const uint32_t acc = ((ks - w.k_beg) | hf | kk) ? 1u : 0u;
                                ptx::tc_mma_bf16(d0, ptx::sw128_kmajor_desc(sa + kk * 32), bdesc,
                                                 idesc, acc);
                            }
                            ptx::tc_commit(&op_empty[ost]);
                            if (++ost == static_cast<uint32_t>(OPS)) {
                                ost = 0;
                                ophase ^= 1u;
                            }
                        }
                    }
                    if (stop) break;
                    ptx::tc_commit(&in_empty[stage]);
                    if (++stage == static_cast<uint32_t>(ST)) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!stop) ptx::tc_commit(&tfull[buf]);
            }
            ptx::tc_commit(drain);
            f8_drain_wait(drain, 0u);
        }
    } else if (warp >= 6 && warp < 6 + kF8ConvWarps) {
        // Converters: warp w widens rows 32 (w % 4) .. 32 (w % 4) + 31 of
        // weight tile (w - 6) / 4 of a step, one row per thread -- the rows
        // of the tensor-memory lanes the warp may access.
        const int t = (warp - 6) >> 2;  // 0, 1
        const int r = 32 * (warp & 3) + lane;
        const uint32_t t_row = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + C::kOpCol0 +
                               32u * static_cast<uint32_t>(t);
        uint32_t stage = 0, phase = 0;    // input ring
        uint32_t ost = 0, ophase = 0;     // operand ring
        bool stop = false;
        if constexpr (C::kTA) {
            // Both 64-column halves of a step at once, as the MMA warps take
            // them: one wait for free stages, one store wait, one arrival
            // per stage.
            for (int u = blockIdx.x; u < total && !stop; u += gridDim.x) {
                const F8Unit w = decode_f8<BN>(u, u_up, s_off, s_pu, s_pd, s_tb, E, KSPLIT, KSU, KSD);
                for (int ks = w.k_beg; ks < w.k_end && !stop; ++ks) {
                    const bool ok =
                        bounded_wait(&in_full[stage], phase, abort_flag, p.err, kErrTimeoutTma) &&
                        bounded_wait(&op_empty[ost], ophase ^ 1u, abort_flag, p.err, kErrTimeoutMma) &&
                        bounded_wait(&op_empty[ost + 1], ophase ^ 1u, abort_flag, p.err,
                                     kErrTimeoutMma);
                    if (!__all_sync(0xffffffffu, ok)) {
                        *abort_flag = 1u;
                        stop = true;
                        break;
                    }
                    ptx::tc_fence_after();
                    // Raw row r: 128 bytes, 16-byte chunk j stored at chunk
                    // j ^ (r & 7) (128-byte swizzle); codes 64hf .. 64hf + 63
                    // (chunks 4hf .. 4hf + 3) go to the tile's 32 columns of
                    // stage ost + hf.
                    const uint8_t *src = ins + stage * C::kInStage + t * kRawTile + r * 128;
                    uint32_t v64[64];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint4 v = *reinterpret_cast<const uint4 *>(src + ((j ^ (r & 7)) << 4));
                        e4m3x4_to_f16x4(v.x, v64[8 * j + 0], v64[8 * j + 1]);
                        e4m3x4_to_f16x4(v.y, v64[8 * j + 2], v64[8 * j + 3]);
                        e4m3x4_to_f16x4(v.z, v64[8 * j + 4], v64[8 * j + 5]);
                        e4m3x4_to_f16x4(v.w, v64[8 * j + 6], v64[8 * j + 7]);
                    }
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        ptx::tmem_st16(t_row + 64u * (ost + hf),
                                       *reinterpret_cast<const uint32_t(*)[16]>(&v64[32 * hf]));
                        ptx::tmem_st16(t_row + 64u * (ost + hf) + 16u,
                                       *reinterpret_cast<const uint32_t(*)[16]>(&v64[32 * hf + 16]));
                    }
                    // The MMA warps read the operands after the arrivals.
                    ptx::tc_wait_st();
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        ptx::mbar_arrive(&op_full[ost]);
                        ptx::mbar_arrive(&op_full[ost + 1]);
                        ptx::mbar_arrive(&in_empty[stage]);
                    }
                    ost += 2;
                    if (ost == static_cast<uint32_t>(OPS)) {
                        ost = 0;
                        ophase ^= 1u;
                    }
                    if (++stage == static_cast<uint32_t>(ST)) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        } else {
            for (int u = blockIdx.x; u < total && !stop; u += gridDim.x) {
                const F8Unit w = decode_f8<BN>(u, u_up, s_off, s_pu, s_pd, s_tb, E, KSPLIT, KSU, KSD);
                for (int ks = w.k_beg; ks < w.k_end && !stop; ++ks) {
                    const bool ok =
                        bounded_wait(&in_full[stage], phase, abort_flag, p.err, kErrTimeoutTma);
                    if (!__all_sync(0xffffffffu, ok)) {
                        *abort_flag = 1u;
                        stop = true;
                        break;
                    }
                    const uint8_t *ra = ins + stage * C::kInStage;
                    for (int hf = 0; hf < 2; ++hf) {
                        const bool oke =
                            bounded_wait(&op_empty[ost], ophase ^ 1u, abort_flag, p.err, kErrTimeoutMma);
                        if (!__all_sync(0xffffffffu, oke)) {
                            *abort_flag = 1u;
                            stop = true;
                            break;
                        }
                        ptx::tc_fence_after();
                        // Raw row r: 128 bytes, 16-byte chunk j stored at chunk
                        // j ^ (r & 7) (128-byte swizzle); this half is chunks
                        // 4hf..4hf+3, i.e. columns 64hf..64hf+63.
                        const uint8_t *src = ra + t * kRawTile + r * 128;
                        uint8_t *op = ops + ost * C::kOpStage;
                        uint8_t *dst = op + t * kW16Tile + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint4 v = *reinterpret_cast<const uint4 *>(
                                src + (((4 * hf + j) ^ (r & 7)) << 4));
                            // 16 codes = columns 16j..16j+15 of the half -> two
                            // 16-byte fp16 chunks 2j and 2j+1 of the operand row.
                            uint4 lo, hi;
                            e4m3x4_to_f16x4(v.x, lo.x, lo.y);
                            e4m3x4_to_f16x4(v.y, lo.z, lo.w);
                            e4m3x4_to_f16x4(v.z, hi.x, hi.y);
                            e4m3x4_to_f16x4(v.w, hi.z, hi.w);
                            *reinterpret_cast<uint4 *>(dst + (((2 * j) ^ (r & 7)) << 4)) = lo;
                            *reinterpret_cast<uint4 *>(dst + (((2 * j + 1) ^ (r & 7)) << 4)) = hi;
                        }
                        // The MMA reads the operand through the async proxy.
                        f8_fence_proxy_async_shared();
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(&op_full[ost]);
                        if (++ost == static_cast<uint32_t>(OPS)) {
                            ost = 0;
                            ophase ^= 1u;
                        }
                    }
                    if (stop) break;
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&in_empty[stage]);
                    if (++stage == static_cast<uint32_t>(ST)) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
    } else if (warp >= 2 && warp <= 5) {
        // Epilogue: warps 2..5, one TMEM lane quarter each.
        const int q = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
        int i = 0;
        for (int u = blockIdx.x; u < total; u += gridDim.x, ++i) {
            const F8Unit w = decode_f8<BN>(u, u_up, s_off, s_pu, s_pd, s_tb, E, KSPLIT, KSU, KSD);
            const int buf = i & 1;
            const uint32_t use = static_cast<uint32_t>(i >> 1);
            if (!bounded_wait_warp(&tfull[buf], use & 1u, abort_flag, p.err, kErrTimeoutMma))
                break;
            ptx::tc_fence_after();
            const uint32_t tb = tmem + lane_base + static_cast<uint32_t>(buf * C::kAccCols);
            const int row_in_blk = 32 * q + lane;
            float sa, sb;
            if (w.up) {
                const int f = w.blk * 128 + row_in_blk;
                sa = p.s1[static_cast<size_t>(w.e) * p.d_ff + f];
                sb = p.s3[static_cast<size_t>(w.e) * p.d_ff + f];
            } else {
                const int o0 = w.blk * 256 + row_in_blk;
                sa = o0 < p.d ? p.s2[static_cast<size_t>(w.e) * p.d + o0] : 0.0f;
                sb = o0 + 128 < p.d
                         ? p.s2[static_cast<size_t>(w.e) * p.d + o0 + 128]
                         : 0.0f;
            }
            for (int c0 = 0; c0 < w.valid; c0 += 32) {
                uint32_t a[32], b[32];
                ptx::tmem_ld32(tb + static_cast<uint32_t>(c0), a);
                ptx::tmem_ld32(tb + static_cast<uint32_t>(BN + c0), b);
                ptx::tc_wait_ld();
                if (w.up) {
                    const int f = w.blk * 128 + row_in_blk;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (c0 + j < w.valid) {
                            const float g = sa * __uint_as_float(a[j]);
                            const float bv = sb * __uint_as_float(b[j]);
                            const float h = __fdividef(p.act ? bv : g * bv, 1.0f + __expf(-g));
                            p.H[static_cast<size_t>(w.r0 + c0 + j) * p.d_ff + f] = __float2half_rn(h);
                        }
                    }
                } else {
                    const int o0 = w.blk * 256 + row_in_blk;
                    const bool has0 = o0 < p.d;
                    const bool has1 = o0 + 128 < p.d;
                    float *Y = p.Y + w.ks * p.part_stride;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (c0 + j < w.valid) {
                            float *yr = Y + static_cast<size_t>(w.r0 + c0 + j) * p.d;
                            if (has0) yr[o0] = sa * __uint_as_float(a[j]);
                            if (has1) yr[o0 + 128] = sb * __uint_as_float(b[j]);
                        }
                    }
                }
            }
            ptx::tc_fence_before();
            if (w.up) {
                // Publish this warp's slice of the H block to the down units
                // (which read it through TMA, the async proxy).
                f8_fence_proxy_async_global();
                __threadfence();
            }
            __syncwarp();
            if (lane == 0) {
                if (w.up) atomicAdd(&p.h_ready[w.tile * MBU + w.blk], 1u);
                ptx::mbar_arrive(&tempty[buf]);
            }
        }
    }

    ptx::grid_dep_launch();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int BN>
cudaError_t launch_fp8_cfg(const FfnFp8Launch &a, cudaStream_t s)
{
    using C = F8Cfg<BN>;
    const int E = a.f.offsets ? a.f.E : 1;
    CUtensorMap tW1, tW3, tW2, tX, tH;
    cudaError_t e = make_tmap_e4m3(&tW1, a.q1, static_cast<uint64_t>(E) * a.f.d_ff, a.f.d);
    if (e == cudaSuccess) e = make_tmap_e4m3(&tW3, a.q3, static_cast<uint64_t>(E) * a.f.d_ff, a.f.d);
    if (e == cudaSuccess) e = make_tmap_e4m3(&tW2, a.q2, static_cast<uint64_t>(E) * a.f.d, a.f.d_ff);
    if (e == cudaSuccess) e = make_tmap_f16_atoms(&tX, a.f.x, a.f.S, a.f.d, BN, 2);
    if (e == cudaSuccess) e = make_tmap_f16_atoms(&tH, a.f.H, a.f.S, a.f.d_ff, BN, 2);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(ffn_fp8_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(C::kSmem));
    if (e != cudaSuccess) return e;
    F8Params p{};
    p.E = E;
    p.d = a.f.d;
    p.d_ff = a.f.d_ff;
    p.S = a.f.S;
    p.ksplit = a.f.ksplit < 1 ? 1 : a.f.ksplit;
    p.part_stride = static_cast<size_t>(a.f.S) * a.f.d;
    p.offsets = a.f.offsets;
    p.s1 = a.s1;
    p.s3 = a.s3;
    p.s2 = a.s2;
    p.H = reinterpret_cast<__half *>(a.f.H);
    p.Y = a.f.Y;
    p.h_ready = a.f.h_ready;
    p.err = a.f.err;
    p.act = a.f.act;
    const long long tiles = (static_cast<long long>(a.f.S) + BN - 1) / BN + E;
    const long long units =
        tiles * (a.f.d_ff / 128) + tiles * ((a.f.d + 255) / 256) * p.ksplit;
    long long grid = device_sm_count();
    if (units < grid) grid = units;
    if (grid < 1) grid = 1;
    return launch_pdl(ffn_fp8_kernel<BN>, dim3(static_cast<unsigned>(grid)), dim3(kF8Threads),
                      C::kSmem, s, a.f.pdl, tW1, tW3, tW2, tX, tH, p);
}

}  // namespace

cudaError_t launch_ffn_fp8(const FfnFp8Launch &a, cudaStream_t s)
{
    switch (ffn_token_tile(a.f.S, a.f.offsets ? a.f.E : 1)) {
    case 32: return launch_fp8_cfg<32>(a, s);
    case 64: return launch_fp8_cfg<64>(a, s);
    default: return launch_fp8_cfg<128>(a, s);
    }
}

}  // namespace moe
