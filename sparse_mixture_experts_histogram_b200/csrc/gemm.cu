// gemm.cu -- grouped expert GEMMs on the 5th-generation tensor cores.
//
// For every expert segment e (rows offsets[e] .. offsets[e+1]-1 of the
// activation matrix B) and every 128-row block of that expert's weights A:
//   up:   D1 = W1_e[blk] B^T, D3 = W3_e[blk] B^T  (two accumulators),
//         H[r, blk] = bf16( silu(D1) * D3 )        -- SwiGLU in the epilogue
//   down: Y[r, blk] = W2_e[blk] H^T                 -- fp32 out
// The weights are the MMA's A operand (M = 128 weight rows) and the tokens
// its B operand (N = the segment's rows, rounded up to 16), so a ragged or
// tiny segment costs only the columns it needs, and decode-sized batches
// stream each hit expert's weights once.
//
// Persistent kernel, one CTA per SM: warp 0 issues TMA copies into a ring of
// shared-memory stages, warp 1 issues tcgen05 MMAs into a double-buffered
// tensor-memory accumulator, warps 2..5 drain finished accumulators
// (tcgen05.ld), apply the epilogue and store; the next tile's MMAs overlap
// the previous tile's epilogue.  Work units (expert, weight block, token
// tile) are numbered from the device-side offsets, with consecutive units
// sharing one weight block so that concurrent CTAs re-read it from L2.
//
// Method: the SwiGLU expert w2(silu(w1 x) * w3 x) ("Mistral 8x7B SMoE
// architecture" (jsqmd.com) sec. 3.1 FeedForward; "Mixtral and MoE
// architecture" FeedForward listing) applied to each expert's own tokens
// ("MoE" (theaiera.top) sec. 10.4); W1 and W3 are consumed side by side so
// the activation runs in the epilogue, the fusion the "万亿 MoE" page
// (m.xxqk.cn) sketches by concatenating the two up-projections.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace moe {

namespace {

constexpr int kGemmThreads = 192;
constexpr int kGemmMaxStages = 12;
constexpr uint32_t kWTileBytes = 128 * 128;  // 128 weight rows x 64 bf16
constexpr size_t kGemmFixedSmem = 1024 /* alignment slack */ + (2 * kGemmMaxStages + 5) * 8 + 16 +
                                  2 * (kMaxE + 1) * sizeof(int32_t) + 64;
constexpr size_t kSmemBudget = 227 * 1024;

template <bool UP, int BN, int ST>
struct Cfg {
    static constexpr int kA = UP ? 2 : 1;
    static constexpr uint32_t kBBytes = BN * 128u;
    static constexpr uint32_t kStageBytes = kA * kWTileBytes + kBBytes;
    static constexpr int kAccCols = UP ? 2 * BN : BN;
    static constexpr uint32_t kTmemCols = 2u * kAccCols;
    static constexpr int kStages = ST;
    static constexpr size_t kSmem = kGemmFixedSmem + static_cast<size_t>(kStages) * kStageBytes;
    static_assert(kTmemCols >= 32 && kTmemCols <= 512 && (kTmemCols & (kTmemCols - 1)) == 0,
                  "tensor memory allocation must be a power of two in [32, 512]");
    static_assert(kStages >= 2 && kStages <= kGemmMaxStages, "pipeline depth");
    static_assert(kSmem <= kSmemBudget, "shared memory");
    // One CTA per SM: the shared memory above keeps a second CTA (and its
    // tensor-memory allocation) off the SM.
    static_assert(kSmem > kSmemBudget / 2, "one CTA per SM");
};

struct GemmParams {
    int E;          // segments
    int M_rows;     // weight rows per expert
    int K;          // reduction length (multiple of 64)
    int S;          // rows of B
    const int32_t *offsets;  // [E+1] or nullptr (one segment [0, S))
    void *out;               // [S, M_rows]
    uint32_t *err;
    int stream_weights;      // 1: each weight block feeds one tile; hint L2 to evict it first
    int ksplit;              // K is split into this many ranges (down only; partial outputs)
    size_t part_stride;      // elements between the partial outputs of consecutive K ranges
};

struct Unit {
    int e, mb, r0, valid, ks;
};

// Work unit u -> (expert, weight block, token tile, K range).  Units of one
// expert are numbered weight-block-major, then token tile, then K range, so
// that CTAs running at the same time share a weight block through L2.
template <int BN>
__device__ __forceinline__ Unit decode_unit(int u, const int32_t *s_pre, const int32_t *s_off,
                                            int E, int ksplit)
{
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_pre[mid] <= u) lo = mid;
        else hi = mid - 1;
    }
    Unit w;
    w.e = lo;
    int local = u - s_pre[lo];
    w.ks = local % ksplit;
    local /= ksplit;
    const int cnt = s_off[lo + 1] - s_off[lo];
    const int ntb = (cnt + BN - 1) / BN;
    w.mb = local / ntb;
    const int tb = local - w.mb * ntb;
    w.r0 = s_off[lo] + tb * BN;
    const int rem = cnt - tb * BN;
    w.valid = rem < BN ? rem : BN;
    return w;
}

__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity)
{
    const uint64_t t0 = ptx::globaltimer();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::globaltimer() - t0 > 100000000ull) break;  // 100 ms
    }
}

template <bool UP, int BN, int ST>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                const __grid_constant__ CUtensorMap tmB, const GemmParams p)
{
    using C = Cfg<UP, BN, ST>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kStages * C::kStageBytes);
    uint64_t *empty = full + kGemmMaxStages;
    uint64_t *tfull = empty + kGemmMaxStages;   // [2]
    uint64_t *tempty = tfull + 2;               // [2]
    uint64_t *drain = tempty + 2;               // [1]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile uint32_t *abort_flag = tmem_slot + 1;
    int32_t *s_off = reinterpret_cast<int32_t *>(tmem_slot + 4);
    int32_t *s_pre = s_off + (kMaxE + 1);

    const int E = p.offsets ? p.E : 1;
    const int MB = p.M_rows / 128;
    const int KS = p.K / 64;
    const int KSPLIT = p.ksplit;

    ptx::grid_dep_launch();
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&tfull[b], 1);
            ptx::mbar_init(&tempty[b], 4);   // one arrival per epilogue warp
        }
        ptx::mbar_init(drain, 1);
        *abort_flag = 0u;
        ptx::fence_barrier_init();
    }
    if (threadIdx.x == 32) {
        ptx::prefetch_tensormap(&tmA0);
        if (UP) ptx::prefetch_tensormap(&tmA1);
        ptx::prefetch_tensormap(&tmB);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, C::kTmemCols);
        ptx::tmem_relinquish();
    }
    // Everything above overlaps the previous kernel; from here on its results
    // (offsets, activations) are read and this kernel's outputs are written.
    ptx::grid_dep_wait();
    if (warp == 2) {
        // Segment table and the unit prefix (units of expert e =
        // ceil(rows_e / BN) token tiles x MB weight blocks).
        const int per = (E + 31) >> 5;
        const int base = lane * per;
        bool bad = false;
        int local = 0;
        for (int i = 0; i < per; ++i) {
            const int e = base + i;
            if (e < E) {
                const int o0 = p.offsets ? p.offsets[e] : 0;
                const int o1 = p.offsets ? p.offsets[e + 1] : p.S;
                s_off[e] = o0;
                if (e == E - 1) s_off[E] = o1;
                const int c = o1 - o0;
                if (o0 < 0 || c < 0 || o1 > p.S) bad = true;
                else local += ((c + BN - 1) / BN) * MB * KSPLIT;
            }
        }
        bad = __any_sync(0xffffffffu, bad);
        if (bad) {
            local = 0;
            if (lane == 0) atomicOr(p.err, kErrOffsets);
        }
        int incl = local;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        int run = incl - local;
        for (int i = 0; i < per; ++i) {
            const int e = base + i;
            if (e < E) {
                s_pre[e] = run;
                if (!bad) {
                    const int c = s_off[e + 1] - s_off[e];
                    run += ((c + BN - 1) / BN) * MB * KSPLIT;
                }
            }
        }
        if (lane == 31) s_pre[E] = incl;
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int total = s_pre[E];

    if (warp == 0) {
        if (lane == 0) {
            uint32_t stage = 0, phase = 0, issued = 0;
            uint32_t last_parity[kGemmMaxStages];
#pragma unroll
            for (int s = 0; s < kGemmMaxStages; ++s) last_parity[s] = 0;
            const uint64_t pol_w =
                p.stream_weights ? ptx::policy_evict_first() : ptx::policy_evict_normal();
            bool stop = false;
            for (int u = blockIdx.x; u < total && !stop; u += gridDim.x) {
                const Unit w = decode_unit<BN>(u, s_pre, s_off, E, KSPLIT);
                const int arow = w.e * p.M_rows + w.mb * 128;
                const int k_end = (w.ks + 1) * KS / KSPLIT;
                for (int ks = w.ks * KS / KSPLIT; ks < k_end; ++ks) {
                    if (!bounded_wait(&empty[stage], phase ^ 1u, abort_flag, p.err,
                                      kErrTimeoutMma)) {
                        stop = true;
                        break;
                    }
                    uint8_t *sa = smem + stage * C::kStageBytes;
                    ptx::mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
                    ptx::tma_load_2d_hint(sa, &tmA0, &full[stage], ks * 64, arow, pol_w);
                    if (UP)
                        ptx::tma_load_2d_hint(sa + kWTileBytes, &tmA1, &full[stage], ks * 64, arow,
                                              pol_w);
                    ptx::tma_load_2d(sa + C::kA * kWTileBytes, &tmB, &full[stage], ks * 64, w.r0);
                    issued |= 1u << stage;
                    last_parity[stage] = phase;
                    if (++stage == static_cast<uint32_t>(C::kStages)) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // Make sure no copy is still landing in shared memory at exit.
            for (int s = 0; s < C::kStages; ++s)
                if (issued & (1u << s)) drain_wait(&full[s], last_parity[s]);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            int i = 0;
            bool stop = false;
            for (int u = blockIdx.x; u < total && !stop; u += gridDim.x, ++i) {
                const Unit w = decode_unit<BN>(u, s_pre, s_off, E, KSPLIT);
                const int n = ((w.valid + 15) >> 4) << 4;
                const int k_beg = w.ks * KS / KSPLIT;
                const int k_end = (w.ks + 1) * KS / KSPLIT;
                const uint32_t idesc = ptx::idesc_bf16_f32(128, n);
                const int buf = i & 1;
                const uint32_t use = static_cast<uint32_t>(i >> 1);
                if (!bounded_wait(&tempty[buf], (use & 1u) ^ 1u, abort_flag, p.err,
                                  kErrTimeoutEpi))
                    break;
                ptx::tc_fence_after();
                const uint32_t d0 = tmem + static_cast<uint32_t>(buf * C::kAccCols);
                for (int ks = k_beg; ks < k_end; ++ks) {
                    if (!bounded_wait(&full[stage], phase, abort_flag, p.err, kErrTimeoutTma)) {
                        stop = true;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t sa = ptx::smem_addr(smem + stage * C::kStageBytes);
                    const uint32_t sb = sa + C::kA * kWTileBytes;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t bdesc = ptx::sw128_kmajor_desc(sb + kk * 32);
                        const uint32_t acc = ((ks - k_beg) | kk) ? 1u : 0u;
                        ptx::tc_mma_bf16(d0, ptx::sw128_kmajor_desc(sa + kk * 32), bdesc, idesc,
                                         acc);
                        if (UP)
                            ptx::tc_mma_bf16(d0 + BN,
                                             ptx::sw128_kmajor_desc(sa + kWTileBytes + kk * 32),
                                             bdesc, idesc, acc);
                    }
                    ptx::tc_commit(&empty[stage]);
                    if (++stage == static_cast<uint32_t>(C::kStages)) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!stop) ptx::tc_commit(&tfull[buf]);
            }
            // Every MMA issued above has finished once this arrives.
            ptx::tc_commit(drain);
            drain_wait(drain, 0u);
        }
    } else {
        const int q = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
        int i = 0;
        for (int u = blockIdx.x; u < total; u += gridDim.x, ++i) {
            const Unit w = decode_unit<BN>(u, s_pre, s_off, E, KSPLIT);
            const int buf = i & 1;
            const uint32_t use = static_cast<uint32_t>(i >> 1);
            if (!bounded_wait_warp(&tfull[buf], use & 1u, abort_flag, p.err, kErrTimeoutMma))
                break;
            ptx::tc_fence_after();
            const int f = w.mb * 128 + 32 * q + lane;  // output column of this thread
            const uint32_t tb = tmem + lane_base + static_cast<uint32_t>(buf * C::kAccCols);
            for (int c0 = 0; c0 < w.valid; c0 += 32) {
                if (UP) {
                    uint32_t a[32], b[32];
                    ptx::tmem_ld32(tb + static_cast<uint32_t>(c0), a);
                    ptx::tmem_ld32(tb + static_cast<uint32_t>(BN + c0), b);
                    ptx::tc_wait_ld();
                    __nv_bfloat16 *H = static_cast<__nv_bfloat16 *>(p.out);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (c0 + j < w.valid) {
                            const float g = __uint_as_float(a[j]);
                            const float h = g * __frcp_rn(1.0f + __expf(-g)) * __uint_as_float(b[j]);
                            H[static_cast<size_t>(w.r0 + c0 + j) * p.M_rows + f] =
                                __float2bfloat16_rn(h);
                        }
                    }
                } else {
                    uint32_t y[32];
                    ptx::tmem_ld32(tb + static_cast<uint32_t>(c0), y);
                    ptx::tc_wait_ld();
                    float *Y = static_cast<float *>(p.out) + w.ks * p.part_stride;
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (c0 + j < w.valid)
                            Y[static_cast<size_t>(w.r0 + c0 + j) * p.M_rows + f] =
                                __uint_as_float(y[j]);
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&tempty[buf]);
        }
    }

    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <bool UP, int BN, int ST>
cudaError_t launch_gemm_cfg(const GemmLaunch &a, cudaStream_t s)
{
    using C = Cfg<UP, BN, ST>;
    CUtensorMap tA0, tA1, tB;
    cudaError_t e = make_tmap_bf16(&tA0, a.A0, static_cast<uint64_t>(a.E) * a.M_rows, a.K, 128);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16(&tA1, UP ? a.A1 : a.A0, static_cast<uint64_t>(a.E) * a.M_rows, a.K, 128);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16(&tB, a.B, a.S, a.K, BN);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(gemm_kernel<UP, BN, ST>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(C::kSmem));
    if (e != cudaSuccess) return e;

    GemmParams p;
    p.E = a.offsets ? a.E : 1;
    p.M_rows = a.M_rows;
    p.K = a.K;
    p.S = a.S;
    p.offsets = a.offsets;
    p.out = a.out;
    p.err = a.err;
    p.stream_weights = a.max_rows <= BN ? 1 : 0;
    p.ksplit = UP ? 1 : (a.ksplit < 1 ? 1 : a.ksplit);
    p.part_stride = static_cast<size_t>(a.S) * a.M_rows;
    // Upper bound of the work units: every segment rounds up to whole tiles.
    const long long tiles = (static_cast<long long>(a.S) + BN - 1) / BN + p.E;
    const long long units = tiles * (a.M_rows / 128) * p.ksplit;
    long long grid = device_sm_count();
    if (units < grid) grid = units;
    if (grid < 1) grid = 1;
    return launch_pdl(gemm_kernel<UP, BN, ST>, dim3(static_cast<unsigned>(grid)),
                      dim3(kGemmThreads), C::kSmem, s, a.pdl, tA0, tA1, tB, p);
}

}  // namespace

int gemm_token_tile(int up, int S, int E_seg)
{
    // Token tile from the average rows per segment: small tiles waste no
    // MMA columns and leave room for a deeper weight pipeline.
    const long long avg = (static_cast<long long>(S) + E_seg - 1) / E_seg;
    if (avg <= 32) return 32;
    if (avg <= 64) return 64;
    if (up || avg <= 128) return 128;
    return 256;
}

int down_ksplit(int S, int E_seg, int d, int d_ff)
{
    // Split K of the down projection when its (segment x weight block) units
    // cannot fill the GPU: pick the split whose unit count fills whole waves
    // of the SMs best, keeping at least 8 K steps per range.
    const int bn = gemm_token_tile(0, S, E_seg);
    const long long hit = std::min<long long>(E_seg, S);
    const long long units = (d / 128) * std::max<long long>(hit, (S + bn - 1) / bn);
    const long long sms = 148;
    if (units >= 2 * sms) return 1;
    const int max_ks = std::max(1, std::min(8, d_ff / 64 / 8));  // 8: the combine sums at most 8 partials
    int best = 1;
    double best_eff = 0.0;
    for (int ks = 1; ks <= max_ks; ++ks) {
        const long long u = units * ks;
        const long long waves = (u + sms - 1) / sms;
        const double eff = static_cast<double>(u) / static_cast<double>(waves * sms);
        if (eff > best_eff + 0.02) {
            best = ks;
            best_eff = eff;
        }
    }
    return best;
}

cudaError_t launch_gemm(const GemmLaunch &a, cudaStream_t s)
{
    const int bn = gemm_token_tile(a.up, a.S, a.offsets ? a.E : 1);
    if (a.up) {
        switch (bn) {
        case 32: return launch_gemm_cfg<true, 32, 5>(a, s);
        case 64: return launch_gemm_cfg<true, 64, 5>(a, s);
        default: return launch_gemm_cfg<true, 128, 4>(a, s);
        }
    }
    switch (bn) {
    case 32: return launch_gemm_cfg<false, 32, 10>(a, s);
    case 64: return launch_gemm_cfg<false, 64, 8>(a, s);
    case 128: return launch_gemm_cfg<false, 128, 6>(a, s);
    default: return launch_gemm_cfg<false, 256, 4>(a, s);
    }
}

}  // namespace moe
