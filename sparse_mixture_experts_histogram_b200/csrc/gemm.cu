// gemm.cu -- the experts' feed-forward as one persistent kernel on the
// 5th-generation tensor cores (tcgen05 MMA, accumulators in tensor memory,
// operands brought in by TMA).
//
// For every expert segment e (rows offsets[e] .. offsets[e+1]-1 of x_perm):
//   up units:   D0 = W1_e[blk] X^T, D1 = W3_e[blk] X^T   (128 weight rows)
//               H[r, blk] = bf16( silu(D0) * D1 )         -- SwiGLU epilogue
//   down units: D0 = W2_e[2m] H^T, D1 = W2_e[2m+1] H^T   (two 128-row blocks)
//               Y[ks][r, 2m], Y[ks][r, 2m+1] = D0, D1      -- fp32, K range ks
// The weights are the MMA's A operand (M = 128 weight rows) and the segment's
// rows its B operand (N = rows, rounded up to 16), so a ragged or tiny
// segment costs only the columns it needs and small batches stream each hit
// expert's weights once.  Both kinds of unit load two 128-row weight tiles and
// one token tile per 64-wide K step, so they share one pipeline.
//
// One CTA per SM.  Warp 0 issues TMA copies into a ring of shared-memory
// stages, warp 1 issues the MMAs into a double-buffered tensor-memory
// accumulator, warps 2..5 drain finished accumulators and store.  Every CTA
// walks the units numbered up-first (expert, block, token tile) and then
// down (expert, block pair, token tile, K range).  A down unit reads, per K
// step, 64 columns of its token tile's H: the up epilogues mark each finished
// (token tile, 128-column block) of H, and the producer waits (bounded) for
// that mark before it copies the columns -- after it has already issued the
// step's W2 copies.  A unit only ever waits for units numbered before it, and
// every CTA takes its units in increasing order, so the lowest unfinished
// unit can always proceed: the waits always end.  Down work starts on the
// first finished H blocks while later up blocks are still running.
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

constexpr int kFfnThreads = 192;
constexpr int kMaxStages = 8;
constexpr uint32_t kWTile = 128 * 128;  // 128 weight rows x 64 bf16 = 16 KB
constexpr int kSlots = 4;  // unit-number ring (see ffn_kernel)
constexpr size_t kFixedSmem = 1024 /* alignment slack */ + (2 * kMaxStages + 5 + 2 * kSlots) * 8 +
                              4 * kSlots + 16 + 4 * (kMaxE + 1) * sizeof(int32_t) + 64;
constexpr size_t kSmemBudget = 227 * 1024;

template <int BN, int ST>
struct FfnCfg {
    static constexpr uint32_t kStageBytes = 2 * kWTile + BN * 128u;
    static constexpr int kAccCols = 2 * BN;  // accumulators D0 and D1 side by side
    static constexpr uint32_t kTmemCols = 2u * kAccCols;
    static constexpr size_t kSmem = kFixedSmem + static_cast<size_t>(ST) * kStageBytes;
    static_assert(kTmemCols >= 32 && kTmemCols <= 512 && (kTmemCols & (kTmemCols - 1)) == 0,
                  "tensor memory allocation must be a power of two in [32, 512]");
    static_assert(ST >= 2 && ST <= kMaxStages, "pipeline depth");
    static_assert(kSmem <= kSmemBudget, "shared memory");
    // One CTA per SM: the shared memory keeps a second CTA (and its tensor
    // memory allocation) off the SM.
    static_assert(kSmem > kSmemBudget / 2, "one CTA per SM");
};

struct FfnParams {
    int E;                  // segments
    int d, d_ff;
    int S;                  // rows of x_perm / H / Y
    int ksplit;             // K ranges of the down projection
    size_t part_stride;     // floats between the partial outputs of consecutive K ranges
    const int32_t *offsets; // [E+1] or nullptr (one segment [0, S))
    __nv_bfloat16 *H;       // [S, d_ff]
    float *Y;               // [ksplit, S, d]
    uint32_t *h_ready;      // [tiles, d_ff/128]: epilogue warps done with (token tile, H block)
    uint32_t *err;
    int stream_weights;     // each weight block feeds one token tile: L2 evict-first
    int act;                // expert activation: 0 silu(g) * b, 1 sigmoid(g) * b
    uint32_t *sched;        // unit counter, zero before the launch; or nullptr: static order
};

struct Unit {
    bool up;
    int e, blk, r0, valid, tile, k_beg, k_end, ks;
};

template <int BN>
__device__ __forceinline__ Unit decode_unit(int u, int u_up, const int32_t *s_off,
                                            const int32_t *s_pu, const int32_t *s_pd,
                                            const int32_t *s_tb, int E, int ksplit, int ksu,
                                            int ksd)
{
    Unit w;
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

__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity)
{
    const uint64_t t0 = ptx::globaltimer();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::globaltimer() - t0 > 100000000ull) break;  // 100 ms
    }
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void fence_proxy_async_global()
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Waits until *ctr >= target (written by other CTAs' epilogues).  Bounded
// like the pipeline waits: gives up after kWaitTimeoutNs or when another role
// of this CTA has given up.
__device__ __forceinline__ bool wait_counter(const uint32_t *ctr, uint32_t target,
                                             volatile uint32_t *abort_flag, uint32_t *gerr)
{
    if (ld_acquire(ctr) >= target) return true;
    const uint64_t t0 = ptx::globaltimer();
    for (uint32_t it = 1;; ++it) {
        __nanosleep(64);
        if (ld_acquire(ctr) >= target) return true;
        if (*abort_flag) return false;
        if ((it & 15u) == 0 && ptx::globaltimer() - t0 > kWaitTimeoutNs) {
            *abort_flag = 1u;
            if (gerr) atomicOr(gerr, kErrTimeoutEpi);
            return false;
        }
    }
}

__device__ __forceinline__ int warp_incl_scan(int v, int lane)
{
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += n;
    }
    return v;
}

template <int BN, int ST>
__global__ void __launch_bounds__(kFfnThreads, 1)
    ffn_kernel(const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmW3,
               const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmX,
               const __grid_constant__ CUtensorMap tmH, const FfnParams p)
{
    using C = FfnCfg<BN, ST>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    uint64_t *full = reinterpret_cast<uint64_t *>(smem + ST * C::kStageBytes);
    uint64_t *empty = full + kMaxStages;
    uint64_t *tfull = empty + kMaxStages;  // [2]
    uint64_t *tempty = tfull + 2;          // [2]
    uint64_t *drain = tempty + 2;          // [1]
    uint64_t *sfull = drain + 1;           // [kSlots] unit number posted
    uint64_t *sempty = sfull + kSlots;     // [kSlots] read by the MMA thread and 4 epilogue warps
    uint32_t *sched_id = reinterpret_cast<uint32_t *>(sempty + kSlots);  // [kSlots]
    uint32_t *tmem_slot = sched_id + kSlots;
    volatile uint32_t *abort_flag = tmem_slot + 1;
    int32_t *s_off = reinterpret_cast<int32_t *>(tmem_slot + 4);
    int32_t *s_pu = s_off + (kMaxE + 1);   // up-unit prefix per expert
    int32_t *s_pd = s_pu + (kMaxE + 1);    // down-unit prefix per expert
    int32_t *s_tb = s_pd + (kMaxE + 1);    // token-tile prefix per expert

    const int E = p.offsets ? p.E : 1;
    const int MBU = p.d_ff / 128;          // up weight blocks per expert
    const int MBD = (p.d + 255) / 256;     // down weight block pairs per expert
    const int KSU = p.d / 64;
    const int KSD = p.d_ff / 64;
    const int KSPLIT = p.ksplit;
    const uint32_t ready_target = 4u;  // the four epilogue warps of the up unit

    if (threadIdx.x == 0) {
        for (int s = 0; s < ST; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&tfull[b], 1);
            ptx::mbar_init(&tempty[b], 4);  // one arrival per epilogue warp
        }
        ptx::mbar_init(drain, 1);
        for (int k = 0; k < kSlots; ++k) {
            ptx::mbar_init(&sfull[k], 1);
            ptx::mbar_init(&sempty[k], 1 + 4);
        }
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
    // Everything above overlaps the previous kernel; from here on its results
    // (offsets, x_perm) are read and this kernel's outputs are written.
    ptx::grid_dep_wait();
    if (warp == 2) {
        // Segment table and the unit / tile prefixes per expert.
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
        bad = __any_sync(0xffffffffu, bad);
        if (bad) {
            nu = nd = nt = 0;
            if (lane == 0) atomicOr(p.err, kErrOffsets);
        }
        const int iu = warp_incl_scan(nu, lane);
        const int id = warp_incl_scan(nd, lane);
        const int it = warp_incl_scan(nt, lane);
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
            uint32_t last_parity[kMaxStages];
#pragma unroll
            for (int s = 0; s < kMaxStages; ++s) last_parity[s] = 0;
            const uint64_t pol_w =
                p.stream_weights ? ptx::policy_evict_first() : ptx::policy_evict_normal();
            bool stop = false;
            // Unit numbers.  With a counter and at least three units per
            // CTA, every unit comes from the counter (the next one fetched
            // while the current one is issued): CTAs that finish early take
            // more, and a down unit's H blocks come from units with smaller
            // numbers, taken earlier by CTAs that are running, so its waits
            // end whatever number of CTAs is resident.  With fewer units per
            // CTA (one or two experts at small batches) the fixed order
            // balances the coarse units better (measured): CTA b takes units
            // b, b + grid, ...  Either way the number is posted to the MMA
            // thread and the epilogue warps through the slot ring.
            const bool dyn = p.sched != nullptr && total >= 3 * static_cast<int>(gridDim.x);
            uint32_t next = dyn ? atomicAdd(p.sched, 1u) : blockIdx.x;
            for (uint32_t i = 0; !stop; ++i) {
                const uint32_t slot = i % kSlots;
                if (!bounded_wait(&sempty[slot], ((i / kSlots) & 1u) ^ 1u, abort_flag, p.err,
                                  kErrTimeoutEpi))
                    break;
                const uint32_t uu = next;
                if (uu < static_cast<uint32_t>(total))
                    next = dyn ? atomicAdd(p.sched, 1u) : uu + gridDim.x;
                sched_id[slot] = uu;
                ptx::mbar_arrive(&sfull[slot]);
                if (uu >= static_cast<uint32_t>(total)) break;
                const int u = static_cast<int>(uu);
                const Unit w =
                    decode_unit<BN>(u, u_up, s_off, s_pu, s_pd, s_tb, E, KSPLIT, KSU, KSD);
                const CUtensorMap *ta0 = w.up ? &tmW1 : &tmW2;
                const CUtensorMap *ta1 = w.up ? &tmW3 : &tmW2;
                const CUtensorMap *tb = w.up ? &tmX : &tmH;
                const int arow0 = w.up ? w.e * p.d_ff + w.blk * 128 : w.e * p.d + w.blk * 256;
                const int arow1 = w.up ? arow0 : arow0 + 128;
                int ready_blk = -1;
                int win = -1;        // first H block of the readiness window
                uint32_t wmask = 0;  // blocks of the window found ready
                for (int ks = w.k_beg; ks < w.k_end; ++ks) {
                    if (!bounded_wait(&empty[stage], phase ^ 1u, abort_flag, p.err,
                                      kErrTimeoutMma)) {
                        stop = true;
                        break;
                    }
                    uint8_t *sa = smem + stage * C::kStageBytes;
                    ptx::mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
                    ptx::tma_load_2d_hint(sa, ta0, &full[stage], ks * 64, arow0, pol_w);
                    ptx::tma_load_2d_hint(sa + kWTile, ta1, &full[stage], ks * 64, arow1, pol_w);
                    issued |= 1u << stage;
                    last_parity[stage] = phase;
                    if (!w.up && (ks >> 1) != ready_blk) {
                        // These 64 columns of H belong to 128-column block ks/2:
                        // wait until its up unit has stored and published it.
                        ready_blk = ks >> 1;
                        if (win < 0 || ready_blk >= win + 32) {
                            win = ready_blk;
                            const int nb = ((w.k_end + 1) >> 1) - ready_blk;
                            wmask = ready_window(&p.h_ready[w.tile * MBU + ready_blk],
                                                 nb < 32 ? nb : 32, ready_target);
                        }
                        if (!((wmask >> (ready_blk - win)) & 1u) &&
                            !wait_counter(&p.h_ready[w.tile * MBU + ready_blk], ready_target,
                                          abort_flag, p.err)) {
                            stop = true;
                            break;
                        }
                        fence_proxy_async_global();
                    }
                    ptx::tma_load_2d(sa + 2 * kWTile, tb, &full[stage], ks * 64, w.r0);
                    if (++stage == static_cast<uint32_t>(ST)) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // Make sure no copy is still landing in shared memory at exit.
            for (int s = 0; s < ST; ++s)
                if (issued & (1u << s)) drain_wait(&full[s], last_parity[s]);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            bool stop = false;
            for (uint32_t i = 0; !stop; ++i) {
                const uint32_t slot = i % kSlots;
                if (!bounded_wait(&sfull[slot], (i / kSlots) & 1u, abort_flag, p.err, kErrTimeoutEpi))
                    break;
                const uint32_t uu = *reinterpret_cast<volatile uint32_t *>(&sched_id[slot]);
                ptx::mbar_arrive(&sempty[slot]);
                if (uu >= static_cast<uint32_t>(total)) break;
                const int u = static_cast<int>(uu);
                const Unit w =
                    decode_unit<BN>(u, u_up, s_off, s_pu, s_pd, s_tb, E, KSPLIT, KSU, KSD);
                const int n = ((w.valid + 15) >> 4) << 4;
                const uint32_t idesc = ptx::idesc_bf16_f32(128, n);
                const int buf = i & 1;
                const uint32_t use = static_cast<uint32_t>(i >> 1);
                if (!bounded_wait(&tempty[buf], (use & 1u) ^ 1u, abort_flag, p.err,
                                  kErrTimeoutEpi))
                    break;
                ptx::tc_fence_after();
                const uint32_t d0 = tmem + static_cast<uint32_t>(buf * C::kAccCols);
                for (int ks = w.k_beg; ks < w.k_end; ++ks) {
                    if (!bounded_wait(&full[stage], phase, abort_flag, p.err, kErrTimeoutTma)) {
                        stop = true;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t sa = ptx::smem_addr(smem + stage * C::kStageBytes);
                    const uint32_t sb = sa + 2 * kWTile;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t bdesc = ptx::sw128_kmajor_desc(sb + kk * 32);
                        const uint32_t acc = ((ks - w.k_beg) | kk) ? 1u : 0u;
                        ptx::tc_mma_bf16(d0, ptx::sw128_kmajor_desc(sa + kk * 32), bdesc, idesc,
                                         acc);
                        ptx::tc_mma_bf16(d0 + BN, ptx::sw128_kmajor_desc(sa + kWTile + kk * 32),
                                         bdesc, idesc, acc);
                    }
                    ptx::tc_commit(&empty[stage]);
                    if (++stage == static_cast<uint32_t>(ST)) {
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
        for (uint32_t i = 0;; ++i) {
            const uint32_t slot = i % kSlots;
            if (!bounded_wait_warp(&sfull[slot], (i / kSlots) & 1u, abort_flag, p.err,
                                   kErrTimeoutEpi))
                break;
            const uint32_t uu = *reinterpret_cast<volatile uint32_t *>(&sched_id[slot]);
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&sempty[slot]);
            if (uu >= static_cast<uint32_t>(total)) break;
            const int u = static_cast<int>(uu);
            const Unit w = decode_unit<BN>(u, u_up, s_off, s_pu, s_pd, s_tb, E, KSPLIT, KSU, KSD);
            const int buf = i & 1;
            const uint32_t use = static_cast<uint32_t>(i >> 1);
            if (!bounded_wait_warp(&tfull[buf], use & 1u, abort_flag, p.err, kErrTimeoutMma))
                break;
            ptx::tc_fence_after();
            const uint32_t tb = tmem + lane_base + static_cast<uint32_t>(buf * C::kAccCols);
            const int row_in_blk = 32 * q + lane;
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
                            const float g = __uint_as_float(a[j]);
                            const float bv = __uint_as_float(b[j]);
                            const float h = __fdividef(p.act ? bv : g * bv, 1.0f + __expf(-g));
                            p.H[static_cast<size_t>(w.r0 + c0 + j) * p.d_ff + f] =
                                __float2bfloat16_rn(h);
                        }
                    }
                } else {
                    const int o0 = w.blk * 256 + row_in_blk;
                    const bool has1 = o0 + 128 < p.d;
                    float *Y = p.Y + w.ks * p.part_stride;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (c0 + j < w.valid) {
                            float *yr = Y + static_cast<size_t>(w.r0 + c0 + j) * p.d;
                            yr[o0] = __uint_as_float(a[j]);
                            if (has1) yr[o0 + 128] = __uint_as_float(b[j]);
                        }
                    }
                }
            }
            ptx::tc_fence_before();
            if (w.up) {
                // Publish this warp's slice of the H block to the down units
                // (which read it through TMA, the async proxy).
                fence_proxy_async_global();
                __threadfence();
            }
            __syncwarp();
            if (lane == 0) {
                if (w.up) atomicAdd(&p.h_ready[w.tile * MBU + w.blk], 1u);
                ptx::mbar_arrive(&tempty[buf]);
            }
        }
    }

    // Dependents (the shared expert, the combine) need this kernel's results:
    // let them launch only once its work is done.
    ptx::grid_dep_launch();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int BN, int ST>
cudaError_t launch_ffn_cfg(const FfnLaunch &a, cudaStream_t s)
{
    using C = FfnCfg<BN, ST>;
    const int E = a.offsets ? a.E : 1;
    CUtensorMap tW1, tW3, tW2, tX, tH;
    cudaError_t e = make_tmap_bf16(&tW1, a.W1, static_cast<uint64_t>(E) * a.d_ff, a.d, 128);
    if (e == cudaSuccess) e = make_tmap_bf16(&tW3, a.W3, static_cast<uint64_t>(E) * a.d_ff, a.d, 128);
    if (e == cudaSuccess) e = make_tmap_bf16(&tW2, a.W2, static_cast<uint64_t>(E) * a.d, a.d_ff, 128);
    if (e == cudaSuccess) e = make_tmap_bf16(&tX, a.x, a.S, a.d, BN);
    if (e == cudaSuccess) e = make_tmap_bf16(&tH, a.H, a.S, a.d_ff, BN);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(ffn_kernel<BN, ST>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(C::kSmem));
    if (e != cudaSuccess) return e;

    FfnParams p{};
    p.E = E;
    p.d = a.d;
    p.d_ff = a.d_ff;
    p.S = a.S;
    p.ksplit = a.ksplit < 1 ? 1 : a.ksplit;
    p.part_stride = static_cast<size_t>(a.S) * a.d;
    p.offsets = a.offsets;
    p.H = reinterpret_cast<__nv_bfloat16 *>(a.H);
    p.Y = a.Y;
    p.h_ready = a.h_ready;
    p.err = a.err;
    p.stream_weights = a.max_rows <= BN ? 1 : 0;
    p.act = a.act;
    p.sched = a.sched;
    // Upper bound of the work units: every segment rounds up to whole tiles.
    const long long tiles = (static_cast<long long>(a.S) + BN - 1) / BN + E;
    const long long units = tiles * (a.d_ff / 128) + tiles * ((a.d + 255) / 256) * p.ksplit;
    long long grid = device_sm_count();
    if (units < grid) grid = units;
    if (grid < 1) grid = 1;
    return launch_pdl(ffn_kernel<BN, ST>, dim3(static_cast<unsigned>(grid)), dim3(kFfnThreads),
                      C::kSmem, s, a.pdl, tW1, tW3, tW2, tX, tH, p);
}

}  // namespace

int ffn_token_tile(int S, int E_seg)
{
    // Token tile from the rows a segment is expected to hold (1.5x the
    // average, so that few segments spill into a second, mostly empty tile
    // that streams the same weights again); small tiles waste no MMA columns
    // and leave room for a deeper weight pipeline.
    const long long expect = (3LL * S + 2LL * E_seg - 1) / (2LL * E_seg);
    if (expect <= 32) return 32;
    if (expect <= 64) return 64;
    return 128;
}

size_t ffn_ready_counters(int S, int E_seg, int d_ff)
{
    // One counter per (token tile, 128-column block of H); tiles are at least
    // 32 rows and every segment adds at most one partial tile.
    return static_cast<size_t>((S + 31) / 32 + E_seg) * static_cast<size_t>(d_ff / 128);
}

int down_ksplit(int S, int E_seg, int d, int d_ff)
{
    // Split K of the down projection when its (segment x weight block pair)
    // units cannot fill the GPU once: pick the split whose unit count fills
    // whole waves of the SMs best, keeping at least 8 K steps per range.
    const int bn = ffn_token_tile(S, E_seg);
    const long long hit = std::min<long long>(E_seg, S);
    const long long units = ((d + 255) / 256) * std::max<long long>(hit, (S + bn - 1) / bn);
    const long long sms = 148;
    if (units >= sms) return 1;
    const int max_ks = std::max(1, std::min(8, d_ff / 64 / 8));
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

cudaError_t launch_ffn(const FfnLaunch &a, cudaStream_t s)
{
    const int rows = a.S_hint > 0 ? a.S_hint : a.S;
    if (a.sched != nullptr && ffn_pair_eligible(rows, a.offsets ? a.E : 1, a.ksplit))
        return launch_ffn_pair(a, a.sched, s);
    if (a.out != nullptr || a.y_bf16) return cudaErrorInvalidValue;  // pair kernel only
    switch (ffn_token_tile(rows, a.offsets ? a.E : 1)) {
    case 32: return launch_ffn_cfg<32, 6>(a, s);
    case 64: return launch_ffn_cfg<64, 5>(a, s);
    default: return launch_ffn_cfg<128, 4>(a, s);
    }
}

}  // namespace moe
