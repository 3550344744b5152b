// route.cu -- router kernel: logits = x Wg^T on the tensor cores (tcgen05,
// accumulators in tensor memory, operands brought in by TMA), then in the
// epilogue the per-token top-k (ties to the lower expert index), the softmax
// over the k selected logits, the per-tile expert histogram with stable
// ranks, and -- in the last tile to finish -- the expert offsets.
//
// One CTA routes 128 tokens (the MMA's M).  Warp 0 issues TMA loads, warp 1
// issues the MMAs, warps 2..5 are the epilogue (thread = token row).
//
// Method: "Mistral 8x7B SMoE architecture" (jsqmd.com) sec. 3.2, the gate
// linear followed by torch.topk and a softmax over the selected values;
// "MoE" (theaiera.top, LLMs-from-scratch ch.10) sec. 10.3 (weights sum to
// 1) and sec. 10.4 (per-expert token lists, here the histogram).
#include <cuda_runtime.h>
#include <math_constants.h>

#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace moe {

namespace {

constexpr int kRouteMaxStages = 8;
constexpr int kRouteThreads = 192;
constexpr uint32_t kRouteABytes = 128 * 128;   // 128 token rows x 64 bf16

struct RouteParams {
    int T, d, E, Npad, stages, ntiles;
    int wmode;      // gate weights: 0 softmax over the selected, 1 softmax over all, 2 sigmoid,
                    // 3 tempered softmax over all with entropy-controlled k
    uint32_t tmem_cols;
    const float *bias;
    int32_t *idx;
    float *w;
    uint32_t *err;
    DispatchOut dout;
    int slots;      // slot mode: assign_slots instead of dispatch_tile
    SlotOut sout;
};

__host__ __device__ constexpr uint32_t route_stage_bytes(int Npad)
{
    return kRouteABytes + static_cast<uint32_t>(Npad) * 128u;
}

constexpr size_t kRouteFixedSmem = 1024 /* alignment slack */ + 2 * kRouteMaxStages * 8 + 8 + 16 +
                                   kMaxE * sizeof(float) + sizeof(DispatchSmem) + 64;

void fill_slots(const RouteLaunch &a, int *slots, SlotOut *o)
{
    *slots = a.slot_pos != nullptr ? 1 : 0;
    o->gcnt = a.gcnt;
    o->pos = a.slot_pos;
    o->perm = a.perm;
    o->perm_stride = a.perm_stride;
}

template <int K>
__device__ __forceinline__ void topk_insert(float (&tv)[K], int (&ti)[K], float v, int e)
{
    if (v > tv[K - 1]) {
#pragma unroll
        for (int j = K - 1; j > 0; --j) {
            if (v > tv[j]) {
                if (v > tv[j - 1]) {
                    tv[j] = tv[j - 1];
                    ti[j] = ti[j - 1];
                } else {
                    tv[j] = v;
                    ti[j] = e;
                }
            }
        }
        if (v > tv[0]) {
            tv[0] = v;
            ti[0] = e;
        }
    }
}

// Gate weights of the k selected logits tv[0..K) (descending):
//   wmode 0: softmax over the selected logits (the method)
//   wmode 1: softmax over all E logits, given their maximum m_all and
//            sum_all = sum_e exp(l_e - m_all); not renormalised over the
//            selected ("Mixtral 8x7B模型架构解析" Router.forward)
//   wmode 2: the sigmoid of each selected logit ("万亿 MoE" forward listing)
//   wmode 3: the softmax of l / tau over all E logits (tau = 0.1), given
//            m_all and sum_all = sum_e exp((l_e - m_all) / tau), not
//            renormalised ("Mixtral 8x7B模型架构解析" entropy_aware_routing)
constexpr float kEntropyInvTau = 10.0f;     // 1 / tau, tau = 0.1
constexpr float kEntropyThreshold = 0.8f;   // nats

template <int K>
__device__ __forceinline__ void gate_weights(const float (&tv)[K], int wmode, float m_all,
                                             float sum_all, float (&w)[K])
{
    if (wmode == 3) {
#pragma unroll
        for (int j = 0; j < K; ++j) w[j] = expf((tv[j] - m_all) * kEntropyInvTau) / sum_all;
    } else if (wmode == 1) {
#pragma unroll
        for (int j = 0; j < K; ++j) w[j] = expf(tv[j] - m_all) / sum_all;
    } else if (wmode == 2) {
#pragma unroll
        for (int j = 0; j < K; ++j) w[j] = 1.0f / (1.0f + expf(-tv[j]));
    } else {
        float s = 0.0f;
#pragma unroll
        for (int j = 0; j < K; ++j) {
            w[j] = expf(tv[j] - tv[0]);
            s += w[j];
        }
#pragma unroll
        for (int j = 0; j < K; ++j) w[j] = w[j] / s;
    }
}

// Slots a token keeps under wmode 3: K when the entropy of the tempered
// softmax exceeds the threshold, K - 1 otherwise.  With Z = sum_e
// exp((l_e - m) / tau) and A = sum_e exp((l_e - m) / tau) (l_e - m), the
// entropy -sum_e p_e ln p_e of p_e = exp((l_e - m) / tau) / Z is
// ln Z - A / (tau Z).
template <int K>
__device__ __forceinline__ int entropy_slots(float z, float a)
{
    const float h = logf(z) - a * kEntropyInvTau / z;
    return h > kEntropyThreshold ? K : K - 1;
}


// Waits for the copies the producer issued into each stage to land, so that
// no copy is still writing shared memory when the CTA exits after an abort.
__device__ __forceinline__ void drain_stages(uint64_t *full, const uint32_t *last_parity,
                                             uint32_t issued_mask, int stages)
{
    for (int s = 0; s < stages; ++s) {
        if (!(issued_mask & (1u << s))) continue;
        const uint64_t t0 = ptx::globaltimer();
        while (!ptx::mbar_try_wait(&full[s], last_parity[s])) {
            if (ptx::globaltimer() - t0 > 100000000ull) break;  // 100 ms
        }
    }
}

template <int K>
__global__ void __launch_bounds__(kRouteThreads, 1)
    route_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmWg,
                 const RouteParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t stage_bytes = route_stage_bytes(p.Npad);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.stages * stage_bytes);
    uint64_t *empty = full + kRouteMaxStages;
    uint64_t *tfull = empty + kRouteMaxStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tfull + 1);
    volatile uint32_t *abort_flag = tmem_slot + 1;
    uint32_t *epi_fail = tmem_slot + 2;
    float *bias_s = reinterpret_cast<float *>(tmem_slot + 4);
    DispatchSmem &ds = *reinterpret_cast<DispatchSmem *>(bias_s + kMaxE);

    const int tile = blockIdx.x;
    const int ksteps = p.d / 64;

    ptx::grid_dep_launch();
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        ptx::mbar_init(tfull, 1);
        *abort_flag = 0u;
        *epi_fail = 0u;
        ptx::fence_barrier_init();
    }
    if (threadIdx.x == 32) {
        ptx::prefetch_tensormap(&tmX);
        ptx::prefetch_tensormap(&tmWg);
    }
    for (int e = threadIdx.x; e < kMaxE; e += blockDim.x)
        bias_s[e] = (p.bias != nullptr && e < p.E) ? p.bias[e] : 0.0f;
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, p.tmem_cols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            uint32_t stage = 0, phase = 0, issued = 0;
            uint32_t last_parity[kRouteMaxStages];
            for (int s = 0; s < kRouteMaxStages; ++s) last_parity[s] = 0;
            for (int ks = 0; ks < ksteps; ++ks) {
                if (!bounded_wait(&empty[stage], phase ^ 1u, abort_flag, p.err, kErrTimeoutMma))
                    break;
                uint8_t *sa = smem + stage * stage_bytes;
                ptx::mbar_arrive_expect_tx(&full[stage], stage_bytes);
                ptx::tma_load_2d(sa, &tmX, &full[stage], ks * 64, tile * kTileTokens);
                ptx::tma_load_2d(sa + kRouteABytes, &tmWg, &full[stage], ks * 64, 0);
                issued |= 1u << stage;
                last_parity[stage] = phase;
                if (++stage == static_cast<uint32_t>(p.stages)) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            drain_stages(full, last_parity, issued, p.stages);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = ptx::idesc_bf16_f32(128, p.Npad);
            uint32_t stage = 0, phase = 0;
            for (int ks = 0; ks < ksteps; ++ks) {
                if (!bounded_wait(&full[stage], phase, abort_flag, p.err, kErrTimeoutTma)) break;
                ptx::tc_fence_after();
                const uint32_t sa = ptx::smem_addr(smem + stage * stage_bytes);
                const uint32_t sb = sa + kRouteABytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    ptx::tc_mma_bf16(tmem, ptx::sw128_kmajor_desc(sa + kk * 32),
                                     ptx::sw128_kmajor_desc(sb + kk * 32), idesc,
                                     (ks | kk) ? 1u : 0u);
                ptx::tc_commit(&empty[stage]);
                if (++stage == static_cast<uint32_t>(p.stages)) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            // Arrives once every MMA issued above has completed (also after
            // an abort, so the epilogue never reads half-written tensor memory
            // while MMAs still run).
            ptx::tc_commit(tfull);
        }
    } else {
        const int q = warp & 3;
        const int row = 32 * q + lane;
        const int t = tile * kTileTokens + row;
        const bool ok_w = bounded_wait_warp(tfull, 0u, abort_flag, p.err, kErrTimeoutMma);
        if (lane == 0 && !ok_w) atomicOr(epi_fail, 1u);
        ptx::named_bar(1, 128);
        const bool ok = (*reinterpret_cast<volatile uint32_t *>(epi_fail) == 0u);
        ptx::tc_fence_after();

        float tv[K];
        int ti[K];
#pragma unroll
        for (int j = 0; j < K; ++j) {
            tv[j] = -CUDART_INF_F;
            ti[j] = -1;
        }
        // Running maximum and sum of exp(l - max) over all E logits (for the
        // softmax over all experts).
        float run_m = -CUDART_INF_F, run_s = 0.0f, run_a = 0.0f;
        if (ok) {
            const uint32_t tbase = tmem + (static_cast<uint32_t>(32 * q) << 16);
            for (int c0 = 0; c0 < p.Npad; c0 += 16) {
                uint32_t r[16];
                ptx::tmem_ld16(tbase + static_cast<uint32_t>(c0), r);
                ptx::tc_wait_ld();
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    const int e = c0 + jj;
                    // A NaN logit (only from non-finite inputs) ranks like -inf.
                    const float l0 = __uint_as_float(r[jj]) + bias_s[e];
                    const float l = (l0 == l0) ? l0 : -CUDART_INF_F;
                    if (e < p.E) {
                        topk_insert<K>(tv, ti, l, e);
                        if (p.wmode == 1 && l > -CUDART_INF_F) {
                            if (l > run_m) {
                                run_s = run_s * expf(run_m - l) + 1.0f;
                                run_m = l;
                            } else {
                                run_s += expf(l - run_m);
                            }
                        } else if (p.wmode == 3 && l > -CUDART_INF_F) {
                            // Tempered running sum Z and A = sum exp(.)(l - m),
                            // both rescaled when the maximum moves.
                            if (run_s == 0.0f) {
                                run_m = l;
                                run_s = 1.0f;
                            } else if (l > run_m) {
                                const float f = expf((run_m - l) * kEntropyInvTau);
                                run_a = f * (run_a + run_s * (run_m - l));
                                run_s = run_s * f + 1.0f;
                                run_m = l;
                            } else {
                                const float q = expf((l - run_m) * kEntropyInvTau);
                                run_s += q;
                                run_a += q * (l - run_m);
                            }
                        }
                    }
                }
            }
            // Logits equal to -inf (or NaN) are never inserted; the slots they
            // leave empty all hold -inf, so -- ties going to the lower index --
            // they take the lowest experts not yet selected, in order.  Every
            // slot then holds a distinct expert in [0, E) (k <= E), the same
            // choice the CUDA-core router makes.
            int cand = 0;
#pragma unroll
            for (int j = 0; j < K; ++j) {
                if (ti[j] < 0) {
                    bool used = true;
                    while (used) {
                        used = false;
#pragma unroll
                        for (int jj = 0; jj < K; ++jj) used |= (ti[jj] == cand);
                        if (used) ++cand;
                    }
                    ti[j] = cand++;
                }
            }
        }
        ptx::tc_fence_before();

        const bool valid = ok && (t < p.T);
        // Slots in use: all K, or K - 1 under the entropy rule (the last
        // slot then holds expert -1 and weight 0).
        const int ku = p.wmode == 3 ? entropy_slots<K>(run_s, run_a) : K;
        if (valid) {
            float wv[K];
            gate_weights<K>(tv, p.wmode, run_m, run_s, wv);
#pragma unroll
            for (int j = 0; j < K; ++j) {
                p.idx[static_cast<size_t>(t) * K + j] = j < ku ? ti[j] : -1;
                p.w[static_cast<size_t>(t) * K + j] = j < ku ? wv[j] : 0.0f;
            }
        }
#pragma unroll
        for (int j = 0; j < K; ++j) ds.sel[row][j] = (valid && j < ku) ? ti[j] : -1;
        if (p.slots)
            assign_slots(ds, tile * kTileTokens, kTileTokens, p.T, p.E, K, p.sout, row,
                         kTileTokens, 1);
        else
            dispatch_tile(ds, row, tile, p.T, p.E, K, p.dout, 1);
    }

    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, p.tmem_cols);
    }
}


// ---------------------------------------------------------------------------
// Router on the CUDA cores, for batches whose T*E*d is small (decode sizes,
// narrow layers): a tensor-core tile of 128 tokens would leave most SMs idle
// and wait on a long serial chain of copies.  One CTA takes kSmallTok tokens:
// their x rows go to shared memory, warp w computes the logits of experts
// e = w, w+8, ... for all of them (16-byte loads of Wg, fp32 FMA, warp
// reduction), then warp i selects token i's top-k by K rounds of a warp-wide
// (largest value, lowest index) reduction and applies the softmax.  The last
// CTA of every 128-token tile runs the same tile histogram / stable ranks /
// offsets step as the tensor-core router.
constexpr int kSmallTok = 4;
constexpr int kSmallThreads = 256;

struct SmallRouteParams {
    int T, d, E;
    int wmode;      // gate weights: 0 softmax over the selected, 1 softmax over all, 2 sigmoid,
                    // 3 tempered softmax over all with entropy-controlled k
    const uint4 *x;
    const uint4 *Wg;
    const float *bias;
    int32_t *idx;
    float *w;
    uint32_t *tile_ctr;
    DispatchOut dout;
    int slots;      // slot mode: assign_slots instead of the per-tile dispatch
    SlotOut sout;
};

// 8 bf16 (one 16-byte vector) to fp32, in element order.
__device__ __forceinline__ void unpack8(const uint4 &a, float (&f)[8])
{
    const uint32_t v[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(v[i] << 16);
        f[2 * i + 1] = __uint_as_float(v[i] & 0xffff0000u);
    }
}

size_t small_route_smem(int d)
{
    return static_cast<size_t>(kSmallTok) * d * 2 + kSmallTok * kMaxE * sizeof(float) +
           sizeof(DispatchSmem);
}

template <int K, int EPW, int U>
__global__ void __launch_bounds__(kSmallThreads) route_small_kernel(const SmallRouteParams p)
{
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ uint32_t s_last;
    const int nv = p.d >> 3;
    uint4 *sx = reinterpret_cast<uint4 *>(smem_raw);
    float *slog = reinterpret_cast<float *>(smem_raw + static_cast<size_t>(kSmallTok) * p.d * 2);
    DispatchSmem &ds = *reinterpret_cast<DispatchSmem *>(slog + kSmallTok * kMaxE);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * kSmallTok;
    const int nt = min(kSmallTok, p.T - t0);

    ptx::grid_dep_wait();
    ptx::grid_dep_launch();
    for (int i = threadIdx.x; i < kSmallTok * nv; i += kSmallThreads) {
        const int tt = i / nv;
        sx[i] = (tt < nt) ? __ldg(p.x + static_cast<size_t>(t0) * nv + i) : make_uint4(0, 0, 0, 0);
    }
    __syncthreads();

    // Warp w computes experts w*EPW .. w*EPW+EPW-1, then the next 8*EPW
    // experts; each lane keeps U*EPW 16-byte loads of Wg in flight.
    // Every CTA reads all of Wg; starting each CTA at a different group of
    // experts spreads the simultaneous reads over the L2 slices instead of
    // sending all CTAs to the same rows at once.  (Only when E is a multiple
    // of EPW, so that a rotated group never wraps.)
    const int rot = (p.E % EPW == 0) ? static_cast<int>((blockIdx.x * EPW) % p.E) : 0;
    for (int e0 = warp * EPW; e0 < p.E; e0 += (kSmallThreads / 32) * EPW) {
        const int eb = e0 + rot < p.E ? e0 + rot : e0 + rot - p.E;  // first expert of the group
        float acc[EPW][kSmallTok];
#pragma unroll
        for (int q = 0; q < EPW; ++q)
#pragma unroll
            for (int tt = 0; tt < kSmallTok; ++tt) acc[q][tt] = 0.0f;
        for (int v0 = lane; v0 < nv; v0 += 32 * U) {
            uint4 wv[U][EPW];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int v = v0 + 32 * u;
#pragma unroll
                for (int q = 0; q < EPW; ++q)
                    wv[u][q] = (v < nv && e0 + q < p.E)
                                   ? __ldg(p.Wg + static_cast<size_t>(eb + q) * nv + v)
                                   : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int v = v0 + 32 * u;
                if (v < nv) {
                    float wf[EPW][8];
#pragma unroll
                    for (int q = 0; q < EPW; ++q) unpack8(wv[u][q], wf[q]);
#pragma unroll
                    for (int tt = 0; tt < kSmallTok; ++tt) {
                        float xf[8];
                        unpack8(sx[tt * nv + v], xf);
#pragma unroll
                        for (int q = 0; q < EPW; ++q)
#pragma unroll
                            for (int i = 0; i < 8; ++i) acc[q][tt] = fmaf(wf[q][i], xf[i], acc[q][tt]);
                    }
                }
            }
        }
#pragma unroll
        for (int q = 0; q < EPW; ++q) {
#pragma unroll
            for (int tt = 0; tt < kSmallTok; ++tt) {
                float a = acc[q][tt];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
                acc[q][tt] = a;
            }
        }
        if (lane == 0) {
#pragma unroll
            for (int q = 0; q < EPW; ++q) {
                const int e = eb + q;
                if (e0 + q < p.E) {
                    const float b = p.bias ? p.bias[e] : 0.0f;
#pragma unroll
                    for (int tt = 0; tt < kSmallTok; ++tt) slog[tt * kMaxE + e] = acc[q][tt] + b;
                }
            }
        }
    }
    __syncthreads();

    if (warp < nt) {
        const int t = t0 + warp;
        // A NaN logit (only from non-finite inputs) ranks like -inf, and
        // every round takes the largest remaining value with the lower index
        // on ties, so each slot gets a distinct expert in [0, E) whatever
        // the values are (k <= E).
        float v[kMaxE / 32];
        uint32_t taken = 0u;  // bit i: expert lane + 32*i already selected
#pragma unroll
        for (int i = 0; i < kMaxE / 32; ++i) {
            const int e = lane + 32 * i;
            const float l = (e < p.E) ? slog[warp * kMaxE + e] : -CUDART_INF_F;
            v[i] = (l == l) ? l : -CUDART_INF_F;
        }
        float tv[K];
        int ti[K];
#pragma unroll
        for (int j = 0; j < K; ++j) {
            float bv = -CUDART_INF_F;
            int be = 0x7fffffff;
#pragma unroll
            for (int i = 0; i < kMaxE / 32; ++i) {
                const int e = lane + 32 * i;
                // e ascends with i: equal values keep the lower index
                if (e < p.E && !(taken & (1u << i)) && (v[i] > bv || be == 0x7fffffff)) {
                    bv = v[i];
                    be = e;
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
                const int oe = __shfl_xor_sync(0xffffffffu, be, off);
                if (ov > bv || (ov == bv && oe < be)) {
                    bv = ov;
                    be = oe;
                }
            }
            tv[j] = bv;
            ti[j] = be;
#pragma unroll
            for (int i = 0; i < kMaxE / 32; ++i)
                if (lane + 32 * i == be) taken |= 1u << i;
        }
        // Sum of exp(l - max) over all E logits (the softmax over all
        // experts); tv[0] is the maximum.
        float sum_all = 0.0f, sum_a = 0.0f;
        if (p.wmode == 1) {
#pragma unroll
            for (int i = 0; i < kMaxE / 32; ++i)
                if (lane + 32 * i < p.E && v[i] > -CUDART_INF_F) sum_all += expf(v[i] - tv[0]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                sum_all += __shfl_xor_sync(0xffffffffu, sum_all, off);
        } else if (p.wmode == 3) {
            // Tempered softmax sum Z and A = sum exp((l - m) / tau) (l - m).
#pragma unroll
            for (int i = 0; i < kMaxE / 32; ++i) {
                if (lane + 32 * i < p.E && v[i] > -CUDART_INF_F) {
                    const float q = expf((v[i] - tv[0]) * kEntropyInvTau);
                    sum_all += q;
                    sum_a += q * (v[i] - tv[0]);
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                sum_all += __shfl_xor_sync(0xffffffffu, sum_all, off);
                sum_a += __shfl_xor_sync(0xffffffffu, sum_a, off);
            }
        }
        if (lane == 0) {
            float wv[K];
            gate_weights<K>(tv, p.wmode, tv[0], sum_all, wv);
            // Slots in use: all K, or K - 1 under the entropy rule.
            const int ku = p.wmode == 3 ? entropy_slots<K>(sum_all, sum_a) : K;
#pragma unroll
            for (int j = 0; j < K; ++j) {
                p.idx[static_cast<size_t>(t) * K + j] = j < ku ? ti[j] : -1;
                p.w[static_cast<size_t>(t) * K + j] = j < ku ? wv[j] : 0.0f;
                ds.sel[warp][j] = j < ku ? ti[j] : -1;
            }
        }
    }
    if (p.slots) {
        __syncthreads();
        assign_slots(ds, t0, nt, p.T, p.E, K, p.sout, threadIdx.x, kSmallThreads, 1);
        return;
    }

    // The last CTA of each 128-token tile groups that tile's pairs by expert.
    __threadfence();
    __syncthreads();
    const int tile = t0 / kTileTokens;
    if (threadIdx.x == 0) {
        const int tile_tokens = min(kTileTokens, p.T - tile * kTileTokens);
        const uint32_t nblk = static_cast<uint32_t>((tile_tokens + kSmallTok - 1) / kSmallTok);
        s_last = (atomicAdd(&p.tile_ctr[tile], 1u) == nblk - 1u) ? 1u : 0u;
    }
    __syncthreads();
    if (!s_last || threadIdx.x >= kTileTokens) return;
    __threadfence();
    const int row = threadIdx.x;
    const int t = tile * kTileTokens + row;
#pragma unroll
    for (int j = 0; j < K; ++j)
        ds.sel[row][j] = (t < p.T) ? __ldcg(&p.idx[static_cast<size_t>(t) * K + j]) : -1;
#pragma unroll
    for (int j = 0; j < K; ++j)  // the selection above always yields [0, E); keep dispatch in bounds regardless
        if (static_cast<unsigned>(ds.sel[row][j]) >= static_cast<unsigned>(p.E)) ds.sel[row][j] = -1;
    dispatch_tile(ds, row, tile, p.T, p.E, K, p.dout, 1);
}

template <int K, int EPW, int U>
cudaError_t launch_route_small_cfg(const RouteLaunch &a, cudaStream_t s)
{
    const size_t smem = small_route_smem(a.d);
    cudaError_t e = cudaFuncSetAttribute(route_small_kernel<K, EPW, U>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    SmallRouteParams p{};
    p.T = a.T;
    p.d = a.d;
    p.E = a.E;
    p.wmode = a.wmode;
    p.x = reinterpret_cast<const uint4 *>(a.x);
    p.Wg = reinterpret_cast<const uint4 *>(a.Wg);
    p.bias = a.bias;
    p.idx = a.idx;
    p.w = a.w;
    p.tile_ctr = a.tile_ctr;
    p.dout.tilecnt = a.tilecnt;
    p.dout.tilebase = a.tilebase;
    p.dout.rank = a.rank;
    p.dout.offsets = a.offsets;
    p.dout.counts = a.counts;
    p.dout.done = a.done;
    p.dout.cap = a.cap;
    p.dout.ntiles = (a.T + kTileTokens - 1) / kTileTokens;
    const int blocks = (a.T + kSmallTok - 1) / kSmallTok;
    fill_slots(a, &p.slots, &p.sout);
    route_small_kernel<K, EPW, U><<<blocks, kSmallThreads, smem, s>>>(p);
    return cudaGetLastError();
}

// Few experts: one expert per warp and eight loads in flight per lane; many
// experts: four (eight for narrow rows) experts per warp.
template <int K>
cudaError_t launch_route_small_k(const RouteLaunch &a, cudaStream_t s)
{
    if (a.E <= 16) return launch_route_small_cfg<K, 1, 8>(a, s);
    // Narrow rows (d <= 512: 64 vectors, two loads per lane cover a row):
    // eight experts per warp, so a pass covers 64 experts with all of its
    // loads in flight at once.
    if (a.d <= 512) return launch_route_small_cfg<K, 8, 2>(a, s);
    return launch_route_small_cfg<K, 4, 4>(a, s);
}

template <int K>
cudaError_t launch_route_k(const RouteLaunch &a, cudaStream_t s)
{
    const int Npad = ((a.E + 15) / 16) * 16 < 16 ? 16 : ((a.E + 15) / 16) * 16;
    const uint32_t sb = route_stage_bytes(Npad);
    int stages = static_cast<int>((227 * 1024 - kRouteFixedSmem) / sb);
    if (stages > kRouteMaxStages) stages = kRouteMaxStages;
    const size_t smem = kRouteFixedSmem + static_cast<size_t>(stages) * sb;
    uint32_t cols = 32;
    while (cols < static_cast<uint32_t>(Npad)) cols <<= 1;

    CUtensorMap tmX, tmWg;
    cudaError_t e = make_tmap_bf16(&tmX, a.x, a.T, a.d, 128);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16(&tmWg, a.Wg, a.E, a.d, static_cast<uint32_t>(Npad));
    if (e != cudaSuccess) return e;

    e = cudaFuncSetAttribute(route_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;

    RouteParams p{};
    p.T = a.T;
    p.d = a.d;
    p.E = a.E;
    p.Npad = Npad;
    p.wmode = a.wmode;
    p.stages = stages;
    p.ntiles = (a.T + kTileTokens - 1) / kTileTokens;
    p.tmem_cols = cols;
    p.bias = a.bias;
    p.idx = a.idx;
    p.w = a.w;
    p.err = a.err;
    p.dout.tilecnt = a.tilecnt;
    p.dout.tilebase = a.tilebase;
    p.dout.rank = a.rank;
    p.dout.offsets = a.offsets;
    p.dout.counts = a.counts;
    p.dout.done = a.done;
    p.dout.cap = a.cap;
    p.dout.ntiles = p.ntiles;
    fill_slots(a, &p.slots, &p.sout);
    route_kernel<K><<<p.ntiles, kRouteThreads, smem, s>>>(tmX, tmWg, p);
    return cudaGetLastError();
}

}  // namespace

// Tensor cores pay off once the router is a real GEMM; below this many
// multiply-adds the CUDA-core router is faster (it spreads over more SMs and
// has a short dependency chain).  Long batches of wide rows also go to the
// tensor cores whatever E is: the CUDA-core router reads all of Wg again for
// every 4 tokens, the tensor-core router once per 128 (measured at d = 4096,
// E = 8: 59 vs 39 us at T = 8192, 29 vs 35 us at T = 2048).
constexpr long long kSmallRouterMacs = 1LL << 30;

bool use_small_router(const RouteLaunch &a)
{
    if (a.T >= 4096 && a.d >= 2048) return false;
    return static_cast<long long>(a.T) * a.E * a.d <= kSmallRouterMacs;
}

cudaError_t launch_route(const RouteLaunch &a, cudaStream_t s)
{
    if (use_small_router(a)) {
        switch (a.k) {
        case 1: return launch_route_small_k<1>(a, s);
        case 2: return launch_route_small_k<2>(a, s);
        case 3: return launch_route_small_k<3>(a, s);
        case 4: return launch_route_small_k<4>(a, s);
        case 5: return launch_route_small_k<5>(a, s);
        case 6: return launch_route_small_k<6>(a, s);
        case 7: return launch_route_small_k<7>(a, s);
        case 8: return launch_route_small_k<8>(a, s);
        default: return cudaErrorInvalidValue;
        }
    }
    switch (a.k) {
    case 1: return launch_route_k<1>(a, s);
    case 2: return launch_route_k<2>(a, s);
    case 3: return launch_route_k<3>(a, s);
    case 4: return launch_route_k<4>(a, s);
    case 5: return launch_route_k<5>(a, s);
    case 6: return launch_route_k<6>(a, s);
    case 7: return launch_route_k<7>(a, s);
    case 8: return launch_route_k<8>(a, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
