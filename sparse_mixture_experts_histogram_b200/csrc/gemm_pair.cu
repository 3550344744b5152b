// gemm_pair.cu -- the experts' feed-forward for large batches: one persistent
// kernel in which each pair of CTAs (a cluster of two) runs 256-row tensor-core
// MMAs together (tcgen05 .cta_group::2).
//
// For every expert segment e (rows offsets[e] .. offsets[e+1]-1 of x_perm),
// cut into token tiles of at most 256 rows of near-equal size:
//   up units   (e, 128-column block of H, tile):
//       even CTA A = [W1_e rows f0..f0+63 ; W3_e rows f0..f0+63]
//       odd CTA  A = [W1_e rows f0+64..f0+127 ; W3_e rows f0+64..f0+127]
//       D (256 x N) = A X^T: each CTA holds its 128 rows -- lanes 0..63 the
//       W1 products, lanes 64..127 the W3 products of the same 64 columns of H
//       H[r, f] = bf16( silu(D_W1) * D_W3 )      -- SwiGLU epilogue
//   down units (e, 256 output columns, tile):
//       even CTA A = W2_e rows o0..o0+127, odd CTA A = rows o0+128..o0+255
//       Y[r, o] = (A H^T)[o, r]                  -- fp32
//       or, for top-k with k <= 2, the gate-weighted combine in place:
//       out[t, o] += w[t, j] * (A H^T)[o, r] for the slot (t, j) of row r
//       ("MoE" (theaiera.top) sec. 10.4, the weighted index_add back to the
//       tokens), onto an out the scatter zeroed; at most two terms reach an
//       element, and two terms added onto zero give one sum in either order
// The weights are the MMA's A operand (M = 256 over the pair), the tile's
// rows its B operand (N = rows rounded up to 16; each CTA holds N/2 of them),
// so a ragged segment costs only the MMA columns it needs.  Per CTA and
// 128-wide K step one stage holds 128 weight rows and 128 token rows (of which
// the MMA reads N/2), each as two 64-column atoms; per 256 x N x 16
// MMA each SM reads half of A and half of B from its shared memory, half what
// two 128-row MMAs sharing one B tile would read.
//
// Scheduling: the units are numbered up first, then down; the even CTA's
// producer takes the next number from a global counter and hands it to every
// role of both CTAs through a small ring of slots in shared memory.  A down
// unit waits (bounded) for the up units of its tile and H blocks, which have
// smaller numbers and so were taken earlier by running CTAs: the waits end
// whatever number of CTAs is resident at a time.
//
// Roles per CTA: warp 0 issues TMA copies into a ring of stages (each CTA its
// own halves, completion counted on the even CTA's barrier), warp 1 of the
// even CTA issues the MMAs into one of two tensor-memory accumulators and
// signals both CTAs, warps 2..9 drain the accumulator: up units exchange the
// W1 and W3 products between lane quarters through shared memory and store
// H; down units write their fp32 outputs (or add them, weighted, into out).
//
// Method: the SwiGLU expert w2(silu(w1 x) * w3 x) ("Mistral 8x7B SMoE
// architecture" (jsqmd.com) sec. 3.1 FeedForward; "Mixtral and MoE
// architecture" FeedForward listing) applied to each expert's own tokens
// ("MoE" (theaiera.top) sec. 10.4); W1 and W3 are consumed together so the
// activation runs in the epilogue, the fusion the "万亿 MoE" page (m.xxqk.cn)
// sketches by concatenating the two up-projections.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace moe {

namespace {

constexpr int kPThreads = 320;           // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue
constexpr int kPEpiWarps = 8;
constexpr int kPStages = 3;
constexpr int kPMaxN = 256;              // token rows per tile (MMA N)
constexpr uint32_t kPATile = 128 * 128;  // 128 weight rows x 64 bf16 (16 KB)
constexpr uint32_t kPBTile = 128 * 128;  // 128 token rows x 64 bf16 (16 KB): a CTA copies
                                         // 128 rows for N/2 > kPBShort (fewer, larger copies
                                         // measured faster than copies of just the rows used)
// Token tiles of at most 2 * kPBShort rows (the two-tile segments of the
// 256-expert layer, about 136 rows each) copy kPBShort rows per CTA instead:
// the weight stream then needs fewer bytes in flight to stay ahead of the
// MMAs, whose work per K step shrinks with N.
constexpr int kPBShort = 80;
constexpr uint32_t kPBShortTile = kPBShort * 128;  // 10 KB, a multiple of the 1 KB swizzle atom
constexpr int kPAtoms = 2;               // 64-column atoms per K step (128 columns)
constexpr uint32_t kPStage = kPAtoms * (kPATile + kPBTile);  // [A atoms][B atoms], 64 KB
constexpr int kPSlots = 4;               // unit-number ring
constexpr uint32_t kPTmemCols = 512;     // two accumulators of 256 columns
constexpr uint32_t kPAccCols = 256;
constexpr int kPChunk = 16;              // accumulator columns per exchange step
constexpr uint32_t kPXchgBytes = 4 * 2 * 2 * 8 * 32 * 4;       // [pair][buf][a|b][8][32] f32
constexpr int kPBarriers = 2 * kPStages + 2 + 2 + 2 * kPSlots + 1 + 8;
constexpr size_t kPSmem = 1024 /* alignment slack */ + kPStages * kPStage + kPXchgBytes +
                          kPBarriers * 8 + 64 + 4 * (kMaxE + 1) * sizeof(int32_t);
// Epilogue warps of both CTAs that publish each (token tile, H block).
constexpr uint32_t kPReadyTarget = 2 * kPEpiWarps;
static_assert(kPSmem <= 227 * 1024, "shared memory");
// Consumers of a unit number: the even CTA's MMA thread and 8 epilogue warps,
// the odd CTA's producer and 8 epilogue warps.
constexpr uint32_t kPSchedConsumers = 1 + kPEpiWarps + 1 + kPEpiWarps;

struct PairParams {
    int E, d, d_ff, S;
    const int32_t *offsets;  // [E+1] or nullptr (one segment [0, S))
    __nv_bfloat16 *H;        // [S, d_ff]
    float *Y;                // [S, d]
    uint32_t *h_ready;       // [tiles, d_ff/128], zero before the launch
    uint32_t *sched;         // unit counter, zero before the launch
    uint32_t *err;
    int act;                 // expert activation: 0 silu(g) * b, 1 sigmoid(g) * b
    // Weighted output (k <= 2): when out is set, the down units add
    // gate_w[s] * y into out[s / k] (s = slot_of_row[row]) instead of
    // writing Y.  Two terms added onto zero give the same sum in either
    // order, so the result does not depend on which unit finishes first.
    float *out;
    const int32_t *slot_of_row;
    const float *gate_w;
    int k;
    int y_bf16;              // Y as bf16 rows (otherwise fp32)
};

struct PUnit {
    bool up;
    int e, blk, r0, valid, n, tile;
};

__device__ __forceinline__ int ceil16(int v) { return (v + 15) & ~15; }

// Tiles of a segment of cnt rows: ceil(cnt/256) tiles of q rows (the last one
// shorter), q = ceil(cnt/tiles) rounded up to 16.
__device__ __forceinline__ int seg_tiles(int cnt) { return (cnt + kPMaxN - 1) / kPMaxN; }

__device__ __forceinline__ PUnit decode_punit(int u, int u_up, const int32_t *s_off,
                                              const int32_t *s_pu, const int32_t *s_pd,
                                              const int32_t *s_tb, int E)
{
    PUnit w;
    w.up = u < u_up;
    const int32_t *pre = w.up ? s_pu : s_pd;
    const int x = w.up ? u : u - u_up;
    int lo = 0, hi = E - 1;
    while (lo < hi) {  // largest e with pre[e] <= x
        const int mid = (lo + hi + 1) >> 1;
        if (pre[mid] <= x) lo = mid;
        else hi = mid - 1;
    }
    w.e = lo;
    const int local = x - pre[lo];
    const int cnt = s_off[lo + 1] - s_off[lo];
    const int nt = seg_tiles(cnt);
    const int q = ceil16((cnt + nt - 1) / nt);
    w.blk = local / nt;
    const int t = local - w.blk * nt;
    w.r0 = s_off[lo] + t * q;
    const int rem = cnt - t * q;
    w.valid = rem < q ? rem : q;
    w.n = ceil16(w.valid);
    w.tile = s_tb[lo] + t;
    return w;
}

__device__ __forceinline__ bool wait_cl(uint64_t *bar, uint32_t parity,
                                        volatile uint32_t *abort_flag, uint32_t *gerr,
                                        uint32_t code)
{
    if (ptx::mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (ptx::mbar_try_wait_cluster(bar, parity)) return true;
        if (*abort_flag) return false;
        if ((it & 63u) == 0 && ptx::globaltimer() - t0 > kWaitTimeoutNs) {
            *abort_flag = 1u;
            if (gerr) atomicOr(gerr, code);
            return false;
        }
    }
}

__device__ __forceinline__ void drain_wait_cl(uint64_t *bar, uint32_t parity)
{
    const uint64_t t0 = ptx::globaltimer();
    while (!ptx::mbar_try_wait_cluster(bar, parity)) {
        if (ptx::globaltimer() - t0 > 100000000ull) break;  // 100 ms
    }
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void fence_proxy_async_global()
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Waits until *ctr >= target (written by other CTAs' epilogues), bounded.
__device__ __forceinline__ bool wait_ready(const uint32_t *ctr, uint32_t target,
                                           volatile uint32_t *abort_flag, uint32_t *gerr)
{
    if (ld_acquire_gpu(ctr) >= target) return true;
    const uint64_t t0 = ptx::globaltimer();
    for (uint32_t it = 1;; ++it) {
        __nanosleep(64);
        if (ld_acquire_gpu(ctr) >= target) return true;
        if (*abort_flag) return false;
        if ((it & 15u) == 0 && ptx::globaltimer() - t0 > kWaitTimeoutNs) {
            *abort_flag = 1u;
            if (gerr) atomicOr(gerr, kErrTimeoutEpi);
            return false;
        }
    }
}

__device__ __forceinline__ int warp_scan_incl(int v, int lane)
{
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += n;
    }
    return v;
}

// silu(g) * b (act 0) or sigmoid(g) * b (act 1).
__device__ __forceinline__ float gate_mul(float g, float b, int act)
{
    return __fdividef(act ? b : g * b, 1.0f + __expf(-g));
}

__global__ void __launch_bounds__(kPThreads, 1)
    ffn_pair_kernel(const __grid_constant__ CUtensorMap tmW1,   // 64-row boxes
                    const __grid_constant__ CUtensorMap tmW3,   // 64-row boxes
                    const __grid_constant__ CUtensorMap tmW2,   // 128 rows x 2 atoms
                    const __grid_constant__ CUtensorMap tmX,    // 128 rows x 2 atoms
                    const __grid_constant__ CUtensorMap tmH,    // 128 rows x 2 atoms
                    const __grid_constant__ CUtensorMap tmXs,   // kPBShort rows x 2 atoms
                    const __grid_constant__ CUtensorMap tmHs,   // kPBShort rows x 2 atoms
                    const PairParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t cta = ptx::cluster_ctarank();  // 0: issues the MMAs
    const bool leader = (cta == 0);

    float *xchg = reinterpret_cast<float *>(smem + kPStages * kPStage);
    uint64_t *full = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(xchg) + kPXchgBytes);
    uint64_t *empty = full + kPStages;
    uint64_t *tfull = empty + kPStages;   // [2]
    uint64_t *tempty = tfull + 2;         // [2]
    uint64_t *sfull = tempty + 2;         // [kPSlots]
    uint64_t *sempty = sfull + kPSlots;   // [kPSlots]
    uint64_t *drain = sempty + kPSlots;   // [1]
    uint64_t *xbar = drain + 1;           // [4 warp pairs][2 exchange buffers]
    uint32_t *sched_id = reinterpret_cast<uint32_t *>(xbar + 8);  // [kPSlots]
    uint32_t *tmem_slot = sched_id + kPSlots;
    volatile uint32_t *abort_flag = tmem_slot + 1;
    int32_t *s_off = reinterpret_cast<int32_t *>(tmem_slot + 12);
    int32_t *s_pu = s_off + (kMaxE + 1);
    int32_t *s_pd = s_pu + (kMaxE + 1);
    int32_t *s_tb = s_pd + (kMaxE + 1);

    const int E = p.offsets ? p.E : 1;
    const int MBU = p.d_ff / 128;        // up blocks per expert (128 columns of H)
    const int MBD = (p.d + 255) / 256;   // down blocks per expert (256 output columns)
    const int KSU = p.d / 128;       // 128-column K steps
    const int KSD = p.d_ff / 128;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPStages; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&tfull[b], 1);
            ptx::mbar_init(&tempty[b], 2 * kPEpiWarps);
        }
        for (int s = 0; s < kPSlots; ++s) {
            ptx::mbar_init(&sfull[s], 1);
            ptx::mbar_init(&sempty[s], kPSchedConsumers);
        }
        ptx::mbar_init(drain, 1);
        for (int b = 0; b < 8; ++b) ptx::mbar_init(&xbar[b], 64);
        *abort_flag = 0u;
        ptx::fence_barrier_init();
    }
    if (threadIdx.x == 32) {
        ptx::prefetch_tensormap(&tmW1);
        ptx::prefetch_tensormap(&tmW3);
        ptx::prefetch_tensormap(&tmW2);
        ptx::prefetch_tensormap(&tmX);
        ptx::prefetch_tensormap(&tmH);
        ptx::prefetch_tensormap(&tmXs);
        ptx::prefetch_tensormap(&tmHs);
    }
    if (warp == 1) {
        ptx::tmem_alloc_pair(tmem_slot, kPTmemCols);
        ptx::tmem_relinquish_pair();
    }
    // Everything above overlaps the previous kernel; from here on its results
    // (offsets, x_perm) are read.
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
                    const int tl = seg_tiles(c);
                    nt += tl;
                    nu += tl * MBU;
                    nd += tl * MBD;
                }
            }
        }
        __syncwarp();  // s_off[e + 1] below may come from the next lane
        bad = __any_sync(0xffffffffu, bad);
        if (bad) {
            nu = nd = nt = 0;
            if (lane == 0 && leader) atomicOr(p.err, kErrOffsets);
        }
        const int iu = warp_scan_incl(nu, lane);
        const int id = warp_scan_incl(nd, lane);
        const int it = warp_scan_incl(nt, lane);
        int ru = iu - nu, rd = id - nd, rt = it - nt;
        for (int i = 0; i < per; ++i) {
            const int e = base + i;
            if (e < E) {
                s_pu[e] = ru;
                s_pd[e] = rd;
                s_tb[e] = rt;
                if (!bad) {
                    const int tl = seg_tiles(s_off[e + 1] - s_off[e]);
                    ru += tl * MBU;
                    rd += tl * MBD;
                    rt += tl;
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
    // Both CTAs' barriers are initialised before either CTA signals the other.
    ptx::cluster_sync();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int u_up = s_pu[E];
    const int total = u_up + s_pd[E];

    // Shared::cluster addresses of the even CTA's barriers and of the odd
    // CTA's ring (the even CTA's producer writes it).
    const uint32_t full0 = ptx::mapa_shared(ptx::smem_addr(full), 0);
    const uint32_t tempty0 = ptx::mapa_shared(ptx::smem_addr(tempty), 0);
    const uint32_t sempty0 = ptx::mapa_shared(ptx::smem_addr(sempty), 0);
    const uint32_t sfull1 = ptx::mapa_shared(ptx::smem_addr(sfull), 1);
    const uint32_t sid1 = ptx::mapa_shared(ptx::smem_addr(sched_id), 1);

    if (warp == 0) {
        if (lane == 0) {
            uint32_t stage = 0, phase = 0, issued = 0;
            uint32_t last_parity[kPStages];
#pragma unroll
            for (int s = 0; s < kPStages; ++s) last_parity[s] = 0;
            const uint64_t pol = ptx::policy_evict_normal();
            bool stop = false;
            // The even CTA takes the number of its next unit while it still
            // issues the copies of the current one, so the atomic's latency
            // never stalls the pipeline at a unit boundary.
            uint32_t next = leader ? atomicAdd(p.sched, 1u) : 0u;
            for (uint32_t i = 0; !stop; ++i) {
                const uint32_t slot = i % kPSlots;
                const uint32_t sph = (i / kPSlots) & 1u;
                uint32_t u;
                if (leader) {
                    if (!wait_cl(&sempty[slot], sph ^ 1u, abort_flag, p.err, kErrTimeoutEpi)) break;
                    u = next < static_cast<uint32_t>(total) ? next : static_cast<uint32_t>(total);
                    sched_id[slot] = u;
                    ptx::st_shared_cluster_u32(sid1 + 4 * slot, u);
                    ptx::mbar_arrive(&sfull[slot]);
                    ptx::mbar_arrive_cluster(sfull1 + 8 * slot);
                    if (u < static_cast<uint32_t>(total)) next = atomicAdd(p.sched, 1u);
                } else {
                    if (!wait_cl(&sfull[slot], sph, abort_flag, p.err, kErrTimeoutEpi)) break;
                    u = *reinterpret_cast<volatile uint32_t *>(&sched_id[slot]);
                    ptx::mbar_arrive_cluster(sempty0 + 8 * slot);
                }
                if (u >= static_cast<uint32_t>(total)) break;
                const PUnit w = decode_punit(static_cast<int>(u), u_up, s_off, s_pu, s_pd, s_tb, E);
                const int ksteps = w.up ? KSU : KSD;
                const int half = w.n >> 1;               // B rows this CTA holds
                const bool shrt = half <= kPBShort;
                const uint32_t tx =
                    2u * kPAtoms * (kPATile + (shrt ? kPBShortTile : kPBTile));
                const int arow = w.up ? w.e * p.d_ff + w.blk * 128 + static_cast<int>(cta) * 64
                                      : w.e * p.d + w.blk * 256 + static_cast<int>(cta) * 128;
                const CUtensorMap *tb = w.up ? (shrt ? &tmXs : &tmX) : (shrt ? &tmHs : &tmH);
                const int brow = w.r0 + static_cast<int>(cta) * half;
                for (int ks = 0; ks < ksteps; ++ks) {
                    if (!wait_cl(&empty[stage], phase ^ 1u, abort_flag, p.err, kErrTimeoutMma)) {
                        stop = true;
                        break;
                    }
                    uint8_t *sa = smem + stage * kPStage;
                    const uint32_t fb = full0 + 8 * stage;
                    if (leader) ptx::mbar_arrive_expect_tx(&full[stage], tx);
                    if (w.up) {
                        // A atom a = [64 W1 rows; the same 64 W3 rows]
#pragma unroll
                        for (int a = 0; a < kPAtoms; ++a) {
                            const int c = ks * 128 + a * 64;
                            ptx::tma_load_2d_pair(sa + a * kPATile, &tmW1, fb, c, arow, pol);
                            ptx::tma_load_2d_pair(sa + a * kPATile + kPATile / 2, &tmW3, fb, c,
                                                  arow, pol);
                        }
                    } else {
                        ptx::tma_load_3d_pair(sa, &tmW2, fb, 0, arow, ks * kPAtoms, pol);
                    }
                    issued |= 1u << stage;
                    last_parity[stage] = phase;
                    if (!w.up) {
                        // These 128 columns of H are block ks: wait until
                        // every epilogue warp of both CTAs of its up unit
                        // stored its part.
                        if (!wait_ready(&p.h_ready[w.tile * MBU + ks], kPReadyTarget, abort_flag,
                                        p.err)) {
                            stop = true;
                            break;
                        }
                        fence_proxy_async_global();
                    }
                    ptx::tma_load_3d_pair(sa + kPAtoms * kPATile, tb, fb, 0, brow, ks * kPAtoms,
                                          pol);
                    if (++stage == static_cast<uint32_t>(kPStages)) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // No copy may still be landing in shared memory at exit.  Only
            // the even CTA can see its full barriers complete; the odd CTA's
            // copies count there too, and the final cluster barrier orders
            // its exit after the even CTA's drain.
            if (leader)
                for (int s = 0; s < kPStages; ++s)
                    if (issued & (1u << s)) drain_wait_cl(&full[s], last_parity[s]);
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            uint32_t stage = 0, phase = 0;
            bool stop = false;
            for (uint32_t i = 0; !stop; ++i) {
                const uint32_t slot = i % kPSlots;
                const uint32_t sph = (i / kPSlots) & 1u;
                if (!wait_cl(&sfull[slot], sph, abort_flag, p.err, kErrTimeoutEpi)) break;
                const uint32_t u = *reinterpret_cast<volatile uint32_t *>(&sched_id[slot]);
                ptx::mbar_arrive(&sempty[slot]);
                if (u >= static_cast<uint32_t>(total)) break;
                const PUnit w = decode_punit(static_cast<int>(u), u_up, s_off, s_pu, s_pd, s_tb, E);
                const uint32_t idesc = ptx::idesc_bf16_f32(256, w.n);
                // B atoms as the producer copied them: kPBShort or 128 rows.
                const uint32_t bstride = (w.n >> 1) <= kPBShort ? kPBShortTile : kPBTile;
                const int buf = static_cast<int>(i & 1u);
                const uint32_t use = i >> 1;
                if (!wait_cl(&tempty[buf], (use & 1u) ^ 1u, abort_flag, p.err, kErrTimeoutEpi))
                    break;
                ptx::tc_fence_after();
                const uint32_t dacc = tmem + static_cast<uint32_t>(buf) * kPAccCols;
                const int ksteps = w.up ? KSU : KSD;
                for (int ks = 0; ks < ksteps; ++ks) {
                    if (!wait_cl(&full[stage], phase, abort_flag, p.err, kErrTimeoutTma)) {
                        stop = true;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t sa = ptx::smem_addr(smem + stage * kPStage);
                    const uint32_t sb = sa + kPAtoms * kPATile;
#pragma unroll
                    for (int a = 0; a < kPAtoms; ++a)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            ptx::tc_mma_bf16_pair(
                                dacc, ptx::sw128_kmajor_desc(sa + a * kPATile + kk * 32),
                                ptx::sw128_kmajor_desc(sb + a * bstride + kk * 32), idesc,
                                (ks | a | kk) ? 1u : 0u);
                    ptx::tc_commit_pair(&empty[stage], 0x3);
                    if (++stage == static_cast<uint32_t>(kPStages)) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!stop) ptx::tc_commit_pair(&tfull[buf], 0x3);
            }
            // Every MMA issued above has finished once this arrives.
            ptx::tc_commit_pair(drain, 0x1);
            drain_wait_cl(drain, 0u);
        }
    } else {
        // Epilogue: warps 2..9.  Warp w reads TMEM lanes 32*(w%4)..+31;
        // the two warps of a lane quarter take alternate column chunks.  The
        // warps meet only at mbarriers with bounded waits, so a warp that
        // gives up never leaves another one blocked.
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
        const int pair = (q & 1) + 2 * half;  // (a, b) warp pairs: quarters (0,2) and (1,3)
        const bool is_a = q < 2;              // lanes 0..63: W1 products (up units)
        const int fl = (q & 1) * 32 + lane;   // column of H within this CTA's 64
        float *xa = xchg + pair * (2 * 2 * 8 * 32);
        uint32_t xuse[2] = {0u, 0u};          // completed phases of this pair's two buffers
        bool stop = false;
        for (uint32_t i = 0; !stop; ++i) {
            const uint32_t slot = i % kPSlots;
            const uint32_t sph = (i / kPSlots) & 1u;
            uint32_t u = 0xffffffffu;  // stays so if the wait gave up
            if (lane == 0) {
                if (wait_cl(&sfull[slot], sph, abort_flag, p.err, kErrTimeoutEpi)) {
                    u = *reinterpret_cast<volatile uint32_t *>(&sched_id[slot]);
                    if (leader) ptx::mbar_arrive(&sempty[slot]);
                    else ptx::mbar_arrive_cluster(sempty0 + 8 * slot);
                }
            }
            u = __shfl_sync(0xffffffffu, u, 0);
            if (u >= static_cast<uint32_t>(total)) break;
            const PUnit w = decode_punit(static_cast<int>(u), u_up, s_off, s_pu, s_pd, s_tb, E);
            const int buf = static_cast<int>(i & 1u);
            const uint32_t use = i >> 1;
            const bool okt = wait_cl(&tfull[buf], use & 1u, abort_flag, p.err, kErrTimeoutMma);
            if (!__all_sync(0xffffffffu, okt)) {
                *abort_flag = 1u;
                break;
            }
            ptx::tc_fence_after();
            const uint32_t tb = tmem + lane_base + static_cast<uint32_t>(buf) * kPAccCols;
            if (w.up) {
                const int hcol = w.blk * 128 + static_cast<int>(cta) * 64 + fl;
                const int nchunks = w.n / kPChunk;
                int xb = 0;
                for (int c = half; c < nchunks; c += 2, xb ^= 1) {
                    uint32_t r[16];
                    ptx::tmem_ld16(tb + static_cast<uint32_t>(c * kPChunk), r);
                    ptx::tc_wait_ld();
                    // a warps keep tokens 0..7 of the chunk and hand 8..15 to
                    // their b partner; b warps the other way round.
                    float *mine = xa + xb * (2 * 8 * 32) + (is_a ? 0 : 8 * 32);
                    float *theirs = xa + xb * (2 * 8 * 32) + (is_a ? 8 * 32 : 0);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        mine[j * 32 + lane] = __uint_as_float(r[is_a ? 8 + j : j]);
                    ptx::mbar_arrive(&xbar[pair * 2 + xb]);
                    const bool okx = bounded_wait(&xbar[pair * 2 + xb], xuse[xb] & 1u, abort_flag,
                                                  p.err, kErrTimeoutEpi);
                    ++xuse[xb];
                    if (!__all_sync(0xffffffffu, okx)) {
                        stop = true;
                        break;
                    }
                    // H[r0 + t, f0 + fl]: the warp's lanes store 32
                    // adjacent columns of one row at a time.
                    const int t0 = c * kPChunk + (is_a ? 0 : 8);
                    __nv_bfloat16 *hrow = p.H + static_cast<size_t>(w.r0 + t0) * p.d_ff + hcol;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float o = theirs[j * 32 + lane];
                        const float g = is_a ? __uint_as_float(r[j]) : o;
                        const float b = is_a ? o : __uint_as_float(r[8 + j]);
                        if (t0 + j < w.valid)
                            hrow[static_cast<size_t>(j) * p.d_ff] =
                                __float2bfloat16_rn(gate_mul(g, b, p.act));
                    }
                }
                if (stop) break;
            } else {
                const int o = w.blk * 256 + static_cast<int>(cta) * 128 + 32 * q + lane;
                const bool has = o < p.d;
                for (int c0 = half * 32; c0 < w.n; c0 += 64) {
                    uint32_t r[32];
                    ptx::tmem_ld32(tb + static_cast<uint32_t>(c0), r);
                    ptx::tc_wait_ld();
                    if (p.out != nullptr) {
                        // Lane j fetches the slot and gate weight of row
                        // r0 + c0 + j; row j's values go to all lanes.
                        int sl = -1;
                        float gw = 0.0f;
                        if (c0 + lane < w.valid) {
                            const int v = p.slot_of_row[w.r0 + c0 + lane];
                            if (static_cast<unsigned>(v) < static_cast<unsigned>(p.S)) {
                                sl = v;
                                gw = p.gate_w[v];
                            }
                        }
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int slj = __shfl_sync(0xffffffffu, sl, j);
                            const float gwj = __shfl_sync(0xffffffffu, gw, j);
                            if (has && slj >= 0)
                                atomicAdd(p.out + static_cast<size_t>(slj / p.k) * p.d + o,
                                          gwj * __uint_as_float(r[j]));
                        }
                    } else if (has && p.y_bf16) {
                        __nv_bfloat16 *yc = reinterpret_cast<__nv_bfloat16 *>(p.Y) +
                                            static_cast<size_t>(w.r0 + c0) * p.d + o;
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (c0 + j < w.valid)
                                yc[static_cast<size_t>(j) * p.d] = __float2bfloat16_rn(__uint_as_float(r[j]));
                    } else if (has) {
                        float *yc = p.Y + static_cast<size_t>(w.r0 + c0) * p.d + o;
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (c0 + j < w.valid) yc[static_cast<size_t>(j) * p.d] = __uint_as_float(r[j]);
                    }
                }
            }
            // The accumulator may be reused once every epilogue warp of both
            // CTAs has read it.
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (leader) ptx::mbar_arrive(&tempty[buf]);
                else ptx::mbar_arrive_cluster(tempty0 + 8 * buf);
            }
            if (w.up) {
                // Publish this warp's part of the H block to the down units
                // (which read it through TMA, the async proxy).
                fence_proxy_async_global();
                __threadfence();
                __syncwarp();
                if (lane == 0) atomicAdd(&p.h_ready[w.tile * MBU + w.blk], 1u);
            }
        }
    }

    // Dependents (the shared expert, the combine) need this kernel's results:
    // let them launch only once its work is done.
    ptx::grid_dep_launch();
    ptx::tc_fence_before();
    __syncthreads();
    // Neither CTA may free tensor memory or exit while the other still
    // signals its barriers or reads the accumulators.
    ptx::cluster_sync();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(tmem, kPTmemCols);
    }
    ptx::cluster_sync();
}

std::atomic<int> g_pair_grid[64];

int pair_grid(cudaLaunchConfig_t &cfg)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    int g = g_pair_grid[dev].load(std::memory_order_relaxed);
    if (g > 0) return g;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, ffn_pair_kernel, &cfg) != cudaSuccess ||
        clusters < 1)
        clusters = device_sm_count() / 2;
    g = 2 * clusters;
    g_pair_grid[dev].store(g, std::memory_order_relaxed);
    return g;
}

}  // namespace

bool ffn_pair_eligible(int S, int E_seg, int ksplit)
{
    return ksplit <= 1 && ffn_token_tile(S, E_seg) >= 128;
}

cudaError_t launch_ffn_pair(const FfnLaunch &a, uint32_t *sched, cudaStream_t s)
{
    const int E = a.offsets ? a.E : 1;
    CUtensorMap tW1, tW3, tW2, tX, tH, tXs, tHs;
    cudaError_t e = make_tmap_bf16(&tW1, a.W1, static_cast<uint64_t>(E) * a.d_ff, a.d, 64);
    if (e == cudaSuccess) e = make_tmap_bf16(&tW3, a.W3, static_cast<uint64_t>(E) * a.d_ff, a.d, 64);
    if (e == cudaSuccess)
        e = make_tmap_bf16_atoms(&tW2, a.W2, static_cast<uint64_t>(E) * a.d, a.d_ff, 128, 2);
    if (e == cudaSuccess) e = make_tmap_bf16_atoms(&tX, a.x, a.S, a.d, 128, 2);
    if (e == cudaSuccess) e = make_tmap_bf16_atoms(&tH, a.H, a.S, a.d_ff, 128, 2);
    if (e == cudaSuccess) e = make_tmap_bf16_atoms(&tXs, a.x, a.S, a.d, kPBShort, 2);
    if (e == cudaSuccess) e = make_tmap_bf16_atoms(&tHs, a.H, a.S, a.d_ff, kPBShort, 2);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(ffn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kPSmem));
    if (e != cudaSuccess) return e;

    PairParams p{};
    p.E = E;
    p.d = a.d;
    p.d_ff = a.d_ff;
    p.S = a.S;
    p.offsets = a.offsets;
    p.H = reinterpret_cast<__nv_bfloat16 *>(a.H);
    p.Y = a.Y;
    p.h_ready = a.h_ready;
    p.sched = sched;
    p.err = a.err;
    p.act = a.act;
    p.out = a.out;
    p.slot_of_row = a.slot_of_row;
    p.gate_w = a.gate_w;
    p.k = a.k < 1 ? 1 : a.k;
    p.y_bf16 = a.y_bf16 ? 1 : 0;

    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kPThreads);
    cfg.dynamicSmemBytes = kPSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(2);
    int grid = pair_grid(cfg);
    // Never more CTAs than units could need (each unit keeps one pair busy).
    const long long tiles = (static_cast<long long>(a.S) + kPMaxN - 1) / kPMaxN + E;
    const long long units = tiles * (a.d_ff / 128) + tiles * ((a.d + 255) / 256);
    if (2 * units < grid) grid = static_cast<int>(2 * units);
    if (grid < 2) grid = 2;
    cfg.gridDim = dim3(static_cast<unsigned>(grid & ~1));
    cfg.numAttrs = a.pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, ffn_pair_kernel, tW1, tW3, tW2, tX, tH, tXs, tHs, p);
}

}  // namespace moe
