// common.cuh -- pieces shared by the kernels: bounded pipeline waits, the
// per-tile expert histogram with stable ranks, and the "last CTA" scan that
// turns the tile histograms into expert offsets.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace moe {

// Error bits of the device error word (same values as the public header).
constexpr uint32_t kErrTimeoutTma = 0x1u;
constexpr uint32_t kErrTimeoutMma = 0x2u;
constexpr uint32_t kErrTimeoutEpi = 0x4u;
constexpr uint32_t kErrOffsets = 0x8u;
constexpr uint32_t kErrIndex = 0x10u;
constexpr uint32_t kErrLayout = 0x20u;

constexpr int kTileTokens = 128;   // tokens per routing tile (= MMA M of the router)
constexpr int kMaxK = 8;
constexpr int kMaxE = 256;
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // 2 s: far above any legitimate wait

// Wait until `bar` completes the phase of the given parity.  Gives up after
// kWaitTimeoutNs, or as soon as another role of the CTA has given up (the
// shared abort flag), so that a broken pipeline ends the kernel with an
// error bit instead of hanging the GPU.  Returns false when it gave up.
__device__ __forceinline__ bool bounded_wait(uint64_t *bar, uint32_t parity,
                                             volatile uint32_t *abort_flag, uint32_t *gerr,
                                             uint32_t code)
{
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if ((it & 63u) == 0 && ptx::globaltimer() - t0 > kWaitTimeoutNs) {
            *abort_flag = 1u;
            if (gerr) atomicOr(gerr, code);
            return false;
        }
    }
}

// Warp-uniform version for warps whose lanes all consume the result (the
// epilogue): every lane waits, and the warp proceeds only if all lanes saw
// the phase complete.
__device__ __forceinline__ bool bounded_wait_warp(uint64_t *bar, uint32_t parity,
                                                  volatile uint32_t *abort_flag, uint32_t *gerr,
                                                  uint32_t code)
{
    const bool ok = bounded_wait(bar, parity, abort_flag, gerr, code);
    const bool all = __all_sync(0xffffffffu, ok);
    if (!all) *abort_flag = 1u;
    return all;
}

// Readiness of up to 32 consecutive H blocks, counters ctr[0..n): bit i set
// when ctr[i] >= target.  Relaxed loads, all issued before any result is
// used, then one acquire fence for all of them (an acquire load per counter
// would order each load after the previous one): a down unit whose blocks
// were published long ago, the common case, pays one memory round trip for
// the window instead of one per K step.  Blocks found not ready are then
// waited for one by one.
__device__ __forceinline__ uint32_t ready_window(const uint32_t *ctr, int n, uint32_t target)
{
    uint32_t v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        v[i] = target;
        if (i < n) asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v[i]) : "l"(ctr + i) : "memory");
    }
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) m |= (v[i] >= target ? 1u : 0u) << i;
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    return m;
}

// Shared memory of one routing tile's histogram / rank computation.
struct DispatchSmem {
    int32_t sel[kTileTokens][kMaxK];   // expert of (row, slot); -1 = no token
    int32_t rnk[kTileTokens][kMaxK];   // rank among the same expert inside the 32-row group
    int32_t cnt[4][kMaxE];             // per 32-row group, per expert counts
    int32_t pre[4][kMaxE];             // exclusive prefix of cnt over the groups
    int32_t tot[kMaxE];
    int32_t total;
    uint32_t is_last;
};

struct DispatchOut {
    int32_t *tilecnt;    // [ntiles, E] per-tile expert counts
    int32_t *tilebase;   // [ntiles, E] first x_perm row of (tile, expert)
    int32_t *rank;       // [T, k] rank of (t, j) among its expert's pairs in its tile
    int32_t *offsets;    // [E+1] expert segment starts (written by the last tile)
    int32_t *counts;     // [E] per-expert pair counts, or nullptr
    uint32_t *done;      // tile completion counter (zero at kernel start)
    int ntiles;
    int cap;             // per-expert capacity (segments hold min(count, cap) rows), or -1
};

// Called by the 128 threads of one routing tile after they filled sm.sel.
// `row` is the calling thread's row (0..127), rows 32q..32q+31 form group q.
// Ranks are stable in token order: pair (t, j) of expert e gets the number of
// tokens t' < t of the same tile that also chose e.  The last tile to finish
// turns all tile counts into expert offsets and tile bases, so that the row
// of (t, j) in x_perm is tilebase[tile, e] + rank[t, j] (dropless, no gaps).
__device__ __forceinline__ void dispatch_tile(DispatchSmem &sm, int row, int tile, int T, int E,
                                              int k, const DispatchOut &o, int bar_id)
{
    const int q = row >> 5;
    const int lane = row & 31;
    uint32_t *mask = reinterpret_cast<uint32_t *>(&sm.cnt[0][0]);  // [4][kMaxE] lane bitmasks
    for (int i = row; i < 4 * kMaxE; i += kTileTokens) mask[i] = 0u;
    ptx::named_bar(bar_id, kTileTokens);

    // Bit `lane` of mask[q][e] is set when row 32q+lane chose expert e (a row
    // never chooses an expert twice).  The rank of (row, j) among its group's
    // rows with the same expert is the number of lower lanes in that mask.
    for (int j = 0; j < k; ++j) {
        const int e = sm.sel[row][j];
        if (e >= 0) atomicOr(&mask[q * kMaxE + e], 1u << lane);
    }
    ptx::named_bar(bar_id, kTileTokens);
    const uint32_t below = (1u << lane) - 1u;
    for (int j = 0; j < k; ++j) {
        const int e = sm.sel[row][j];
        if (e >= 0) sm.rnk[row][j] = __popc(mask[q * kMaxE + e] & below);
    }
    ptx::named_bar(bar_id, kTileTokens);  // every rank read its mask before it is replaced
    // cnt[g][e] = popc(mask[g][e]), in place.
    for (int i = row; i < 4 * kMaxE; i += kTileTokens)
        sm.cnt[0][i] = __popc(mask[i]);
    ptx::named_bar(bar_id, kTileTokens);

    const bool single = (o.ntiles == 1);
    for (int e = row; e < E; e += kTileTokens) {
        int run = 0;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            sm.pre[g][e] = run;
            run += sm.cnt[g][e];
        }
        if (single) sm.tot[e] = run;
        else o.tilecnt[(size_t)tile * E + e] = run;
    }
    ptx::named_bar(bar_id, kTileTokens);

    const int t = tile * kTileTokens + row;
    if (t < T) {
        for (int j = 0; j < k; ++j) {
            const int e = sm.sel[row][j];
            o.rank[(size_t)t * k + j] = (e >= 0) ? sm.pre[q][e] + sm.rnk[row][j] : -1;
        }
    }
    if (!single) {
        __threadfence();
        ptx::named_bar(bar_id, kTileTokens);
        if (row == 0) sm.is_last = (atomicAdd(o.done, 1u) == (uint32_t)o.ntiles - 1u) ? 1u : 0u;
        ptx::named_bar(bar_id, kTileTokens);
        if (!sm.is_last) return;
        __threadfence();

        // Last tile: per expert, exclusive prefix of the tile counts (relative
        // tile bases) and the expert total.
        for (int e = row; e < E; e += kTileTokens) {
            int run = 0;
            int tl = 0;
            for (; tl + 8 <= o.ntiles; tl += 8) {
                int c[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) c[u] = __ldcg(&o.tilecnt[(size_t)(tl + u) * E + e]);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    o.tilebase[(size_t)(tl + u) * E + e] = run;
                    run += c[u];
                }
            }
            for (; tl < o.ntiles; ++tl) {
                const int c = __ldcg(&o.tilecnt[(size_t)tl * E + e]);
                o.tilebase[(size_t)tl * E + e] = run;
                run += c;
            }
            sm.tot[e] = run;
        }
    }
    ptx::named_bar(bar_id, kTileTokens);

    // Exclusive scan of the expert totals (E <= 256) by the first warp.
    if (q == 0) {
        const int per = (E + 31) >> 5;
        const int base = lane * per;
        // With a capacity an expert's segment holds only its first `cap`
        // pairs in token order.
        if (o.cap >= 0)
            for (int i = 0; i < per; ++i)
                if (base + i < E) sm.tot[base + i] = min(sm.tot[base + i], o.cap);
        __syncwarp();
        int local = 0;
        for (int i = 0; i < per; ++i)
            if (base + i < E) local += sm.tot[base + i];
        int incl = local;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        int run = incl - local;
        for (int i = 0; i < per; ++i) {
            if (base + i < E) {
                const int c = sm.tot[base + i];
                sm.tot[base + i] = run;
                run += c;
            }
        }
        if (lane == 31) sm.total = incl;
    }
    ptx::named_bar(bar_id, kTileTokens);

    for (int e = row; e <= E; e += kTileTokens) {
        const int off = (e < E) ? sm.tot[e] : sm.total;
        o.offsets[e] = off;
        if (e < E && o.counts) o.counts[e] = ((e + 1 < E) ? sm.tot[e + 1] : sm.total) - off;
    }
    if (single) {
        for (int e = row; e < E; e += kTileTokens) o.tilebase[e] = sm.tot[e];
    } else {
        const int n = o.ntiles * E;
        for (int i = row; i < n; i += kTileTokens) o.tilebase[i] += sm.tot[i % E];
        if (row == 0) *o.done = 0u;
    }
}

// Slot assignment without a token order: every (token, slot) pair gets a
// position inside its expert's segment from one global atomic per (CTA,
// expert) plus its rank among the CTA's own pairs.  Positions are unique and
// dense but their order inside a segment depends on scheduling; a row's
// expert output does not depend on where the row sits, so the layer's result
// is the same whatever order comes out.  When the grid has finished, gcnt
// holds every expert's total; the expert kernel turns the totals into
// segment starts itself, so no CTA of the router waits for the others.
struct SlotOut {
    int32_t *gcnt;     // [E] pairs per expert (zero before the launch)
    int32_t *pos;      // [T, k] position of the pair inside its expert's segment (-1: none)
    int32_t *perm;     // [E, perm_stride] token at each position of each expert
    int perm_stride;   // >= T
};

// Called by threads tid = 0..nthr-1 (a multiple of 32) of a CTA whose tokens
// t0 .. t0+ntok-1 chose ds.sel[r][j] (-1 = none); `bar_id` is a named
// barrier over exactly those threads.
__device__ __forceinline__ void assign_slots(DispatchSmem &ds, int t0, int ntok, int T, int E,
                                             int k, const SlotOut &o, int tid, int nthr,
                                             int bar_id)
{
    int32_t *hist = ds.cnt[0];
    int32_t *base = ds.pre[0];
    for (int e = tid; e < E; e += nthr) hist[e] = 0;
    ptx::named_bar(bar_id, nthr);
    const int npairs = ntok * k;
    for (int i = tid; i < npairs; i += nthr) {
        const int r = i / k;
        const int j = i - r * k;
        const int e = ds.sel[r][j];
        ds.rnk[r][j] = e >= 0 ? atomicAdd(&hist[e], 1) : -1;
    }
    ptx::named_bar(bar_id, nthr);
    for (int e = tid; e < E; e += nthr) {
        const int c = hist[e];
        base[e] = c ? atomicAdd(&o.gcnt[e], c) : 0;
    }
    ptx::named_bar(bar_id, nthr);
    for (int i = tid; i < npairs; i += nthr) {
        const int r = i / k;
        const int j = i - r * k;
        const int t = t0 + r;
        if (t < T) {
            const int e = ds.sel[r][j];
            int p = -1;
            if (e >= 0) {
                p = base[e] + ds.rnk[r][j];
                o.perm[static_cast<size_t>(e) * o.perm_stride + p] = t;
            }
            o.pos[static_cast<size_t>(t) * k + j] = p;
        }
    }
}

}  // namespace moe
