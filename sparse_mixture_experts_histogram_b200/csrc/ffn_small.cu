// ffn_small.cu -- the experts' feed-forward for narrow layers (d <= 1024),
// one persistent kernel with no dependency between CTAs.
//
// A work item is (expert e, token tile of BN rows, a range of 128-column
// chunks of the hidden width).  The item's BN rows of x (the tokens at
// positions r0.. of e's token list) are gathered once into shared memory, in
// the K-major 128-byte-swizzled layout the tensor cores read, and stay there
// for the whole item.  For every chunk c of its range the CTA then runs
//   up:    D0 = W1_e[c] X^T, D1 = W3_e[c] X^T        (tensor memory)
//   H:     silu(D0) * D1 -> bf16 -> shared memory, in the same operand layout
//   down:  Y += W2_e[:, c] H^T for every 128-row block of d (Y lives in
//          tensor memory for the whole item)
// and after its last chunk writes Y as one fp32 partial output
// [split, S, d], rows offsets[e] + position; the combine sums the splits of
// a row in a fixed order.  Every weight byte is read once, x rows are read
// once per item, H never leaves the SM, and a CTA waits only on its own
// warps.  The MMA warp issues up(c+1) before down(c), so the epilogue warps
// turn chunk c into H while the tensor cores already work on chunk c+1 (two
// up accumulators, two H buffers).
//
// Tensor memory: 2 up accumulators of 2*BN columns + (d/128) Y blocks of BN
// columns, at most 512.  Roles: warp 0 TMA producer (weights only), warp 1
// MMA issuer, warps 2..17 gather the item's x rows (16-byte cp.async) and
// run the epilogues, four warps per TMEM lane quarter taking turns at 8-token
// steps, so that the epilogue the tensor cores wait for after an item's last
// chunk, and the partial-output write, are short.
//
// Method: the SwiGLU expert w2(silu(w1 x) * w3 x) ("Mistral 8x7B SMoE
// architecture" (jsqmd.com) sec. 3.1 FeedForward) on each expert's own tokens
// ("MoE" (theaiera.top) sec. 10.4: index the tokens routed to the expert);
// splitting the hidden width and summing the partial down projections is the
// same sum over the hidden units.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace moe {

namespace {

constexpr int kEpiWarps = 16;                     // four per tensor-memory lane quarter
constexpr int kEpiPer = kEpiWarps / 4;            // warps per lane quarter
constexpr int kGatherRows = 4 * kEpiWarps;        // rows one gather pass covers
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kMaxStages = 6;
constexpr uint32_t kWTile = 128 * 128;  // 128 weight rows x 64 bf16
constexpr size_t kSmemBudget = 227 * 1024;
constexpr int kMaxTile = 64;            // token rows per item, at most
// barriers: full/empty [kMaxStages], ub_full/ub_empty/h_full/h_empty [2],
// y_full, y_empty, x_full, drain; then the TMEM address, the abort flag and
// the segment tables.  No alignment slack: the dynamic shared memory window
// starts on a 1024-byte boundary (the kernel checks it), which the 128-byte
// swizzled operand tiles need; without the slack a d = 512 layer keeps four
// weight stages next to its resident x rows.
constexpr size_t kFixedSmem = (2 * kMaxStages + 12) * 8 + 16 + (2 * (kMaxE + 1) + 4) * 4;

template <int BN, int MBD>
struct SmallCfg {
    static constexpr int KSU = 2 * MBD;                  // 64-column steps of d
    static constexpr uint32_t kStageBytes = 2 * kWTile;  // two 128-row weight tiles
    static constexpr uint32_t kXAtom = BN * 128u;        // BN rows x 64 bf16
    static constexpr uint32_t kXBytes = KSU * kXAtom;    // the item's rows of x, all of d
    static constexpr uint32_t kHAtom = BN * 128u;
    static constexpr uint32_t kHBytes = 2 * kHAtom;      // one H chunk: 128 hidden columns
    static constexpr int kUpCols = 2 * BN;               // D0 | D1
    static constexpr int kYCol0 = 2 * kUpCols;           // after two up accumulators
    static constexpr int kCols = kYCol0 + MBD * BN;      // MBD = d / 128 Y blocks
    static constexpr uint32_t kTmemCols = kCols <= 32 ? 32 : kCols <= 64 ? 64 : kCols <= 128 ? 128
                                        : kCols <= 256 ? 256 : 512;
    static constexpr size_t kRest = kFixedSmem + kXBytes + 2 * kHBytes;
    static constexpr int kFit = static_cast<int>((kSmemBudget - kRest) / kStageBytes);
    static constexpr int ST = kFit < kMaxStages ? kFit : kMaxStages;
    static constexpr size_t kSmem = kRest + static_cast<size_t>(ST) * kStageBytes;
    static_assert(kCols <= 512, "tensor memory");
    static_assert(kRest < kSmemBudget, "shared memory");
    static_assert(kSmem > kSmemBudget / 2, "one CTA per SM");
    static_assert(ST >= 3, "pipeline depth");
    static_assert(BN <= kMaxTile && BN % 32 == 0, "token rows per item");
};

struct SmallParams {
    int E, d, d_ff, S;
    int nsplit_max;         // at most this many chunk ranges per token tile
    int sms;                // SMs the work should cover in one wave
    int *nsplit_out;        // the count chosen (= partial outputs per row), for the combine
    size_t part_stride;     // floats between partial outputs
    const int32_t *counts;  // [E] rows of every segment (the router's totals)
    int32_t *offsets_out;   // [E+1] segment starts, written by CTA 0 for the combine
    const int32_t *perm;    // [E, perm_stride] token at each position of each segment
    int perm_stride;
    const __nv_bfloat16 *x; // [x_rows, d]
    int x_rows;
    float *Y;               // [nsplit, S, d]
    uint32_t *err;
    int act;                // expert activation: 0 silu(g) * b, 1 sigmoid(g) * b
};

struct Item {
    int e, r0, valid, c_beg, c_end, sp;
};

template <int BN>
__device__ __forceinline__ Item decode_item(int u, const int32_t *s_off, const int32_t *s_pre,
                                            int E, int nsplit, int mbu)
{
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_pre[mid] <= u) lo = mid;
        else hi = mid - 1;
    }
    Item it;
    it.e = lo;
    int local = u - s_pre[lo];
    it.sp = local % nsplit;
    const int tb = local / nsplit;
    const int cnt = s_off[lo + 1] - s_off[lo];
    it.r0 = s_off[lo] + tb * BN;
    const int rem = cnt - tb * BN;
    it.valid = rem < BN ? rem : BN;
    it.c_beg = it.sp * mbu / nsplit;
    it.c_end = (it.sp + 1) * mbu / nsplit;
    return it;
}

__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity)
{
    const uint64_t t0 = ptx::globaltimer();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::globaltimer() - t0 > 100000000ull) break;  // 100 ms
    }
}

__device__ __forceinline__ void fence_proxy_async_shared()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.wait_all;" ::: "memory");
}

template <int BN, int MBD>
__global__ void __launch_bounds__(kThreads, 1)
    ffn_small_kernel(const __grid_constant__ CUtensorMap tmW1,
                     const __grid_constant__ CUtensorMap tmW3,
                     const __grid_constant__ CUtensorMap tmW2, const SmallParams p)
{
    using C = SmallCfg<BN, MBD>;
    constexpr int ST = C::ST;
    constexpr int KSU = C::KSU;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (ptx::smem_addr(smem) & 1023u) {
        // Nothing is set up yet; every thread leaves.
        if (threadIdx.x == 0) atomicOr(p.err, kErrLayout);
        return;
    }
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    uint8_t *xbuf = smem + ST * C::kStageBytes;  // the item's x rows, KSU atoms
    uint8_t *hbuf = xbuf + C::kXBytes;           // 2 H chunks
    uint64_t *full = reinterpret_cast<uint64_t *>(hbuf + 2 * C::kHBytes);
    uint64_t *empty = full + kMaxStages;
    uint64_t *ub_full = empty + kMaxStages;  // [2]
    uint64_t *ub_empty = ub_full + 2;        // [2]
    uint64_t *h_full = ub_empty + 2;         // [2]
    uint64_t *h_empty = h_full + 2;          // [2]
    uint64_t *y_full = h_empty + 2;
    uint64_t *y_empty = y_full + 1;
    uint64_t *x_full = y_empty + 1;
    uint64_t *drain = x_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile uint32_t *abort_flag = tmem_slot + 1;
    int32_t *s_off = reinterpret_cast<int32_t *>(tmem_slot + 4);
    int32_t *s_pre = s_off + (kMaxE + 1);
    int32_t *s_nsplit = s_pre + (kMaxE + 1);

    const int E = p.E;
    const int MBU = p.d_ff / 128;
    constexpr int NPAIR = (MBD + 1) / 2;

    if (threadIdx.x == 0) {
        for (int s = 0; s < ST; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&ub_full[b], 1);
            ptx::mbar_init(&ub_empty[b], kEpiWarps);
            ptx::mbar_init(&h_full[b], kEpiWarps);
            ptx::mbar_init(&h_empty[b], 1);
        }
        ptx::mbar_init(y_full, 1);
        ptx::mbar_init(y_empty, kEpiWarps);
        ptx::mbar_init(x_full, kEpiWarps);
        ptx::mbar_init(drain, 1);
        *abort_flag = 0u;
        ptx::fence_barrier_init();
    }
    if (threadIdx.x == 32) {
        ptx::prefetch_tensormap(&tmW1);
        ptx::prefetch_tensormap(&tmW3);
        ptx::prefetch_tensormap(&tmW2);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, C::kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::grid_dep_wait();
    if (warp == 2) {
        // Segment starts are the exclusive prefix of the router's per-expert
        // totals (CTA 0 writes them out for the combine).  Then token tiles
        // per expert and the number of chunk ranges per tile: as many as fit
        // one wave of items on the SMs (the same choice in every CTA, since
        // all read the same totals).
        const int per = (E + 31) >> 5;
        const int base = lane * per;
        bool bad = false;
        int cnt[kMaxE / 32];
        int rows = 0, nt = 0;
#pragma unroll
        for (int i = 0; i < kMaxE / 32; ++i) {
            const int e = base + i;
            int c = 0;
            if (i < per && e < E) {
                c = p.counts[e];
                if (c < 0 || c > p.perm_stride) {
                    bad = true;
                    c = 0;
                }
            }
            cnt[i] = c;
            rows += c;
            nt += (c + BN - 1) / BN;
        }
        int incl_rows = rows;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl_rows, off);
            if (lane >= off) incl_rows += v;
        }
        if (__shfl_sync(0xffffffffu, incl_rows, 31) > p.S) bad = true;
        bad = __any_sync(0xffffffffu, bad);
        if (bad) {
            nt = 0;
            if (lane == 0) atomicOr(p.err, kErrOffsets);
        }
        int o = incl_rows - rows;
#pragma unroll
        for (int i = 0; i < kMaxE / 32; ++i) {
            const int e = base + i;
            if (i < per && e < E) {
                const int oe = bad ? 0 : o;
                s_off[e] = oe;
                if (blockIdx.x == 0) p.offsets_out[e] = oe;
                o += cnt[i];
            }
        }
        if (lane == 31) {
            const int end = bad ? 0 : incl_rows;
            s_off[E] = end;
            if (blockIdx.x == 0) p.offsets_out[E] = end;
        }
        __syncwarp();
        int incl = nt;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        const int tiles = __shfl_sync(0xffffffffu, incl, 31);
        int ns = tiles > 0 ? p.sms / tiles : 1;
        ns = ns < 1 ? 1 : (ns > p.nsplit_max ? p.nsplit_max : ns);
        int run = (incl - nt) * ns;
        for (int i = 0; i < per; ++i) {
            const int e = base + i;
            if (e < E) {
                s_pre[e] = run;
                if (!bad) run += ((s_off[e + 1] - s_off[e] + BN - 1) / BN) * ns;
            }
        }
        if (lane == 31) {
            s_pre[E] = incl * ns;
            s_nsplit[0] = ns;
            if (blockIdx.x == 0) *p.nsplit_out = ns;
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int total = s_pre[E];
    const int nsplit = s_nsplit[0];

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            uint32_t stage = 0, phase = 0, issued = 0;
            uint32_t last_parity[kMaxStages];
#pragma unroll
            for (int s = 0; s < kMaxStages; ++s) last_parity[s] = 0;
            // Every weight byte is read once: let the weight stream leave L2
            // first, so that the gathered x rows, the token lists and the
            // partial outputs the combine reads back stay there (measured
            // 9-12% faster on the sweep than the default policy).
            const uint64_t pol = ptx::policy_evict_first();
            bool stop = false;
            auto next_stage = [&]() -> uint8_t * {
                if (!bounded_wait(&empty[stage], phase ^ 1u, abort_flag, p.err, kErrTimeoutMma))
                    return nullptr;
                ptx::mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
                return smem + stage * C::kStageBytes;
            };
            auto advance = [&]() {
                issued |= 1u << stage;
                last_parity[stage] = phase;
                if (++stage == static_cast<uint32_t>(ST)) {
                    stage = 0;
                    phase ^= 1u;
                }
            };
            for (int u = blockIdx.x; u < total && !stop; u += gridDim.x) {
                const Item it = decode_item<BN>(u, s_off, s_pre, E, nsplit, MBU);
                const int nc = it.c_end - it.c_beg;
                for (int j = 0; j <= nc && !stop; ++j) {
                    if (j < nc) {  // up: W1, W3 rows of chunk c
                        const int arow = it.e * p.d_ff + (it.c_beg + j) * 128;
                        for (int ks = 0; ks < KSU; ++ks) {
                            uint8_t *sa = next_stage();
                            if (!sa) { stop = true; break; }
                            ptx::tma_load_2d_hint(sa, &tmW1, &full[stage], ks * 64, arow, pol);
                            ptx::tma_load_2d_hint(sa + kWTile, &tmW3, &full[stage], ks * 64, arow, pol);
                            advance();
                        }
                    }
                    if (j >= 1 && !stop) {  // down: W2 columns of chunk c-1, all rows of d
                        const int col = (it.c_beg + j - 1) * 128;
                        for (int pr = 0; pr < NPAIR && !stop; ++pr) {
                            const int arow = it.e * p.d + pr * 256;
                            for (int kh = 0; kh < 2; ++kh) {
                                uint8_t *sa = next_stage();
                                if (!sa) { stop = true; break; }
                                ptx::tma_load_2d_hint(sa, &tmW2, &full[stage], col + kh * 64, arow, pol);
                                ptx::tma_load_2d_hint(sa + kWTile, &tmW2, &full[stage], col + kh * 64,
                                                      arow + 128, pol);
                                advance();
                            }
                        }
                    }
                }
            }
            for (int s = 0; s < ST; ++s)
                if (issued & (1u << s)) drain_wait(&full[s], last_parity[s]);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            int n = 0, items = 0;
            bool stop = false;
            const uint32_t sx = ptx::smem_addr(xbuf);
            for (int u = blockIdx.x; u < total && !stop; u += gridDim.x) {
                const Item it = decode_item<BN>(u, s_off, s_pre, E, nsplit, MBU);
                const int nc = it.c_end - it.c_beg;
                const uint32_t idesc = ptx::idesc_bf16_f32(128, ((it.valid + 15) >> 4) << 4);
                if (!bounded_wait(x_full, static_cast<uint32_t>(items) & 1u, abort_flag, p.err,
                                  kErrTimeoutEpi))
                    break;
                for (int j = 0; j <= nc && !stop; ++j) {
                    if (j < nc) {
                        const int ub = (n + j) & 1;
                        const uint32_t use = static_cast<uint32_t>((n + j) >> 1);
                        if (!bounded_wait(&ub_empty[ub], (use & 1u) ^ 1u, abort_flag, p.err,
                                          kErrTimeoutEpi)) { stop = true; break; }
                        ptx::tc_fence_after();
                        const uint32_t d0 = tmem + static_cast<uint32_t>(ub * C::kUpCols);
                        for (int ks = 0; ks < KSU; ++ks) {
                            if (!bounded_wait(&full[stage], phase, abort_flag, p.err, kErrTimeoutTma)) {
                                stop = true;
                                break;
                            }
                            ptx::tc_fence_after();
                            const uint32_t sa = ptx::smem_addr(smem + stage * C::kStageBytes);
                            const uint32_t sb = sx + static_cast<uint32_t>(ks) * C::kXAtom;
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint64_t bd = ptx::sw128_kmajor_desc(sb + kk * 32);
                                const uint32_t acc = (ks | kk) ? 1u : 0u;
                                ptx::tc_mma_bf16(d0, ptx::sw128_kmajor_desc(sa + kk * 32), bd, idesc, acc);
                                ptx::tc_mma_bf16(d0 + BN, ptx::sw128_kmajor_desc(sa + kWTile + kk * 32), bd,
                                                 idesc, acc);
                            }
                            ptx::tc_commit(&empty[stage]);
                            if (++stage == static_cast<uint32_t>(ST)) {
                                stage = 0;
                                phase ^= 1u;
                            }
                        }
                        if (stop) break;
                        ptx::tc_commit(&ub_full[ub]);
                    }
                    if (j >= 1) {
                        const int jj = j - 1;
                        const int hb = (n + jj) & 1;
                        const uint32_t use = static_cast<uint32_t>((n + jj) >> 1);
                        if (jj == 0 && !bounded_wait(y_empty, (static_cast<uint32_t>(items) & 1u) ^ 1u,
                                                     abort_flag, p.err, kErrTimeoutEpi)) {
                            stop = true;
                            break;
                        }
                        if (!bounded_wait(&h_full[hb], use & 1u, abort_flag, p.err, kErrTimeoutEpi)) {
                            stop = true;
                            break;
                        }
                        ptx::tc_fence_after();
                        const uint32_t hsa = ptx::smem_addr(hbuf + hb * C::kHBytes);
                        for (int pr = 0; pr < NPAIR && !stop; ++pr) {
                            const uint32_t y0 = tmem + static_cast<uint32_t>(C::kYCol0 + 2 * pr * BN);
                            const bool has1 = 2 * pr + 1 < MBD;
                            for (int kh = 0; kh < 2; ++kh) {
                                if (!bounded_wait(&full[stage], phase, abort_flag, p.err,
                                                  kErrTimeoutTma)) {
                                    stop = true;
                                    break;
                                }
                                ptx::tc_fence_after();
                                const uint32_t sa = ptx::smem_addr(smem + stage * C::kStageBytes);
                                const uint32_t sb = hsa + kh * C::kHAtom;
#pragma unroll
                                for (int kk = 0; kk < 4; ++kk) {
                                    const uint64_t bd = ptx::sw128_kmajor_desc(sb + kk * 32);
                                    const uint32_t acc = (jj | kh | kk) ? 1u : 0u;
                                    ptx::tc_mma_bf16(y0, ptx::sw128_kmajor_desc(sa + kk * 32), bd, idesc, acc);
                                    if (has1)
                                        ptx::tc_mma_bf16(y0 + BN, ptx::sw128_kmajor_desc(sa + kWTile + kk * 32),
                                                         bd, idesc, acc);
                                }
                                ptx::tc_commit(&empty[stage]);
                                if (++stage == static_cast<uint32_t>(ST)) {
                                    stage = 0;
                                    phase ^= 1u;
                                }
                            }
                        }
                        if (stop) break;
                        ptx::tc_commit(&h_empty[hb]);
                    }
                }
                if (stop) break;
                // Arrives when every MMA of the item is done: Y is complete and
                // the x rows may be replaced by the next item's.
                ptx::tc_commit(y_full);
                n += nc;
                ++items;
            }
            ptx::tc_commit(drain);
            drain_wait(drain, 0u);
        }
    } else {
        // ---------------------------------------------------------------- gather + epilogue
        // Warps 2..17: lane quarter q = warp % 4 of tensor memory; the
        // kEpiPer warps of a quarter take turns at eight-token steps.
        const int q = warp & 3;
        const int turn = (warp - 2) >> 2;  // 0 .. kEpiPer-1
        const int g = threadIdx.x - 64;  // 0..255
        const int f = 32 * q + lane;     // hidden column of the chunk / row of a Y block
        const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
        const uint32_t kk = static_cast<uint32_t>(f & 63);
        const uint32_t hcol_off = (f >> 6) * C::kHAtom + (kk & 7u) * 2u;
        const uint32_t hchunk = kk >> 3;
        const uint32_t sx = ptx::smem_addr(xbuf);
        // Gather share of this thread: 16-byte piece gc of rows gr, gr+32, ...
        // of every 64-column atom.
        const uint32_t gc = static_cast<uint32_t>(g & 7);
        const int gr = g >> 3;  // 0..31
        int n = 0, items = 0;
        bool stop = false;
        for (int u = blockIdx.x; u < total && !stop; u += gridDim.x) {
            const Item it = decode_item<BN>(u, s_off, s_pre, E, nsplit, MBU);
            const int nc = it.c_end - it.c_beg;
            {
                // x rows of the item's tokens; rows past the segment's end
                // repeat its first token (their columns are never stored).
                // The previous item's MMAs are all done (its y_full was seen).
                const int32_t *pl = p.perm + static_cast<size_t>(it.e) * p.perm_stride +
                                    (it.r0 - s_off[it.e]);
                constexpr int kPasses = (BN + kGatherRows - 1) / kGatherRows;
                int tok[kPasses];
#pragma unroll
                for (int m = 0; m < kPasses; ++m) {
                    const int r = gr + kGatherRows * m;
                    int t = __ldg(pl + (r < it.valid ? r : 0));
                    if (static_cast<unsigned>(t) >= static_cast<unsigned>(p.x_rows)) {
                        atomicOr(p.err, kErrIndex);
                        t = 0;
                    }
                    tok[m] = t;
                }
#pragma unroll
                for (int m = 0; m < kPasses; ++m) {
                    const int r = gr + kGatherRows * m;
                    if (r >= BN) break;
                    const __nv_bfloat16 *src = p.x + static_cast<size_t>(tok[m]) * p.d + gc * 8;
                    const uint32_t dst = sx + static_cast<uint32_t>(r) * 128u +
                                         ((gc ^ (static_cast<uint32_t>(r) & 7u)) << 4);
#pragma unroll
                    for (int ks = 0; ks < KSU; ++ks)
                        cp_async16(dst + static_cast<uint32_t>(ks) * C::kXAtom, src + ks * 64);
                }
                cp_async_wait_all();
                fence_proxy_async_shared();  // x rows are read by the tensor cores (async proxy)
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(x_full);
            }
            for (int j = 0; j < nc; ++j) {
                const int ub = (n + j) & 1;
                const uint32_t use = static_cast<uint32_t>((n + j) >> 1);
                if (!bounded_wait_warp(&ub_full[ub], use & 1u, abort_flag, p.err, kErrTimeoutMma) ||
                    !bounded_wait_warp(&h_empty[ub], (use & 1u) ^ 1u, abort_flag, p.err,
                                       kErrTimeoutMma)) {
                    stop = true;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t tb = tmem + lane_base + static_cast<uint32_t>(ub * C::kUpCols);
                uint8_t *hb = hbuf + ub * C::kHBytes + hcol_off;
                // Eight tokens per step: a short loop body keeps the code the
                // epilogue runs small (it is cold at the start of every launch).
#pragma unroll 1
                for (int c0 = 8 * turn; c0 < it.valid; c0 += 8 * kEpiPer) {
                    uint32_t a[8], b[8];
                    ptx::tmem_ld8(tb + static_cast<uint32_t>(c0), a);
                    ptx::tmem_ld8(tb + static_cast<uint32_t>(BN + c0), b);
                    ptx::tc_wait_ld();
                    uint8_t *hrow = hb + c0 * 128;
#pragma unroll
                    for (int jt = 0; jt < 8; ++jt) {
                        if (c0 + jt < it.valid) {
                            const float gv = __uint_as_float(a[jt]);
                            const float bv = __uint_as_float(b[jt]);
                            const float h = __fdividef(p.act ? bv : gv * bv, 1.0f + __expf(-gv));
                            // row c0+jt (c0 is a multiple of 8, so the row's swizzle
                            // phase is jt), column f, 128-byte-swizzled layout
                            *reinterpret_cast<__nv_bfloat16 *>(hrow + jt * 128 + ((hchunk ^ jt) << 4)) =
                                __float2bfloat16_rn(h);
                        }
                    }
                }
                ptx::tc_fence_before();
                fence_proxy_async_shared();  // H is read by the tensor cores (async proxy)
                __syncwarp();
                if (lane == 0) {
                    ptx::mbar_arrive(&ub_empty[ub]);
                    ptx::mbar_arrive(&h_full[ub]);
                }
            }
            if (stop) break;
            // Y of the item: MBD blocks of 128 output columns, rows r0.. of split sp.
            if (!bounded_wait_warp(y_full, static_cast<uint32_t>(items) & 1u, abort_flag, p.err,
                                   kErrTimeoutMma)) {
                stop = true;
                break;
            }
            ptx::tc_fence_after();
            float *Y = p.Y + it.sp * p.part_stride;
#pragma unroll 1
            for (int m = 0; m < MBD; ++m) {
                const uint32_t yb = tmem + lane_base + static_cast<uint32_t>(C::kYCol0 + m * BN);
                float *yc = Y + static_cast<size_t>(it.r0) * p.d + m * 128 + f;
#pragma unroll 1
                for (int c0 = 8 * turn; c0 < it.valid; c0 += 8 * kEpiPer) {
                    uint32_t y[8];
                    ptx::tmem_ld8(yb + static_cast<uint32_t>(c0), y);
                    ptx::tc_wait_ld();
#pragma unroll
                    for (int jt = 0; jt < 8; ++jt)
                        if (c0 + jt < it.valid)
                            yc[static_cast<size_t>(c0 + jt) * p.d] = __uint_as_float(y[jt]);
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(y_empty);
            n += nc;
            ++items;
        }
    }

    ptx::grid_dep_launch();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int BN, int MBD>
cudaError_t launch_small_cfg(const FfnLaunch &a, int nsplit_max, int *nsplit_out, cudaStream_t s)
{
    using C = SmallCfg<BN, MBD>;
    if (a.perm == nullptr || a.counts == nullptr || a.offsets_out == nullptr || a.x_rows < 1)
        return cudaErrorInvalidValue;
    CUtensorMap tW1, tW3, tW2;
    cudaError_t e = make_tmap_bf16(&tW1, a.W1, static_cast<uint64_t>(a.E) * a.d_ff, a.d, 128);
    if (e == cudaSuccess) e = make_tmap_bf16(&tW3, a.W3, static_cast<uint64_t>(a.E) * a.d_ff, a.d, 128);
    if (e == cudaSuccess) e = make_tmap_bf16(&tW2, a.W2, static_cast<uint64_t>(a.E) * a.d, a.d_ff, 128);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(ffn_small_kernel<BN, MBD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(C::kSmem));
    if (e != cudaSuccess) return e;
    SmallParams p{};
    p.act = a.act;
    p.E = a.E;
    p.d = a.d;
    p.d_ff = a.d_ff;
    p.S = a.S;
    p.nsplit_max = nsplit_max;
    p.sms = device_sm_count();
    p.nsplit_out = nsplit_out;
    p.part_stride = static_cast<size_t>(a.S) * a.d;
    p.counts = a.counts;
    p.offsets_out = a.offsets_out;
    p.perm = a.perm;
    p.perm_stride = a.perm_stride;
    p.x = reinterpret_cast<const __nv_bfloat16 *>(a.x);
    p.x_rows = a.x_rows;
    p.Y = a.Y;
    p.err = a.err;
    const long long items = ((static_cast<long long>(a.S) + BN - 1) / BN + a.E) * nsplit_max;
    long long grid = device_sm_count();
    if (items < grid) grid = items;
    if (grid < 1) grid = 1;
    return launch_pdl(ffn_small_kernel<BN, MBD>, dim3(static_cast<unsigned>(grid)),
                      dim3(kThreads), C::kSmem, s, a.pdl, tW1, tW3, tW2, p);
}

template <int MBD>
cudaError_t launch_small_d(const FfnLaunch &a, int nsplit_max, int *nsplit_out, cudaStream_t s)
{
    constexpr int kBN = (4 + MBD) * 64 <= 512 ? 64 : 32;
    return launch_small_cfg<kBN, MBD>(a, nsplit_max, nsplit_out, s);
}

}  // namespace

bool ffn_small_supported(int d) { return d >= 128 && d <= 1024 && d % 128 == 0; }

int ffn_small_tile(int d) { return (4 + d / 128) * 64 <= 512 ? 64 : 32; }

int ffn_small_splits(int S, int E, int d, int d_ff)
{
    // Upper bound of the chunk ranges per token tile the kernel may choose
    // (it picks SMs / tiles from the actual tiles, at least ceil(S / BN) of
    // them): no more ranges than hidden chunks and never more than 32.
    (void)E;
    const int bn = ffn_small_tile(d);
    const long long min_tiles = std::max<long long>(1, (static_cast<long long>(S) + bn - 1) / bn);
    const long long cap = std::max<long long>(1, 148 / min_tiles);
    return static_cast<int>(std::max<long long>(1, std::min<long long>({cap, d_ff / 128, 32})));
}

cudaError_t launch_ffn_small(const FfnLaunch &a, int nsplit_max, int *nsplit_out, cudaStream_t s)
{
    switch (a.d / 128) {
    case 1: return launch_small_d<1>(a, nsplit_max, nsplit_out, s);
    case 2: return launch_small_d<2>(a, nsplit_max, nsplit_out, s);
    case 3: return launch_small_d<3>(a, nsplit_max, nsplit_out, s);
    case 4: return launch_small_d<4>(a, nsplit_max, nsplit_out, s);
    case 5: return launch_small_d<5>(a, nsplit_max, nsplit_out, s);
    case 6: return launch_small_d<6>(a, nsplit_max, nsplit_out, s);
    case 7: return launch_small_d<7>(a, nsplit_max, nsplit_out, s);
    case 8: return launch_small_d<8>(a, nsplit_max, nsplit_out, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
