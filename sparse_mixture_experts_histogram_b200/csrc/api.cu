// api.cu -- the C ABI declared in include/moe.h: argument checks, workspace
// layout, tensor-map encoding and the launch sequence of each entry point.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "internal.h"
#include "moe.h"

namespace moe {

namespace {

constexpr size_t kAlign = 256;
constexpr size_t kHeaderBytes = 256;  // error word @0, routing counter @4, ranks counter @8,
                                      // partial outputs per row of the expert kernel @12,
                                      // work counters of the routed @16 and shared @20
                                      // expert kernels

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

constexpr int kMaxRanksHost = 8;  // ranks of one expert-parallel group (kMaxRanks of ep.cu)

struct Layout {
    size_t tilectr, hready, hready_s, gcnt;
    size_t zero_bytes;  // [0, zero_bytes) is cleared at the start of every call
    size_t tilecnt, tilebase, rank, offsets, counts, idx, w, row, slotpos, slotrow, perm, xperm, H,
        Y, Hs, Ys, total;
};

// Token lists of the slot mode: one row of perm_stride entries per expert.
int perm_stride(int T) { return (T + 15) / 16 * 16; }

// Partial expert outputs the routed experts' kernel writes per row: the
// narrow-layer kernel splits the hidden width, the general one may split the
// down projection's K.
int ffn_splits(int S, int E, int d, int d_ff)
{
    return ffn_small_supported(d) ? ffn_small_splits(S, E, d, d_ff) : down_ksplit(S, E, d, d_ff);
}

// Workspace of moe_forward_ex (a superset of every other entry point's need).
Layout forward_layout(int T, int d, int E, int d_ff, int k, int d_ffs)
{
    Layout L{};
    size_t o = kHeaderBytes;
    auto take = [&](size_t bytes) {
        const size_t r = o;
        o += align_up(bytes);
        return r;
    };
    const size_t ntiles = (static_cast<size_t>(T) + 127) / 128;
    const size_t S = static_cast<size_t>(T) * k;
    L.tilectr = take(ntiles * 4);
    L.hready = take(ffn_ready_counters(static_cast<int>(S), E, d_ff) * 4);
    L.hready_s = d_ffs > 0 ? take(ffn_ready_counters(T, 1, d_ffs) * 4) : 0;
    L.gcnt = take(static_cast<size_t>(E) * 4);
    L.zero_bytes = o;
    L.tilecnt = take(ntiles * E * 4);
    L.tilebase = take(ntiles * E * 4);
    L.rank = take(S * 4);
    L.offsets = take((static_cast<size_t>(E) + 1) * 4);
    L.counts = take(static_cast<size_t>(E) * 4);
    L.idx = take(S * 4);
    L.w = take(S * 4);
    L.row = take(S * 4);
    L.slotpos = take(S * 4);
    L.slotrow = take(S * 4);
    L.perm = take(static_cast<size_t>(E) * perm_stride(T) * 4);
    L.xperm = take(S * d * 2);
    L.H = take(S * d_ff * 2);
    L.Y = take(S * d * 4 * static_cast<size_t>(ffn_splits(static_cast<int>(S), E, d, d_ff)));
    if (d_ffs > 0) {
        L.Hs = take(static_cast<size_t>(T) * d_ffs * 2);
        L.Ys = take(static_cast<size_t>(T) * d * 4);
    } else {
        L.Hs = L.Ys = 0;
    }
    L.total = o;
    return L;
}

moe_status check_shapes(int T, int d, int E, int d_ff, int k, int d_ffs)
{
    if (T < 1 || d < 1 || E < 1 || d_ff < 1 || k < 1 || d_ffs < 0) return MOE_ERR_INVALID_ARG;
    if (k > E) return MOE_ERR_INVALID_ARG;
    if (k > 8 || E > 256 || T > (1 << 24)) return MOE_ERR_UNSUPPORTED;
    if (d % 128 || d_ff % 128 || d_ffs % 128) return MOE_ERR_UNSUPPORTED;
    if (d > 16384 || d_ff > 65536 || d_ffs > 65536) return MOE_ERR_UNSUPPORTED;
    const long long S = static_cast<long long>(T) * k;
    const long long w = std::max({d, d_ff, d_ffs});
    if (S * w >= (1LL << 31)) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_ptr(const void *p) { return p != nullptr && aligned16(p); }

moe_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// ---------------------------------------------------------------- driver bits
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

void load_encode()
{
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}

PFN_cuMemGetAddressRange_v3020 g_range = nullptr;
std::once_flag g_range_once;

void load_range()
{
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_range = reinterpret_cast<PFN_cuMemGetAddressRange_v3020>(fn);
}

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];

}  // namespace

cudaError_t make_tmap_bf16(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                           uint32_t box_rows)
{
    std::call_once(g_encode_once, load_encode);
    if (g_encode == nullptr) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base),
                                dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_bf16_atoms(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                                 uint32_t box_rows, uint32_t atoms)
{
    std::call_once(g_encode_once, load_encode);
    if (g_encode == nullptr) return cudaErrorNotSupported;
    // (column within a 64-wide atom, row, atom): the atom index strides by
    // 128 bytes, so a box of `atoms` atoms lands as that many consecutive
    // [box_rows x 64] 128-byte-swizzled tiles.
    const cuuint64_t dims[3] = {64, rows, cols / 64};
    const cuuint64_t strides[2] = {cols * 2, 128};
    const cuuint32_t box[3] = {64, box_rows, atoms};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base),
                                dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_e4m3(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols)
{
    std::call_once(g_encode_once, load_encode);
    if (g_encode == nullptr) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols};
    const cuuint32_t box[2] = {128, 128};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base),
                                dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_f16(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                          uint32_t box_rows)
{
    std::call_once(g_encode_once, load_encode);
    if (g_encode == nullptr) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base),
                                dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_f16_atoms(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                                uint32_t box_rows, uint32_t atoms)
{
    std::call_once(g_encode_once, load_encode);
    if (g_encode == nullptr) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {64, rows, cols / 64};
    const cuuint64_t strides[2] = {cols * 2, 128};
    const cuuint32_t box[3] = {64, box_rows, atoms};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void *>(base),
                                dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int device_sm_count()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    int n = g_sm_count[dev].load(std::memory_order_relaxed);
    if (n > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
        n = 148;
    g_sm_count[dev].store(n, std::memory_order_relaxed);
    return n;
}

// ------------------------------------------------------- expert parallelism
// Receive rows per rank: every rank may send each of its T_max tokens to at
// most min(k, E/R) experts of one owner.
long long ep_recv_rows_ll(int T_max, int E, int k, int R)
{
    if (T_max < 1 || R < 1 || R > kMaxRanksHost || E < R || E % R != 0 || k < 1 || k > E) return 0;
    return static_cast<long long>(R) * T_max * std::min(k, E / R);
}

// Workspace of one rank: the dispatch's part (sized by the call's T), then
// the expert kernel's part, placed after the dispatch part of T_max so that
// it does not move with the T of a step.
struct EpLayout {
    size_t tilecnt, tilebase, rank, offsets, base, ok, disp_end;
    size_t ffnctr;      // expert kernel: work counter @0, readiness counters @kAlign
    size_t H, total;
};

EpLayout ep_layout(int T, int T_max, int E, int d_ff, int k, int R)
{
    EpLayout L{};
    auto dispatch_part = [&](int Tn, EpLayout &D) {
        size_t o = kHeaderBytes;
        auto take = [&](size_t bytes) {
            const size_t r = o;
            o += align_up(bytes);
            return r;
        };
        const size_t ntiles = (static_cast<size_t>(Tn) + 127) / 128;
        D.tilecnt = take(ntiles * E * 4);
        D.tilebase = take(ntiles * E * 4);
        D.rank = take(static_cast<size_t>(Tn) * k * 4);
        D.offsets = take((static_cast<size_t>(E) + 1) * 4);
        D.base = take(static_cast<size_t>(E) * 4);
        D.ok = take(4);
        D.disp_end = o;
    };
    EpLayout M{};
    dispatch_part(T_max, M);
    dispatch_part(T, L);
    const int rows = static_cast<int>(ep_recv_rows_ll(T_max, E, k, R));
    size_t o = M.disp_end;
    L.ffnctr = o;
    o += align_up(kAlign + ffn_ready_counters(rows, E / R, d_ff) * 4);
    L.H = o;
    o += align_up(static_cast<size_t>(rows) * d_ff * 2);
    L.total = o;
    return L;
}

// Shapes of one rank of an expert-parallel layer.
moe_status ep_check(int T, int d, int E, int d_ff, int k, int R)
{
    if (R < 1 || T < 1 || E < 1 || k < 1) return MOE_ERR_INVALID_ARG;
    if (R > kMaxRanksHost) return MOE_ERR_UNSUPPORTED;
    if (E % R != 0 || k > E) return MOE_ERR_INVALID_ARG;
    moe_status st = check_shapes(T, d, E, d_ff, k, 0);
    if (st != MOE_OK) return st;
    const long long rows = ep_recv_rows_ll(T, E, k, R);
    return check_shapes(static_cast<int>(std::min<long long>(rows, 1 << 30)), d, E / R, d_ff, 1, 0);
}

}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_size_ex(int T, int d, int E, int d_ff, int k, int d_ff_shared)
{
    if (check_shapes(T, d, E, d_ff, k, d_ff_shared) != MOE_OK) return 0;
    return forward_layout(T, d, E, d_ff, k, d_ff_shared).total;
}

size_t moe_workspace_size(int T, int d, int E, int d_ff, int k)
{
    return moe_workspace_size_ex(T, d, E, d_ff, k, 0);
}

const char *moe_status_string(moe_status s)
{
    switch (s) {
    case MOE_OK: return "MOE_OK: success";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: invalid argument (null or misaligned pointer, bad size, k > E)";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: sizes outside the supported range";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace smaller than moe_workspace_size()";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA call or kernel launch failed";
    case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE: the device error word is set";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT: a device-side bounded wait ran out";
    }
    return "unknown moe_status";
}

static moe_status route_impl(int T, int d, int E, int k, const moe_bf16 *x, const moe_bf16 *Wg,
                             const float *bias, int32_t *idx, float *w, int32_t *counts,
                             int32_t *offsets, uint8_t *ws, const Layout &L, cudaStream_t s,
                             bool slots = false, int wmode = 0, int cap = -1)
{
    RouteLaunch a{};
    a.wmode = wmode;
    a.cap = cap;
    a.T = T;
    a.d = d;
    a.E = E;
    a.k = k;
    a.x = x;
    a.Wg = Wg;
    a.bias = bias;
    a.idx = idx;
    a.w = w;
    a.counts = counts;
    a.offsets = offsets;
    a.tilecnt = reinterpret_cast<int32_t *>(ws + L.tilecnt);
    a.tilebase = reinterpret_cast<int32_t *>(ws + L.tilebase);
    a.rank = reinterpret_cast<int32_t *>(ws + L.rank);
    a.done = reinterpret_cast<uint32_t *>(ws + 4);
    a.tile_ctr = reinterpret_cast<uint32_t *>(ws + L.tilectr);
    a.err = reinterpret_cast<uint32_t *>(ws);
    if (slots) {
        a.slot_pos = reinterpret_cast<int32_t *>(ws + L.slotpos);
        a.perm = reinterpret_cast<int32_t *>(ws + L.perm);
        a.gcnt = reinterpret_cast<int32_t *>(ws + L.gcnt);
        a.perm_stride = perm_stride(T);
    }
    return from_cuda(launch_route(a, s));
}

moe_status moe_route_variant(int T, int d, int E, int k, const moe_bf16 *x, const moe_bf16 *Wg,
                             const float *router_bias, int weights, int32_t *idx, float *w,
                             int32_t *counts, void *ws, size_t ws_bytes, moe_stream_t stream);

moe_status moe_route(int T, int d, int E, int k, const moe_bf16 *x, const moe_bf16 *Wg,
                     const float *router_bias, int32_t *idx, float *w, int32_t *counts, void *ws,
                     size_t ws_bytes, moe_stream_t stream)
{
    return moe_route_variant(T, d, E, k, x, Wg, router_bias, MOE_WEIGHTS_SOFTMAX_TOPK, idx, w,
                             counts, ws, ws_bytes, stream);
}

moe_status moe_route_variant(int T, int d, int E, int k, const moe_bf16 *x, const moe_bf16 *Wg,
                             const float *router_bias, int weights, int32_t *idx, float *w,
                             int32_t *counts, void *ws, size_t ws_bytes, moe_stream_t stream)
{
    if (weights < 0 || weights > MOE_WEIGHTS_ENTROPY) return MOE_ERR_INVALID_ARG;
    if (weights == MOE_WEIGHTS_ENTROPY && k < 2) return MOE_ERR_INVALID_ARG;
    moe_status st = check_shapes(T, d, E, 128, k, 0);
    if (st != MOE_OK) return st;
    if (!ok_ptr(x) || !ok_ptr(Wg) || !ok_ptr(idx) || !ok_ptr(w) || !ok_ptr(ws))
        return MOE_ERR_INVALID_ARG;
    if (router_bias != nullptr && !aligned16(router_bias)) return MOE_ERR_INVALID_ARG;
    if (counts != nullptr && !aligned16(counts)) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe_workspace_size(T, d, E, 128, k)) return MOE_ERR_WORKSPACE;
    const Layout L = forward_layout(T, d, E, 128, k, 0);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    st = from_cuda(cudaMemsetAsync(wsb, 0, L.zero_bytes, s));
    if (st != MOE_OK) return st;
    return route_impl(T, d, E, k, x, Wg, router_bias, idx, w, counts,
                      reinterpret_cast<int32_t *>(wsb + L.offsets), wsb, L, s, false, weights);
}

moe_status moe_permute(int T, int d, int E, int k, const moe_bf16 *x, const int32_t *idx,
                       int32_t *offsets, int32_t *row_of_slot, moe_bf16 *x_perm, void *ws,
                       size_t ws_bytes, moe_stream_t stream)
{
    moe_status st = check_shapes(T, d, E, 128, k, 0);
    if (st != MOE_OK) return st;
    if (!ok_ptr(x) || !ok_ptr(idx) || !ok_ptr(offsets) || !ok_ptr(row_of_slot) ||
        !ok_ptr(x_perm) || !ok_ptr(ws))
        return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe_workspace_size(T, d, E, 128, k)) return MOE_ERR_WORKSPACE;
    const Layout L = forward_layout(T, d, E, 128, k, 0);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    st = from_cuda(cudaMemsetAsync(wsb, 0, kHeaderBytes, s));
    if (st != MOE_OK) return st;
    RanksLaunch r{};
    r.T = T;
    r.E = E;
    r.k = k;
    r.idx = idx;
    r.offsets = offsets;
    r.tilecnt = reinterpret_cast<int32_t *>(wsb + L.tilecnt);
    r.tilebase = reinterpret_cast<int32_t *>(wsb + L.tilebase);
    r.rank = reinterpret_cast<int32_t *>(wsb + L.rank);
    r.done = reinterpret_cast<uint32_t *>(wsb + 8);
    r.err = reinterpret_cast<uint32_t *>(wsb);
    st = from_cuda(launch_ranks(r, s));
    if (st != MOE_OK) return st;
    ScatterLaunch c{};
    c.cap = -1;
    c.T = T;
    c.d = d;
    c.E = E;
    c.k = k;
    c.x = x;
    c.idx = idx;
    c.rank = r.rank;
    c.tilebase = r.tilebase;
    c.x_perm = x_perm;
    c.row_of_slot = row_of_slot;
    c.err = r.err;
    c.pdl = true;
    return from_cuda(launch_scatter(c, s));
}

static moe_status mark(void *const *events, int i, cudaStream_t s);

static moe_status ffn_impl(int S, int d, int E, int d_ff, int max_rows, const moe_bf16 *x,
                           const int32_t *offsets, const moe_bf16 *W1, const moe_bf16 *W3,
                           const moe_bf16 *W2, moe_bf16 *H, float *y, uint32_t *h_ready,
                           uint32_t *sched, uint32_t *err, cudaStream_t s, bool pdl, int ksplit,
                           int act = 0, float *out = nullptr, const int32_t *slot_of_row = nullptr,
                           const float *gate_w = nullptr, int k = 1, bool y_bf16 = false)
{
    FfnLaunch f{};
    f.act = act;
    f.y_bf16 = y_bf16;
    f.out = out;
    f.slot_of_row = slot_of_row;
    f.gate_w = gate_w;
    f.k = k;
    f.E = E;
    f.d = d;
    f.d_ff = d_ff;
    f.S = S;
    f.max_rows = max_rows;
    f.ksplit = ksplit;
    f.offsets = offsets;
    f.W1 = W1;
    f.W3 = W3;
    f.W2 = W2;
    f.x = x;
    f.H = H;
    f.Y = y;
    f.h_ready = h_ready;
    f.sched = sched;
    f.err = err;
    f.pdl = pdl;
    return from_cuda(launch_ffn(f, s));
}

moe_status moe_expert_ffn(int S, int d, int E, int d_ff, const moe_bf16 *x_perm,
                          const int32_t *offsets, const moe_bf16 *W1, const moe_bf16 *W3,
                          const moe_bf16 *W2, float *y_perm, void *ws, size_t ws_bytes,
                          moe_stream_t stream)
{
    moe_status st = check_shapes(S, d, E, d_ff, 1, 0);
    if (st != MOE_OK) return st;
    if (!ok_ptr(x_perm) || !ok_ptr(offsets) || !ok_ptr(W1) || !ok_ptr(W3) || !ok_ptr(W2) ||
        !ok_ptr(y_perm) || !ok_ptr(ws))
        return MOE_ERR_INVALID_ARG;
    const size_t ctr = align_up(ffn_ready_counters(S, E, d_ff) * 4);
    const size_t need = kHeaderBytes + ctr + align_up(static_cast<size_t>(S) * d_ff * 2);
    if (ws_bytes < need) return MOE_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    st = from_cuda(cudaMemsetAsync(wsb, 0, kHeaderBytes + ctr, s));
    if (st != MOE_OK) return st;
    return ffn_impl(S, d, E, d_ff, S, x_perm, offsets, W1, W3, W2,
                    reinterpret_cast<moe_bf16 *>(wsb + kHeaderBytes + ctr), y_perm,
                    reinterpret_cast<uint32_t *>(wsb + kHeaderBytes),
                    reinterpret_cast<uint32_t *>(wsb + 16), reinterpret_cast<uint32_t *>(wsb), s,
                    false, 1);
}

moe_status moe_combine(int T, int d, int k, const float *y_perm, const int32_t *row_of_slot,
                       const float *w, const float *shared_y, float *out, moe_stream_t stream)
{
    if (T < 1 || d < 1 || k < 1) return MOE_ERR_INVALID_ARG;
    if (k > 8 || T > (1 << 24) || d % 128 || d > 16384) return MOE_ERR_UNSUPPORTED;
    if (!ok_ptr(y_perm) || !ok_ptr(row_of_slot) || !ok_ptr(w) || !ok_ptr(out))
        return MOE_ERR_INVALID_ARG;
    if (shared_y != nullptr && !aligned16(shared_y)) return MOE_ERR_INVALID_ARG;
    CombineLaunch c{};
    c.T = T;
    c.d = d;
    c.k = k;
    c.ksplit = 1;
    c.y = y_perm;
    c.row_of_slot = row_of_slot;
    c.w = w;
    c.shared_y = shared_y;
    c.out = out;
    c.pdl = false;
    return from_cuda(launch_combine(c, reinterpret_cast<cudaStream_t>(stream)));
}

// Records event i (if any) on the stream; inside stream capture as a graph
// event node.
static moe_status mark(void *const *events, int i, cudaStream_t s)
{
    if (events == nullptr || events[i] == nullptr) return MOE_OK;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return MOE_ERR_CUDA;
    cudaEvent_t ev = static_cast<cudaEvent_t>(events[i]);
    if (cs == cudaStreamCaptureStatusActive)
        return from_cuda(cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal));
    return from_cuda(cudaEventRecord(ev, s));
}

// A second stream per device for the shared expert, created on first use
// (non-blocking, so it never orders against the legacy default stream).  A
// call forks onto it with an event recorded on the caller's stream and joins
// back with another, so the work stays ordered with the caller's stream and
// the call can still be captured into a CUDA graph.
std::mutex g_side_mu;
cudaStream_t g_side[64];

cudaStream_t side_stream()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(g_side_mu);
    if (g_side[dev] == nullptr) {
        cudaStream_t st = nullptr;
        if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
        g_side[dev] = st;
    }
    return g_side[dev];
}

// The shared expert's rows come from the CTA-pair kernel (complete sums, so
// bf16 like the routed ones) whenever its single segment is large enough.
static bool ys_bf16_for(int T) { return ffn_pair_eligible(T, 1, 1); }

static moe_status shared_impl(int T, int d, int d_ffs, const moe_bf16 *x, const moe_bf16 *Ws1,
                              const moe_bf16 *Ws3, const moe_bf16 *Ws2, uint8_t *wsb,
                              const Layout &L, uint32_t *err, cudaStream_t s, int act, bool ys_bf16)
{
    return ffn_impl(T, d, 1, d_ffs, T, x, nullptr, Ws1, Ws3, Ws2,
                    reinterpret_cast<moe_bf16 *>(wsb + L.Hs), reinterpret_cast<float *>(wsb + L.Ys),
                    reinterpret_cast<uint32_t *>(wsb + L.hready_s),
                    reinterpret_cast<uint32_t *>(wsb + 20), err, s, false, 1, act, nullptr, nullptr,
                    nullptr, 1, ys_bf16);
}

static moe_status forward_impl(int T, int d, int E, int d_ff, int k, const moe_bf16 *x,
                               const moe_bf16 *Wg, const float *router_bias, const moe_bf16 *W1,
                               const moe_bf16 *W3, const moe_bf16 *W2, int d_ff_shared,
                               const moe_bf16 *Ws1, const moe_bf16 *Ws3, const moe_bf16 *Ws2,
                               float *out, void *ws, size_t ws_bytes, moe_stream_t stream,
                               void *const *events, const moe_variant *variant = nullptr)
{
    moe_status st = check_shapes(T, d, E, d_ff, k, d_ff_shared);
    if (st != MOE_OK) return st;
    const int wmode = variant ? variant->weights : MOE_WEIGHTS_SOFTMAX_TOPK;
    const int act = variant ? variant->activation : MOE_ACT_SILU;
    const double cf = variant ? variant->capacity_factor : 0.0;
    if (wmode < 0 || wmode > MOE_WEIGHTS_ENTROPY || act < 0 || act > 1 || !(cf >= 0.0) ||
        cf > 1e9)
        return MOE_ERR_INVALID_ARG;
    if (wmode == MOE_WEIGHTS_ENTROPY && k < 2) return MOE_ERR_INVALID_ARG;
    if (wmode == MOE_WEIGHTS_ENTROPY && cf > 0.0) return MOE_ERR_UNSUPPORTED;
    // Per-expert capacity floor(cf * T * k / E); no expert ever receives more
    // than T pairs, so a capacity of T or more drops nothing.
    int cap = -1;
    if (cf > 0.0) {
        const double c = std::floor(cf * static_cast<double>(static_cast<long long>(T) * k) /
                                    static_cast<double>(E));
        if (c < static_cast<double>(T)) cap = static_cast<int>(c);
    }
    if (!ok_ptr(x) || !ok_ptr(Wg) || !ok_ptr(W1) || !ok_ptr(W3) || !ok_ptr(W2) || !ok_ptr(out) ||
        !ok_ptr(ws))
        return MOE_ERR_INVALID_ARG;
    if (router_bias != nullptr && !aligned16(router_bias)) return MOE_ERR_INVALID_ARG;
    if (d_ff_shared > 0 && (!ok_ptr(Ws1) || !ok_ptr(Ws3) || !ok_ptr(Ws2)))
        return MOE_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(ws) % kAlign) return MOE_ERR_INVALID_ARG;
    const Layout L = forward_layout(T, d, E, d_ff, k, d_ff_shared);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    uint32_t *err = reinterpret_cast<uint32_t *>(wsb);
    const int S = T * k;
    int32_t *idx = reinterpret_cast<int32_t *>(wsb + L.idx);
    float *w = reinterpret_cast<float *>(wsb + L.w);
    int32_t *offsets = reinterpret_cast<int32_t *>(wsb + L.offsets);
    int32_t *row = reinterpret_cast<int32_t *>(wsb + L.row);
    moe_bf16 *xperm = reinterpret_cast<moe_bf16 *>(wsb + L.xperm);
    moe_bf16 *H = reinterpret_cast<moe_bf16 *>(wsb + L.H);
    float *Y = reinterpret_cast<float *>(wsb + L.Y);

    st = from_cuda(cudaMemsetAsync(wsb, 0, L.zero_bytes, s));
    if (st != MOE_OK) return st;
    // Narrow layers run the slot mode: the router hands every expert its
    // token list and its total, and the expert kernel derives the segment
    // starts and gathers the rows of x itself, so there is no permuted copy
    // of x and no scatter launch in between.
    // Dropping by capacity needs the token order of each expert's pairs,
    // which only the token-ordered dispatch (ranks, scatter) keeps.
    const bool narrow = ffn_small_supported(d) && cap < 0;
    // Overlapping launches pay off for small layers; for large ones they only
    // take SM slots early (measured: neutral to slightly negative).
    const bool pdl = events == nullptr && S <= 4096;
    // A token never picks one expert twice, so no segment exceeds T rows.
    // (The capacity path of a narrow layer runs the general expert kernel on
    // the permuted copy, without a K split.)
    const int ksplit = (cap >= 0 && ffn_small_supported(d)) ? 1 : ffn_splits(S, E, d, d_ff);
    // With k <= 2, no shared expert and the CTA-pair expert kernel (which
    // never splits K), the down units write the gate-weighted sum into out
    // themselves: at most two terms reach each element, and two terms added
    // onto zero give one result in either order.  No Y round trip and no
    // combine launch then.
    const bool pair = !narrow && ffn_pair_eligible(S, E, ksplit);
    const bool fused_out = pair && k <= 2 && d_ff_shared == 0;
    // The CTA-pair kernel's rows are complete sums (it never splits K); they
    // go to the combine as bf16, which halves the bytes of the per-slot
    // round trip (each row rounded once, as H is).  K-split partials stay
    // fp32.
    const bool y_bf16 = pair && !fused_out;
    const bool ys_bf16 = d_ff_shared > 0 && ys_bf16_for(T);
    int32_t *slotrow = reinterpret_cast<int32_t *>(wsb + L.slotrow);
    if ((st = mark(events, 0, s)) != MOE_OK) return st;
    st = route_impl(T, d, E, k, x, Wg, router_bias, idx, w,
                    reinterpret_cast<int32_t *>(wsb + L.counts), offsets, wsb, L, s, narrow, wmode,
                    cap);
    if (st != MOE_OK) return st;

    // The shared expert needs neither the routing nor the dispatch: with a
    // side stream it runs next to the scatter (which takes no shared memory,
    // so its blocks fit beside the expert kernel's) and the routed experts.
    // The traced form keeps it in line, between its events.
    const float *shared_y = nullptr;
    cudaStream_t s2 = nullptr;
    // Joins the side stream back into the caller's stream when the call
    // leaves this scope, on an early error return too.
    struct Join {
        cudaStream_t s;
        cudaEvent_t ev = nullptr;
        moe_status now()
        {
            if (ev == nullptr) return MOE_OK;
            const cudaError_t e = cudaStreamWaitEvent(s, ev, 0);
            cudaEventDestroy(ev);
            ev = nullptr;
            return from_cuda(e);
        }
        ~Join() { now(); }
    } join{s};
    if (d_ff_shared > 0 && events == nullptr && (s2 = side_stream()) != nullptr) {
        cudaEvent_t ev_fork = nullptr;
        if ((st = from_cuda(cudaEventCreateWithFlags(&ev_fork, cudaEventDisableTiming))) != MOE_OK)
            return st;
        st = from_cuda(cudaEventRecord(ev_fork, s));
        if (st == MOE_OK) st = from_cuda(cudaStreamWaitEvent(s2, ev_fork, 0));
        cudaEventDestroy(ev_fork);
        if (st != MOE_OK) return st;
        st = shared_impl(T, d, d_ff_shared, x, Ws1, Ws3, Ws2, wsb, L, err, s2, act, ys_bf16_for(T));
        cudaEvent_t ev = nullptr;
        if (st == MOE_OK) st = from_cuda(cudaEventCreateWithFlags(&ev, cudaEventDisableTiming));
        if (st == MOE_OK) {
            st = from_cuda(cudaEventRecord(ev, s2));
            if (st == MOE_OK) join.ev = ev;
            else cudaEventDestroy(ev);
        }
        if (st != MOE_OK) return st;
        shared_y = reinterpret_cast<const float *>(wsb + L.Ys);
    }

    if ((st = mark(events, 1, s)) != MOE_OK) return st;
    if (!narrow) {
        ScatterLaunch c{};
        c.cap = cap;
        c.offsets = offsets;
        c.T = T;
        c.d = d;
        c.E = E;
        c.k = k;
        c.x = x;
        c.idx = idx;
        c.rank = reinterpret_cast<int32_t *>(wsb + L.rank);
        c.tilebase = reinterpret_cast<int32_t *>(wsb + L.tilebase);
        c.x_perm = xperm;
        c.row_of_slot = row;
        c.slot_of_row = fused_out ? slotrow : nullptr;
        c.out_zero = fused_out ? out : nullptr;
        c.allow_empty = wmode == MOE_WEIGHTS_ENTROPY;
        c.err = err;
        c.pdl = pdl;
        st = from_cuda(launch_scatter(c, s));
        if (st != MOE_OK) return st;
    }

    if ((st = mark(events, 2, s)) != MOE_OK) return st;
    if (narrow) {
        FfnLaunch f{};
        f.act = act;
        f.E = E;
        f.d = d;
        f.d_ff = d_ff;
        f.S = S;
        f.max_rows = T;
        f.ksplit = ksplit;
        f.offsets = offsets;
        f.W1 = W1;
        f.W3 = W3;
        f.W2 = W2;
        f.x = x;
        f.H = nullptr;
        f.Y = Y;
        f.h_ready = nullptr;
        f.err = err;
        f.pdl = pdl;
        f.perm = reinterpret_cast<const int32_t *>(wsb + L.perm);
        f.perm_stride = perm_stride(T);
        f.x_rows = T;
        f.counts = reinterpret_cast<const int32_t *>(wsb + L.gcnt);
        f.offsets_out = offsets;
        st = from_cuda(launch_ffn_small(f, ksplit, reinterpret_cast<int *>(wsb + 12), s));
    } else {
        st = ffn_impl(S, d, E, d_ff, T, xperm, offsets, W1, W3, W2, H, Y,
                      reinterpret_cast<uint32_t *>(wsb + L.hready),
                      reinterpret_cast<uint32_t *>(wsb + 16), err, s, pdl, ksplit, act,
                      fused_out ? out : nullptr, slotrow, w, k, y_bf16);
    }
    if (st != MOE_OK) return st;

    if ((st = mark(events, 3, s)) != MOE_OK) return st;
    if (d_ff_shared > 0 && s2 == nullptr) {
        st = shared_impl(T, d, d_ff_shared, x, Ws1, Ws3, Ws2, wsb, L, err, s, act, ys_bf16);
        if (st != MOE_OK) return st;
        shared_y = reinterpret_cast<const float *>(wsb + L.Ys);
    }
    if ((st = join.now()) != MOE_OK) return st;
    if ((st = mark(events, 4, s)) != MOE_OK) return st;
    if (fused_out) return mark(events, 5, s);

    CombineLaunch cb{};
    cb.T = T;
    cb.d = d;
    cb.k = k;
    cb.ksplit = ksplit;
    cb.ksplit_dev = narrow ? reinterpret_cast<const int *>(wsb + 12) : nullptr;
    cb.y = Y;
    if (narrow) {
        cb.idx = idx;
        cb.slot_pos = reinterpret_cast<const int32_t *>(wsb + L.slotpos);
        cb.offsets = offsets;
    } else {
        cb.row_of_slot = row;
    }
    cb.w = w;
    cb.shared_y = shared_y;
    cb.out = out;
    cb.y_bf16 = y_bf16;
    cb.shared_bf16 = ys_bf16;
    cb.pdl = false;  // after a persistent kernel an early launch only takes SM slots
    st = from_cuda(launch_combine(cb, s));
    if (st != MOE_OK) return st;
    return mark(events, 5, s);
}

moe_status moe_forward_ex(int T, int d, int E, int d_ff, int k, const moe_bf16 *x,
                          const moe_bf16 *Wg, const float *router_bias, const moe_bf16 *W1,
                          const moe_bf16 *W3, const moe_bf16 *W2, int d_ff_shared,
                          const moe_bf16 *Ws1, const moe_bf16 *Ws3, const moe_bf16 *Ws2,
                          float *out, void *ws, size_t ws_bytes, moe_stream_t stream)
{
    return forward_impl(T, d, E, d_ff, k, x, Wg, router_bias, W1, W3, W2, d_ff_shared, Ws1, Ws3,
                        Ws2, out, ws, ws_bytes, stream, nullptr);
}

moe_status moe_forward_variant(int T, int d, int E, int d_ff, int k, const moe_bf16 *x,
                               const moe_bf16 *Wg, const float *router_bias, const moe_bf16 *W1,
                               const moe_bf16 *W3, const moe_bf16 *W2, int d_ff_shared,
                               const moe_bf16 *Ws1, const moe_bf16 *Ws3, const moe_bf16 *Ws2,
                               const moe_variant *variant, float *out, void *ws, size_t ws_bytes,
                               moe_stream_t stream)
{
    return forward_impl(T, d, E, d_ff, k, x, Wg, router_bias, W1, W3, W2, d_ff_shared, Ws1, Ws3,
                        Ws2, out, ws, ws_bytes, stream, nullptr, variant);
}

static moe_status fp8_impl(int T, int d, int E, int d_ff, int k, const moe_bf16 *x,
                           const moe_bf16 *Wg, const float *router_bias, const uint8_t *W1q,
                           const float *s1, const uint8_t *W3q, const float *s3,
                           const uint8_t *W2q, const float *s2, float *out, void *ws,
                           size_t ws_bytes, moe_stream_t stream, void *const *events)
{
    moe_status st = check_shapes(T, d, E, d_ff, k, 0);
    if (st != MOE_OK) return st;
    if (!ok_ptr(x) || !ok_ptr(Wg) || !ok_ptr(W1q) || !ok_ptr(W3q) || !ok_ptr(W2q) ||
        !ok_ptr(s1) || !ok_ptr(s3) || !ok_ptr(s2) || !ok_ptr(out) || !ok_ptr(ws))
        return MOE_ERR_INVALID_ARG;
    if (router_bias != nullptr && !aligned16(router_bias)) return MOE_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(ws) % kAlign) return MOE_ERR_INVALID_ARG;
    const Layout L = forward_layout(T, d, E, d_ff, k, 0);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    uint32_t *err = reinterpret_cast<uint32_t *>(wsb);
    const int S = T * k;
    int32_t *idx = reinterpret_cast<int32_t *>(wsb + L.idx);
    float *w = reinterpret_cast<float *>(wsb + L.w);
    int32_t *offsets = reinterpret_cast<int32_t *>(wsb + L.offsets);
    int32_t *row = reinterpret_cast<int32_t *>(wsb + L.row);
    float *Y = reinterpret_cast<float *>(wsb + L.Y);
    st = from_cuda(cudaMemsetAsync(wsb, 0, L.zero_bytes, s));
    if (st != MOE_OK) return st;
    const bool pdl = events == nullptr && S <= 4096;
    // Router in bf16 (unchanged), token-ordered dispatch with the rows
    // converted to fp16, the FP8 expert kernel, the combine.
    if ((st = mark(events, 0, s)) != MOE_OK) return st;
    st = route_impl(T, d, E, k, x, Wg, router_bias, idx, w,
                    reinterpret_cast<int32_t *>(wsb + L.counts), offsets, wsb, L, s);
    if (st != MOE_OK) return st;
    if ((st = mark(events, 1, s)) != MOE_OK) return st;
    ScatterLaunch c{};
    c.cap = -1;
    c.T = T;
    c.d = d;
    c.E = E;
    c.k = k;
    c.x = x;
    c.idx = idx;
    c.rank = reinterpret_cast<int32_t *>(wsb + L.rank);
    c.tilebase = reinterpret_cast<int32_t *>(wsb + L.tilebase);
    c.x_perm = reinterpret_cast<uint16_t *>(wsb + L.xperm);
    c.row_of_slot = row;
    c.err = err;
    c.pdl = pdl;
    c.to_f16 = true;
    st = from_cuda(launch_scatter(c, s));
    if (st != MOE_OK) return st;
    // The workspace holds ffn_splits(...) partial outputs per row.
    const int ksplit = std::min(down_ksplit(S, E, d, d_ff), ffn_splits(S, E, d, d_ff));
    FfnFp8Launch f{};
    f.f.E = E;
    f.f.d = d;
    f.f.d_ff = d_ff;
    f.f.S = S;
    f.f.max_rows = T;
    f.f.ksplit = ksplit;
    f.f.offsets = offsets;
    f.f.x = reinterpret_cast<const uint16_t *>(wsb + L.xperm);
    f.f.H = reinterpret_cast<uint16_t *>(wsb + L.H);
    f.f.Y = Y;
    f.f.h_ready = reinterpret_cast<uint32_t *>(wsb + L.hready);
    f.f.err = err;
    f.f.pdl = pdl;
    f.q1 = W1q;
    f.q3 = W3q;
    f.q2 = W2q;
    f.s1 = s1;
    f.s3 = s3;
    f.s2 = s2;
    if ((st = mark(events, 2, s)) != MOE_OK) return st;
    st = from_cuda(launch_ffn_fp8(f, s));
    if (st != MOE_OK) return st;
    if ((st = mark(events, 3, s)) != MOE_OK) return st;
    if ((st = mark(events, 4, s)) != MOE_OK) return st;
    CombineLaunch cb{};
    cb.T = T;
    cb.d = d;
    cb.k = k;
    cb.ksplit = ksplit;
    cb.y = Y;
    cb.row_of_slot = row;
    cb.w = w;
    cb.out = out;
    cb.pdl = false;
    st = from_cuda(launch_combine(cb, s));
    if (st != MOE_OK) return st;
    return mark(events, 5, s);
}

moe_status moe_forward_fp8(int T, int d, int E, int d_ff, int k, const moe_bf16 *x,
                           const moe_bf16 *Wg, const float *router_bias, const uint8_t *W1q,
                           const float *s1, const uint8_t *W3q, const float *s3,
                           const uint8_t *W2q, const float *s2, float *out, void *ws,
                           size_t ws_bytes, moe_stream_t stream)
{
    return fp8_impl(T, d, E, d_ff, k, x, Wg, router_bias, W1q, s1, W3q, s3, W2q, s2, out, ws,
                    ws_bytes, stream, nullptr);
}

moe_status moe_forward_fp8_traced(int T, int d, int E, int d_ff, int k, const moe_bf16 *x,
                                  const moe_bf16 *Wg, const float *router_bias,
                                  const uint8_t *W1q, const float *s1, const uint8_t *W3q,
                                  const float *s3, const uint8_t *W2q, const float *s2,
                                  float *out, void *ws, size_t ws_bytes, moe_stream_t stream,
                                  void *const *events, int n_events)
{
    if (events == nullptr || n_events != MOE_TRACE_EVENTS) return MOE_ERR_INVALID_ARG;
    return fp8_impl(T, d, E, d_ff, k, x, Wg, router_bias, W1q, s1, W3q, s3, W2q, s2, out, ws,
                    ws_bytes, stream, events);
}

moe_status moe_forward_traced(int T, int d, int E, int d_ff, int k, const moe_bf16 *x,
                              const moe_bf16 *Wg, const float *router_bias, const moe_bf16 *W1,
                              const moe_bf16 *W3, const moe_bf16 *W2, int d_ff_shared,
                              const moe_bf16 *Ws1, const moe_bf16 *Ws3, const moe_bf16 *Ws2,
                              float *out, void *ws, size_t ws_bytes, moe_stream_t stream,
                              void *const *events, int n_events)
{
    if (events == nullptr || n_events != MOE_TRACE_EVENTS) return MOE_ERR_INVALID_ARG;
    return forward_impl(T, d, E, d_ff, k, x, Wg, router_bias, W1, W3, W2, d_ff_shared, Ws1, Ws3,
                        Ws2, out, ws, ws_bytes, stream, events);
}

moe_status moe_forward(int T, int d, int E, int d_ff, int k, const moe_bf16 *x,
                       const moe_bf16 *Wg, const moe_bf16 *W1, const moe_bf16 *W3,
                       const moe_bf16 *W2, float *out, void *ws, size_t ws_bytes,
                       moe_stream_t stream)
{
    return moe_forward_ex(T, d, E, d_ff, k, x, Wg, nullptr, W1, W3, W2, 0, nullptr, nullptr,
                          nullptr, out, ws, ws_bytes, stream);
}

moe_status moe_selftest_wait_timeout(void *ws, size_t ws_bytes, moe_stream_t stream)
{
    if (!ok_ptr(ws) || ws_bytes < kHeaderBytes) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    moe_status st = from_cuda(cudaMemsetAsync(ws, 0, kHeaderBytes, s));
    if (st != MOE_OK) return st;
    return from_cuda(launch_wait_timeout(static_cast<uint32_t *>(ws), s));
}

moe_status moe_get_device_error(const void *ws, uint32_t *code, moe_stream_t stream)
{
    if (ws == nullptr) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    uint32_t word = 0;
    if (cudaMemcpy(&word, ws, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (code) *code = word;
    if (word == 0) return MOE_OK;
    if (word & (MOE_DEVERR_TIMEOUT_TMA | MOE_DEVERR_TIMEOUT_MMA | MOE_DEVERR_TIMEOUT_EPI))
        return MOE_ERR_TIMEOUT;
    return MOE_ERR_DEVICE;
}


// ------------------------------------------------------- expert parallelism

int moe_ep_recv_rows(int T_max, int E, int k, int R)
{
    const long long rows = ep_recv_rows_ll(T_max, E, k, R);
    return rows > (1LL << 30) ? 0 : static_cast<int>(rows);
}

size_t moe_ep_workspace_size(int T_max, int d, int E, int d_ff, int k, int R)
{
    if (ep_check(T_max, d, E, d_ff, k, R) != MOE_OK) return 0;
    return ep_layout(T_max, T_max, E, d_ff, k, R).total;
}

int moe_ep_ffn_splits(int rows_hint, int d, int E_local, int d_ff)
{
    if (rows_hint < 1 || E_local < 1 || d < 128 || d_ff < 128) return 0;
    return down_ksplit(rows_hint, E_local, d, d_ff);
}

int moe_ep_output_bf16(int rows_hint, int d, int E_local, int d_ff)
{
    // The CTA-pair kernel writes complete rows (it never splits K), so they
    // can be bf16; the split-K kernel writes fp32 partials.
    const int ks = moe_ep_ffn_splits(rows_hint, d, E_local, d_ff);
    return ks == 1 && ffn_pair_eligible(rows_hint, E_local, 1) ? 1 : 0;
}

moe_status moe_ep_dispatch(int T, int d, int E, int k, int R, int rank, const moe_bf16 *x,
                           const int32_t *idx, const int32_t *counts_all,
                           moe_bf16 *const *recv_x, int recv_rows, int32_t *pos_of_slot,
                           int32_t *recv_offsets, void *ws, size_t ws_bytes, moe_stream_t stream)
{
    // A rank may have no tokens in a step: it sends nothing but still owns
    // experts, so its plan (its receive segments) is computed all the same.
    if (T < 0) return MOE_ERR_INVALID_ARG;
    const int Tl = T > 0 ? T : 1;  // sizes of the checks and of the workspace layout
    moe_status st = ep_check(Tl, d, E, 128, k, R);
    if (st != MOE_OK) return st;
    if (rank < 0 || rank >= R || recv_rows < 1 || recv_x == nullptr) return MOE_ERR_INVALID_ARG;
    if ((T > 0 && (!ok_ptr(x) || !ok_ptr(idx) || !ok_ptr(pos_of_slot))) || !ok_ptr(counts_all) ||
        !ok_ptr(recv_offsets) || !ok_ptr(ws))
        return MOE_ERR_INVALID_ARG;
    for (int r = 0; r < R; ++r)
        if (!ok_ptr(recv_x[r])) return MOE_ERR_INVALID_ARG;
    const EpLayout L = ep_layout(Tl, Tl, E, 128, k, R);
    if (ws_bytes < L.disp_end) return MOE_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    st = from_cuda(cudaMemsetAsync(wsb, 0, kHeaderBytes, s));
    if (st != MOE_OK) return st;
    EpDispatchLaunch a{};
    a.T = T;
    a.d = d;
    a.E = E;
    a.k = k;
    a.R = R;
    a.rank = rank;
    a.recv_rows = recv_rows;
    a.x = x;
    a.idx = idx;
    a.counts_all = counts_all;
    a.offsets = reinterpret_cast<int32_t *>(wsb + L.offsets);
    a.tilecnt = reinterpret_cast<int32_t *>(wsb + L.tilecnt);
    a.tilebase = reinterpret_cast<int32_t *>(wsb + L.tilebase);
    a.rank_of_pair = reinterpret_cast<int32_t *>(wsb + L.rank);
    a.done = reinterpret_cast<uint32_t *>(wsb + 8);
    a.base = reinterpret_cast<int32_t *>(wsb + L.base);
    a.ok = reinterpret_cast<uint32_t *>(wsb + L.ok);
    a.recv_x = recv_x;
    a.pos_of_slot = pos_of_slot;
    a.recv_offsets = recv_offsets;
    a.err = reinterpret_cast<uint32_t *>(wsb);
    return from_cuda(launch_ep_dispatch(a, s));
}

moe_status moe_ep_expert_ffn(int T_max, int d, int E, int d_ff, int k, int R, int rows_hint,
                             int ksplit, int y_bf16, const moe_bf16 *recv_x,
                             const int32_t *recv_offsets, const moe_bf16 *W1, const moe_bf16 *W3,
                             const moe_bf16 *W2, void *recv_y, void *ws, size_t ws_bytes,
                             moe_stream_t stream)
{
    moe_status st = ep_check(T_max, d, E, d_ff, k, R);
    if (st != MOE_OK) return st;
    const int E_local = E / R;
    const int recv_rows = moe_ep_recv_rows(T_max, E, k, R);
    if (recv_rows < 1 || rows_hint < 1) return MOE_ERR_INVALID_ARG;
    if (ksplit != moe_ep_ffn_splits(rows_hint, d, E_local, d_ff)) return MOE_ERR_INVALID_ARG;
    if (y_bf16 != 0 && (y_bf16 != 1 || !moe_ep_output_bf16(rows_hint, d, E_local, d_ff)))
        return MOE_ERR_INVALID_ARG;
    if (!ok_ptr(recv_x) || !ok_ptr(recv_offsets) || !ok_ptr(W1) || !ok_ptr(W3) || !ok_ptr(W2) ||
        !ok_ptr(recv_y) || !ok_ptr(ws))
        return MOE_ERR_INVALID_ARG;
    const EpLayout L = ep_layout(T_max, T_max, E, d_ff, k, R);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    // Counters only: the error word keeps what the dispatch of this step found.
    const size_t ctr = kAlign + ffn_ready_counters(recv_rows, E_local, d_ff) * 4;
    st = from_cuda(cudaMemsetAsync(wsb + L.ffnctr, 0, ctr, s));
    if (st != MOE_OK) return st;
    FfnLaunch f{};
    f.E = E_local;
    f.d = d;
    f.d_ff = d_ff;
    f.S = recv_rows;
    f.S_hint = rows_hint;
    f.max_rows = std::min(recv_rows, R * T_max);
    f.ksplit = ksplit;
    f.offsets = recv_offsets;
    f.W1 = W1;
    f.W3 = W3;
    f.W2 = W2;
    f.x = recv_x;
    f.H = reinterpret_cast<moe_bf16 *>(wsb + L.H);
    f.Y = static_cast<float *>(recv_y);
    f.y_bf16 = y_bf16 != 0;
    f.h_ready = reinterpret_cast<uint32_t *>(wsb + L.ffnctr + kAlign);
    f.sched = reinterpret_cast<uint32_t *>(wsb + L.ffnctr);
    f.err = reinterpret_cast<uint32_t *>(wsb);
    f.pdl = false;
    f.k = 1;
    return from_cuda(launch_ffn(f, s));
}

moe_status moe_ep_combine(int T, int d, int E, int k, int R, int recv_rows, int ksplit,
                          int y_bf16, const int32_t *idx, const int32_t *pos_of_slot,
                          const float *w, const void *const *recv_y, const float *shared_y,
                          float *out, moe_stream_t stream)
{
    if (T == 0 && d >= 1 && E >= 1 && k >= 1 && R >= 1) return MOE_OK;  // no tokens, no rows
    if (T < 1 || d < 1 || E < 1 || k < 1 || R < 1 || recv_rows < 1 || ksplit < 1)
        return MOE_ERR_INVALID_ARG;
    if (y_bf16 != 0 && (y_bf16 != 1 || ksplit != 1)) return MOE_ERR_INVALID_ARG;
    if (R > kMaxRanksHost || k > 8 || T > (1 << 24) || d % 128 || d > 16384 || E > 256 ||
        ksplit > 8)
        return MOE_ERR_UNSUPPORTED;
    if (E % R != 0 || k > E || recv_y == nullptr) return MOE_ERR_INVALID_ARG;
    if (!ok_ptr(idx) || !ok_ptr(pos_of_slot) || !ok_ptr(w) || !ok_ptr(out))
        return MOE_ERR_INVALID_ARG;
    if (shared_y != nullptr && !aligned16(shared_y)) return MOE_ERR_INVALID_ARG;
    for (int r = 0; r < R; ++r)
        if (!ok_ptr(recv_y[r])) return MOE_ERR_INVALID_ARG;
    EpCombineLaunch c{};
    c.T = T;
    c.d = d;
    c.E = E;
    c.k = k;
    c.R = R;
    c.recv_rows = recv_rows;
    c.ksplit = ksplit;
    c.idx = idx;
    c.pos_of_slot = pos_of_slot;
    c.w = w;
    c.recv_y = recv_y;
    c.y_bf16 = y_bf16 != 0;
    c.shared_y = shared_y;
    c.out = out;
    return from_cuda(launch_ep_combine(c, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_ipc_get_handle(const void *dev_ptr, void *handle, size_t *offset)
{
    if (dev_ptr == nullptr || handle == nullptr || offset == nullptr) return MOE_ERR_INVALID_ARG;
    std::call_once(g_range_once, load_range);
    if (g_range == nullptr) return MOE_ERR_CUDA;
    CUdeviceptr base = 0;
    size_t bytes = 0;
    if (g_range(&base, &bytes, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS)
        return MOE_ERR_INVALID_ARG;
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, reinterpret_cast<void *>(base)) != cudaSuccess) return MOE_ERR_CUDA;
    static_assert(sizeof(h) == MOE_IPC_HANDLE_BYTES, "IPC handle size");
    std::memcpy(handle, &h, sizeof(h));
    *offset = static_cast<size_t>(reinterpret_cast<uintptr_t>(dev_ptr) - base);
    return MOE_OK;
}

moe_status moe_ipc_open_handle(const void *handle, void **base)
{
    if (handle == nullptr || base == nullptr) return MOE_ERR_INVALID_ARG;
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle, sizeof(h));
    if (cudaIpcOpenMemHandle(base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

moe_status moe_ipc_close(void *base)
{
    if (base == nullptr) return MOE_ERR_INVALID_ARG;
    return from_cuda(cudaIpcCloseMemHandle(base));
}

}  // extern "C"
