// noalloc.cu -- moe_expert_ffn_static: the expert FFN (both grouped GEMMs)
// with its scratch in a fixed device array owned by the library, for callers
// that cannot allocate device memory.
//
// Who needs it: code that runs where no allocator may be called -- a plugin
// or kernel-library hook that a host program calls with only its tensors
// (the host program owns every device allocation and gives out none), or a
// latency-critical loop that must not enter the driver's allocator between
// set-up and teardown.  Such a caller still owns the inputs and outputs; the
// only memory it cannot provide is the intermediate H = silu(W1 x) * (W3 x).
//
// The scratch is a file-scope __device__ array, so every GPU that loads the
// library holds kStaticScratchBytes of it until the process exits.  In host
// code the array's name is only a host-side stand-in: its device address is
// looked up with cudaGetSymbolAddress (with the device current) on the first
// call made on that device, and that address is what the kernels receive.
// The lookup is repeated when the device's context has changed since (after
// a cudaDeviceReset the array lives at a new address).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

#include "internal.h"
#include "moe.h"

namespace moe {

namespace {

constexpr size_t kStaticScratchBytes = MOE_STATIC_SCRATCH_BYTES;  // 32 MiB
constexpr size_t kStaticHeaderBytes = 256;                // device error word, then H
constexpr int kStaticMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_static_mutex;
void *g_static_ptr[kStaticMaxDevices] = {};
unsigned long long g_static_ctx[kStaticMaxDevices] = {};

PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;
std::once_flag g_ctx_once;

void load_ctx_fns()
{
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
}

// Unique id of the context current on this thread, or 0 if there is none
// (yet) or it cannot be asked for.
unsigned long long current_ctx_id()
{
    std::call_once(g_ctx_once, load_ctx_fns);
    if (g_ctx_current == nullptr || g_ctx_id == nullptr) return 0;
    CUcontext ctx = nullptr;
    if (g_ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    unsigned long long id = 0;
    if (g_ctx_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of g_static_scratch on device `dev` (the current device).
// Returns nullptr if the lookup failed.
void *static_scratch_address(int dev)
{
    std::lock_guard<std::mutex> lock(g_static_mutex);
    const unsigned long long id = current_ctx_id();
    if (g_static_ptr[dev] == nullptr || id == 0 || id != g_static_ctx[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) return nullptr;
        g_static_ptr[dev] = p;
        g_static_ctx[dev] = current_ctx_id();
    }
    return g_static_ptr[dev];
}

// Bytes of the fixed scratch a call of these sizes needs: the header (error
// word), the readiness counters of the expert kernel and H [S, d_ff] bf16.
size_t static_need(int S, int E, int d_ff)
{
    const size_t ctr_bytes = (ffn_ready_counters(S, E, d_ff) * 4 + 255) / 256 * 256;
    return kStaticHeaderBytes + ctr_bytes + static_cast<size_t>(S) * d_ff * 2;
}

}  // namespace

}  // namespace moe

using namespace moe;

extern "C" moe_status moe_expert_ffn_static(int S, int d, int E, int d_ff,
                                            const moe_bf16 *x_perm, const int32_t *offsets,
                                            const moe_bf16 *W1, const moe_bf16 *W3,
                                            const moe_bf16 *W2, float *y_perm,
                                            moe_stream_t stream)
{
    if (S < 1 || d < 1 || E < 1 || d_ff < 1) return MOE_ERR_INVALID_ARG;
    if (E > 256 || S > (1 << 24) || d % 128 || d_ff % 128 || d > 16384 || d_ff > 65536)
        return MOE_ERR_UNSUPPORTED;
    const long long wmax = d > d_ff ? d : d_ff;
    if (static_cast<long long>(S) * wmax >= (1LL << 31)) return MOE_ERR_UNSUPPORTED;
    const void *ptrs[] = {x_perm, offsets, W1, W3, W2, y_perm};
    for (const void *p : ptrs)
        if (p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u)) return MOE_ERR_INVALID_ARG;
    // The tile counters and H [S, d_ff] bf16 must fit in the fixed scratch
    // behind the header.
    if (static_need(S, E, d_ff) > kStaticScratchBytes) return MOE_ERR_WORKSPACE;
    const size_t ctr_bytes = (ffn_ready_counters(S, E, d_ff) * 4 + 255) / 256 * 256;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kStaticMaxDevices)
        return MOE_ERR_CUDA;
    uint8_t *scratch = static_cast<uint8_t *>(static_scratch_address(dev));
    if (scratch == nullptr) return MOE_ERR_CUDA;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // The error word and the tile counters must start at zero; H is fully
    // written before it is read.
    if (cudaMemsetAsync(scratch, 0, kStaticHeaderBytes + ctr_bytes, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    FfnLaunch f{};
    f.E = E;
    f.d = d;
    f.d_ff = d_ff;
    f.S = S;
    f.max_rows = S;
    f.ksplit = 1;
    f.offsets = offsets;
    f.W1 = W1;
    f.W3 = W3;
    f.W2 = W2;
    f.x = x_perm;
    f.H = reinterpret_cast<uint16_t *>(scratch + kStaticHeaderBytes + ctr_bytes);
    f.Y = y_perm;
    f.h_ready = reinterpret_cast<uint32_t *>(scratch + kStaticHeaderBytes);
    f.err = reinterpret_cast<uint32_t *>(scratch);
    f.pdl = false;
    if (launch_ffn(f, s) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

extern "C" moe_status moe_expert_ffn_static_error(uint32_t *code, moe_stream_t stream)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kStaticMaxDevices)
        return MOE_ERR_CUDA;
    const uint8_t *scratch = static_cast<const uint8_t *>(static_scratch_address(dev));
    if (scratch == nullptr) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return MOE_ERR_CUDA;
    uint32_t word = 0;
    if (cudaMemcpy(&word, scratch, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (code) *code = word;
    if (word == 0) return MOE_OK;
    if (word & (MOE_DEVERR_TIMEOUT_TMA | MOE_DEVERR_TIMEOUT_MMA | MOE_DEVERR_TIMEOUT_EPI))
        return MOE_ERR_TIMEOUT;
    return MOE_ERR_DEVICE;
}

extern "C" size_t moe_expert_ffn_static_bytes(int S, int E, int d_ff)
{
    if (S < 1 || E < 1 || E > 256 || d_ff < 128 || d_ff % 128 || d_ff > 65536 || S > (1 << 24))
        return 0;
    return static_need(S, E, d_ff);
}
