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
// looked up once per device with cudaGetSymbolAddress (with that device
// current) on the first call made on that device, and that address is what
// the kernels receive.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "internal.h"
#include "moe.h"

namespace moe {

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB
constexpr size_t kStaticHeaderBytes = 256;                // device error word, then H
constexpr int kStaticMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_static_mutex;
void *g_static_ptr[kStaticMaxDevices] = {};

// Device address of g_static_scratch on the current device (looked up once
// per device).  Returns nullptr if the lookup failed.
void *static_scratch_address(int dev)
{
    std::lock_guard<std::mutex> lock(g_static_mutex);
    if (g_static_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) return nullptr;
        g_static_ptr[dev] = p;
    }
    return g_static_ptr[dev];
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
    const size_t ctr_bytes = (ffn_ready_counters(S, E, d_ff) * 4 + 255) / 256 * 256;
    const size_t h_bytes = static_cast<size_t>(S) * d_ff * 2;
    if (ctr_bytes + h_bytes > kStaticScratchBytes - kStaticHeaderBytes) return MOE_ERR_WORKSPACE;

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
