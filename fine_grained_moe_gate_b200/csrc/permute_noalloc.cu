// moe_permute_noalloc: the expert-contiguous permutation of moe_permute for
// callers that cannot give the library any scratch memory -- for example a
// host framework that owns all device memory and exposes no allocator to
// its plugins, or a deployment that reserves a fixed device-memory budget
// up front and forbids allocating at run time (cudaMalloc/cudaFree can also
// synchronise the device, which such callers may not allow).
//
// Its scratch (the per-chunk expert histogram the stable ranking needs) is a
// fixed array in this library's device image instead of a caller workspace.
// Every GPU that loads the library holds this array until the process exits.
#include "../../include/moe_gate.h"
#include "kernels.h"

#include <cuda_runtime.h>

#include <mutex>

namespace {

// Room for ceil(T / 128) * E int32 counters: 65536 of them (256 KiB), e.g.
// T = 32768 tokens with E = 256 experts.
constexpr size_t kNoAllocScratchBytes = 256 * 1024;
static __device__ __align__(256) int32_t g_permute_scratch[kNoAllocScratchBytes / sizeof(int32_t)];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the array on the current device.  The array's name in
// host code is only a host-side handle, so its address is looked up once
// per device, with that device current, and cached.
moe_status scratch_on_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_permute_noalloc(const void* x, const int32_t* topk_idx, const int32_t* counts, moe_shape sh,
                                          void* x_perm, int32_t* offsets, int32_t* perm_tok, int32_t* inv_row,
                                          void* stream) {
    const size_t need = moe_permute_workspace_size(sh);
    if (need > kNoAllocScratchBytes) return MOE_ERR_UNSUPPORTED;  // larger than the built-in scratch
    void* scratch = nullptr;
    if (need > 0) {
        moe_status s = scratch_on_current_device(&scratch);
        if (s != MOE_OK) return s;
    }
    // The histogram pass writes every counter it later reads, so nothing in
    // the array has to start at zero; the previous call's contents are
    // simply overwritten.
    return moe_permute(x, topk_idx, counts, sh, x_perm, offsets, perm_tok, inv_row, scratch, kNoAllocScratchBytes,
                       stream);
}
