// moe_noalloc.cu -- moe_forward_noalloc: the layer for small batches without any allocation.
//
// Some callers may not allocate device memory at all: code that runs while a CUDA graph is being
// captured (where a new allocation would break or serialise the capture), inference loops with
// a fixed memory budget that must not touch an allocator in steady state, and plug-ins whose
// host framework owns every allocation.  For them this entry point uses a scratch area that is
// part of the library image: a file-scope __device__ array, present on every GPU that loads the
// library and held until the process exits.  Nothing else about the layer changes: the call
// goes through moe_forward with that area as its workspace.
#include <mutex>

#include "moe_internal.cuh"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(4) << 20;   // 4 MiB per GPU
constexpr int kMaxDevices = 64;

__device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_mu;
void *g_scratch[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per device; the
// host-side symbol itself is not a device address).
moe_status scratch_for_current_device(uint8_t **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
        g_scratch[dev] = p;
    }
    *out = static_cast<uint8_t *>(g_scratch[dev]);
    return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_forward_noalloc(const moe_arena *arena, const float *d_x,
                                          const float *d_logits, int T, int k, float *d_out,
                                          uint32_t *d_status, void *stream) {
    // every check moe_forward would make, before anything is enqueued
    moe_status st = moe::check_forward_args(arena, d_x, d_logits, T, k, d_out, 0);
    if (st != MOE_OK) return st;
    if (T > moe::kDecodeMaxT) return MOE_ERR_INVALID_ARG;
    if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3)) return MOE_ERR_ALIGNMENT;
    const moe::WsLayout L = moe::ws_layout(arena, T, k, 0);
    if (L.total > kNoallocScratchBytes) return MOE_ERR_UNSUPPORTED;
    uint8_t *ws = nullptr;
    st = scratch_for_current_device(&ws);
    if (st != MOE_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the status word and the kernel's counters (the first bytes of the layout) must start at
    // zero; the previous call's contents are otherwise left as they are
    if (cudaMemsetAsync(ws, 0, L.sync + 4 * sizeof(uint32_t), s) != cudaSuccess)
        return MOE_ERR_CUDA;
    st = moe_forward(arena, d_x, d_logits, T, k, d_out, ws, kNoallocScratchBytes, 0, stream);
    if (st != MOE_OK) return st;
    if (d_status && cudaMemcpyAsync(d_status, ws + L.status, sizeof(uint32_t),
                                    cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}
