// ba_fwd_noalloc: the forward pass for callers that cannot allocate device
// memory, with its scratch in a fixed array compiled into the library.
//
// Who needs it: a host framework that owns every byte of device memory
// through its own pool and gives kernels only their inputs and outputs, or a
// plugin running inside such a framework without access to its allocator.
// Such a caller cannot obtain the workspace ba_fwd asks for, so this entry
// point brings its own.
//
// The scratch is one file-scope __device__ array of kScratchBytes; every GPU
// that loads the library holds it until the process exits. Its device address
// is looked up once per device, on the first call made with that device
// current, and cached for the life of the process (a context destroyed and
// created again may place the array elsewhere, so the entry point is not for
// use across a device reset). All calls share the array: two calls whose
// work may overlap on the GPU (different streams, or different host threads
// without ordering) race on it. Every byte the forward reads from the scratch
// is written earlier in the same call (the work-list kernel rewrites the
// status word, the tile prefix and the tile table), so nothing left behind by
// a previous call needs clearing.
#include "ba.h"

#include <atomic>
#include <cuda_runtime.h>
#include <mutex>

namespace {

constexpr size_t kScratchBytes = size_t(1) << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_fwd_scratch[kScratchBytes];

std::atomic<void *> g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mutex;

// Device address of g_fwd_scratch on the current device, or nullptr.
void *scratch_address()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    void *addr = g_scratch_addr[dev].load();
    if (addr) return addr;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    addr = g_scratch_addr[dev].load();
    if (!addr) {
        if (cudaGetSymbolAddress(&addr, g_fwd_scratch) != cudaSuccess) return nullptr;
        g_scratch_addr[dev].store(addr);
    }
    return addr;
}

} // namespace

extern "C" ba_status ba_fwd_noalloc(const ba_problem *p, const void *q, const void *k, const void *v,
                                    const int32_t *seq_offsets, int32_t block, int32_t window,
                                    const uint8_t *skip, void *out, float *lse, ba_stream_t stream)
{
    const size_t need = ba_fwd_workspace_size(p, block, window);
    if (need == 0 || need > kScratchBytes) return BA_ERR_INVALID_ARG;
    void *scratch = scratch_address();
    if (!scratch) return BA_ERR_CUDA;
    return ba_fwd(p, q, k, v, seq_offsets, block, window, skip, out, lse, scratch, kScratchBytes, stream);
}
