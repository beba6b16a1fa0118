// noalloc.cu -- chunkwise forward for callers that cannot allocate device memory.
//
// Some hosts give a library only the input and output pointers and nothing
// else: plugin interfaces of inference runtimes that own every byte of device
// memory, or hot paths where cudaMalloc is not allowed because it can
// synchronise the whole device or fail under a budget fixed at start-up.  Such
// a caller cannot hand muir_chunk_fwd the workspace it needs.  This entry
// point runs the very same forward, with its workspace in a fixed-size array
// that is part of the library's device image instead of caller memory.
//
// Costs and limits a user should know:
// - Every GPU that loads the library holds kStaticScratchBytes (16 MiB) for
//   this array until the process exits, whether or not it is used.
// - Shapes whose workspace (muir_chunk_fwd_workspace) exceeds 16 MiB are
//   rejected with MUIR_ERR_WORKSPACE before anything is enqueued.
// - All calls share the one array.  Two calls whose work overlaps on the GPU
//   (different streams, or different host threads without ordering) race on
//   it and produce garbage; serialise them, e.g. on one stream.
// - The array keeps whatever the last call left in it.  The forward writes
//   every scratch element before reading it, so nothing has to be cleared
//   between calls.
// - The first call on each device looks up the array's device address
//   (cudaGetSymbolAddress) with that device current and keeps it for later
//   calls; make that first call before any stream capture.  The address
//   belongs to the device's primary context: after cudaDeviceReset (or any
//   other teardown of that context) the kept address is stale, so a process
//   that resets a device must not call this entry point on it again.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/muir.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

// The workspace of muir_chunk_fwd_noalloc.  In host code this name is only a
// handle for the runtime: its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_fwd_scratch[kStaticScratchBytes];

std::mutex g_lock;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_fwd_scratch on the current device, looked up once per device.
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> guard(g_lock);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        err = cudaGetSymbolAddress(&p, g_fwd_scratch);
        if (err != cudaSuccess) return err;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" muir_status muir_chunk_fwd_noalloc(const muir_shape* shape, const void* q,
                                              const void* k, const void* v, const void* g,
                                              const void* e, const void* w, const void* gamma,
                                              const float* S0, void* o, float* S_final,
                                              void* stream) {
    const size_t need = muir_chunk_fwd_workspace(shape);
    if (need == 0)  // invalid shape: let the regular entry point report which check failed
        return muir_chunk_fwd(shape, q, k, v, g, e, w, gamma, S0, o, S_final, nullptr, nullptr,
                              nullptr, nullptr, 0, stream);
    if (need > kStaticScratchBytes) return MUIR_ERR_WORKSPACE;
    // The library holds sm_100a code only: on another device the symbol lookup
    // would fail; report that as every other entry point does.
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return MUIR_ERR_CUDA;
    if (major != 10) return MUIR_ERR_UNSUPPORTED;
    void* ws = nullptr;
    if (scratch_address(&ws) != cudaSuccess) return MUIR_ERR_CUDA;
    return muir_chunk_fwd(shape, q, k, v, g, e, w, gamma, S0, o, S_final, nullptr, nullptr, nullptr,
                          ws, kStaticScratchBytes, stream);
}
