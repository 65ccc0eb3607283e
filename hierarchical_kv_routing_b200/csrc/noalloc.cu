// hga_forward_prefill_noalloc: the prefill path for callers that cannot
// allocate device memory, running on a fixed scratch array that lives in
// this library's device image.
//
// Who needs it: code that runs where a cudaMalloc is not available or not
// allowed at call time, for example a serving loop whose device memory is
// all owned by another allocator (a framework's caching allocator, or a
// fixed arena sized at start-up), where a raw cudaMalloc may fail or may
// synchronise the device in the middle of a latency-critical step; or a
// plug-in called from a host runtime that hands it only input and output
// buffers.  Those callers pass inputs and outputs and nothing else.
//
// The scratch (rotated keys, chunk and group summaries, routed ids) is one
// file-scope __device__ array of kNoAllocScratchBytes.  Every GPU that loads
// this library holds that much memory until the process exits.  In host
// code the array's name is only a host-side stand-in, so its device address
// is looked up with cudaGetSymbolAddress, once per device, with that device
// current, on the first call made on that device.
#include <cuda_runtime.h>

#include <mutex>

#include "hga_internal.cuh"

namespace hga {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_noalloc_mu;
void *g_noalloc_addr[kNoAllocMaxDevices] = {};
}  // namespace

}  // namespace hga

extern "C" hga_status hga_forward_prefill_noalloc(const hga_dims *dims, const hga_params *prm,
                                                  const void *q, const void *k, const void *v,
                                                  const int32_t *pos, void *out, float *lse,
                                                  void *stream) {
    using namespace hga;
    // the smallest prefill workspace (0 for malformed arguments: hga_forward
    // then reports them); with room to spare hga_forward also keeps the
    // rotated queries in the scratch
    const size_t need = hga_prefill_workspace_min(dims, prm);
    if (need > kNoAllocScratchBytes) return HGA_ERR_WORKSPACE;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e);
    if (dev < 0 || dev >= kNoAllocMaxDevices) return HGA_ERR_UNSUPPORTED;
    void *base = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_noalloc_mu);
        if (!g_noalloc_addr[dev]) {
            e = cudaGetSymbolAddress(&g_noalloc_addr[dev], g_noalloc_scratch);
            if (e != cudaSuccess) {
                g_noalloc_addr[dev] = nullptr;
                return cuda_status(e);
            }
        }
        base = g_noalloc_addr[dev];
    }
    hga_io io = {};
    io.q = q;
    io.k = k;
    io.v = v;
    io.pos = pos;
    io.out = out;
    io.lse = lse;
    return hga_forward(HGA_PREFILL, dims, prm, &io, base, kNoAllocScratchBytes, stream);
}
