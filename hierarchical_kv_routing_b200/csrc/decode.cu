// Decode step: placeholder until the decode kernels land.
#include "hga_internal.cuh"

namespace hga {

size_t decode_workspace_bytes(const Geo &) { return 0; }

hga_status launch_decode(const Geo &, const Rope &, int, const hga_io &, void *, cudaStream_t) {
    return HGA_ERR_UNSUPPORTED;
}

}  // namespace hga
