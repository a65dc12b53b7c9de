// Chunked prefill attention (placeholder until the tcgen05 kernel lands).
#include "kvq_internal.cuh"

namespace kvq {

size_t prefill_workspace_bytes(const Layout&, const Batch&) { return 0; }

cudaError_t launch_prefill(const Layout&, int, const Batch&, int, int, const void*, void*, float, void*, size_t, int,
                           cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace kvq
