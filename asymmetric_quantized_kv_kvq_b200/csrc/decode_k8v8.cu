// Split-KV decode kernels for K8V8 caches.
#include "decode_launch.cuh"

namespace kvq {
template cudaError_t launch_decode_kv<8, 8>(const Layout&, int, const Batch&, const DecodePlan&, int, const void*,
                                              void*, const void*, const void*, float, void*, cudaStream_t, bool*);
template int decode_chunk_tokens_kv<8, 8>(int, int, int);
}  // namespace kvq
