// Split-KV decode kernels for K4V4 caches.
#include "decode_launch.cuh"

namespace kvq {
template cudaError_t launch_decode_kv<4, 4>(const Layout&, int, const Batch&, const DecodePlan&, int, const void*,
                                              void*, const void*, const void*, float, void*, cudaStream_t, bool*);
template int decode_chunk_tokens_kv<4, 4>(int, int, int);
}  // namespace kvq
