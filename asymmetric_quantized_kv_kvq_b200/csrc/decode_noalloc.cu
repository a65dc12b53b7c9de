// kvq_decode_attn_noalloc: decode attention whose scratch lives in a fixed
// array compiled into the library, for callers that cannot allocate device
// memory themselves.
//
// Who needs it: code that runs inside a host application which owns all device
// memory and hands a plugin only its inputs and outputs (inference servers'
// custom operators with a fixed memory budget, engines whose caching allocator
// has reserved the whole GPU so that a cudaMalloc would fail), and serving
// loops that must not call cudaMalloc / cudaFree at all because those calls can
// synchronise the device.  Such a caller still passes q and out; the
// split-KV partial results go to the array below instead of a caller buffer.
//
// The array is a file-scope __device__ object: every GPU that loads the
// library holds KVQ_NOALLOC_SCRATCH_BYTES of it until the process exits.  In
// host code its name is only a host-side stand-in, so the device address is
// looked up once per device with cudaGetSymbolAddress (with that device
// current) and cached; that set-up happens on the first call on each device.
// All calls share the array: calls that overlap on the GPU (two streams, or
// two threads) race on it, so callers must order them.  Nothing in it has to
// start at zero: every partial slot the decode reads in a call is written
// earlier in the same call.
#include <mutex>

#include "kvq_internal.cuh"

namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[KVQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

extern "C" KVQ_API kvq_status kvq_decode_attn_noalloc(kvq_cache* cache, int32_t layer, int32_t n_seqs,
                                                      const int32_t* seq_ids, int32_t n_q_heads, const void* q,
                                                      void* out, float softmax_scale, kvq_stream_t stream) {
  size_t need = 0;
  if (kvq_status s = kvq_decode_workspace_size(cache, n_seqs, n_q_heads, &need)) return s;
  if (need > KVQ_NOALLOC_SCRATCH_BYTES)
    return kvq::set_last_error(KVQ_ERR_WORKSPACE,
                               "kvq_decode_attn_noalloc: this batch needs more scratch than the fixed "
                               "KVQ_NOALLOC_SCRATCH_BYTES (8 MiB); split the batch or call kvq_decode_attn "
                               "with a caller-owned workspace");
  // a host-only cache, or a current device other than the cache's, is refused
  // before the scratch address is looked up (which would touch the device)
  int dev = 0;
  if (kvq_status s = kvq::launch_device(cache, &dev)) return s;
  if (dev < 0 || dev >= kMaxDevices)
    return kvq::set_last_error(KVQ_ERR_UNSUPPORTED, "kvq_decode_attn_noalloc: device index out of range");
  void* ptr = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
      if (cudaGetSymbolAddress(&g_scratch_ptr[dev], g_decode_scratch) != cudaSuccess) {
        g_scratch_ptr[dev] = nullptr;
        return kvq::set_last_error(KVQ_ERR_CUDA, "kvq_decode_attn_noalloc: cudaGetSymbolAddress failed");
      }
    }
    ptr = g_scratch_ptr[dev];
  }
  return kvq_decode_attn(cache, layer, n_seqs, seq_ids, n_q_heads, q, out, softmax_scale, ptr,
                         KVQ_NOALLOC_SCRATCH_BYTES, stream);
}
