// Host-side launch of the split-KV decode kernels for one (K bits, V bits)
// pair; instantiated in one translation unit per pair.  Quantized caches run
// decode_q_kernel (warp roles, combine and optional append fused in); fp16
// caches run decode_split_kernel followed by the LSE combine kernel.
#pragma once

#include "decode_kernel.cuh"
#include "decode_q.cuh"

namespace kvq {

template <int KB, int VB, int D, int G>
cudaError_t launch_decode_one(const Layout& L, int layer, const Batch& b, const DecodePlan& plan, int n_q_heads,
                              const void* q, void* out, float scale_log2, void* ws, cudaStream_t s) {
  using T = DecodeTraits<KB, VB, D, G>;
  static bool configured = false;   // per instantiation; set once per process
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<KB, VB, D, G>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, T::SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  DecodeArgs a;
  a.L = L;
  a.layer = layer;
  a.n_q_heads = n_q_heads;
  a.q = static_cast<const __half*>(q);
  a.out = static_cast<__half*>(out);
  const int64_t slots = int64_t(plan.max_ctas) + plan.n_items;
  a.ws_o = static_cast<float*>(ws);
  a.ws_ml = a.ws_o + slots * G * D;
  a.scale_log2 = scale_log2;
  a.total_chunks = plan.total_chunks;
  a.cpc = plan.chunks_per_cta;
  a.chunk = plan.chunk_tokens;
  decode_split_kernel<KB, VB, D, G><<<plan.n_cta, T::NT, T::SMEM, s>>>(a, b);
  return cudaGetLastError();
}

template <int KB, int VB, int D, int G, int CT>
cudaError_t launch_decode_q_one(const Layout& L, int layer, const Batch& b, const DecodePlan& plan, int n_q_heads,
                                const void* q, void* out, const void* k_new, const void* v_new, float scale_log2,
                                void* ws, cudaStream_t s) {
  using T = QDec<KB, VB, D, G, CT>;
  static bool configured = false;   // per instantiation; set once per process
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(decode_q_kernel<KB, VB, D, G, CT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         T::SMEM);
    if (e != cudaSuccess) return e;
    // the in-kernel register split (setmaxnreg) adds up to the launch allocation; a build that
    // launched with fewer registers per thread would leave a growing warpgroup waiting
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, decode_q_kernel<KB, VB, D, G, CT>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != T::REG_L) return cudaErrorInvalidDeviceFunction;
    configured = true;
  }
  DecodeQArgs a;
  a.L = L;
  a.layer = layer;
  a.n_q_heads = n_q_heads;
  a.q = static_cast<const __half*>(q);
  a.out = static_cast<__half*>(out);
  a.k_new = static_cast<const __half*>(k_new);
  a.v_new = static_cast<const __half*>(v_new);
  const int64_t slots = int64_t(plan.max_ctas) + plan.n_items;
  a.ws_o = static_cast<float*>(ws);
  a.ws_ml = a.ws_o + slots * G * D;
  a.counters = L.counters;
  a.scale_log2 = scale_log2;
  a.total_chunks = plan.total_chunks;
  a.cpc = plan.chunks_per_cta;
  a.chunk = plan.chunk_tokens;
  decode_q_kernel<KB, VB, D, G, CT><<<plan.n_cta, T::NT, T::SMEM, s>>>(a, b);
  return cudaGetLastError();
}

// Decode launch for the (KB, VB) cache format.  k_new / v_new (fused append)
// are only taken by the quantized kernel; *combined tells the caller whether
// the split partials were already merged inside the kernel.
template <int KB, int VB>
cudaError_t launch_decode_kv(const Layout& L, int layer, const Batch& b, const DecodePlan& plan, int n_q_heads,
                             const void* q, void* out, const void* k_new, const void* v_new, float scale_log2,
                             void* ws, cudaStream_t s, bool* combined) {
  const int G = n_q_heads / L.n_kv_heads;
  if constexpr (KB != 16 && VB != 16) {
    *combined = true;
    // 256-token stages when the chunk is a whole 256 tokens (pages of 256k tokens) and three of them
    // fit in shared memory; 128-token stages otherwise
#define KVQ_DECQ(D_, G_)                                                                                         \
  if (L.head_dim == D_ && G == G_) {                                                                             \
    if constexpr (QDec<KB, VB, D_, G_, 256>::FITS)                                                               \
      if (plan.chunk_tokens == 256)                                                                              \
        return launch_decode_q_one<KB, VB, D_, G_, 256>(L, layer, b, plan, n_q_heads, q, out, k_new, v_new,      \
                                                        scale_log2, ws, s);                                      \
    return launch_decode_q_one<KB, VB, D_, G_, 128>(L, layer, b, plan, n_q_heads, q, out, k_new, v_new,          \
                                                    scale_log2, ws, s);                                          \
  }
    KVQ_DECQ(128, 1) KVQ_DECQ(128, 2) KVQ_DECQ(128, 4) KVQ_DECQ(128, 8)
    KVQ_DECQ(64, 1) KVQ_DECQ(64, 2) KVQ_DECQ(64, 4) KVQ_DECQ(64, 8)
#undef KVQ_DECQ
  } else {
    *combined = false;
    (void)k_new;
    (void)v_new;
#define KVQ_DEC(D_, G_) \
  if (L.head_dim == D_ && G == G_) return launch_decode_one<KB, VB, D_, G_>(L, layer, b, plan, n_q_heads, q, out, scale_log2, ws, s);
    KVQ_DEC(128, 1) KVQ_DEC(128, 2) KVQ_DEC(128, 4) KVQ_DEC(128, 8)
    KVQ_DEC(64, 1) KVQ_DEC(64, 2) KVQ_DEC(64, 4) KVQ_DEC(64, 8)
#undef KVQ_DEC
  }
  return cudaErrorInvalidValue;
}

// Stage capacity (tokens) of the kernel that runs for (D, G) on pages of page_tokens tokens.
template <int KB, int VB>
int decode_chunk_tokens_kv(int D, int G, int page_tokens) {
  if constexpr (KB != 16 && VB != 16) {
    const bool p256 = page_tokens % 256 == 0;
#define KVQ_CQ(D_, G_) \
  if (D == D_ && G == G_) return p256 && QDec<KB, VB, D_, G_, 256>::FITS ? 256 : 128;
    KVQ_CQ(128, 1) KVQ_CQ(128, 2) KVQ_CQ(128, 4) KVQ_CQ(128, 8)
    KVQ_CQ(64, 1) KVQ_CQ(64, 2) KVQ_CQ(64, 4) KVQ_CQ(64, 8)
#undef KVQ_CQ
    return 128;
  } else {
    (void)page_tokens;
#define KVQ_C(D_, G_) \
  if (D == D_ && G == G_) return DecodeTraits<KB, VB, D_, G_>::C;
    KVQ_C(128, 1) KVQ_C(128, 2) KVQ_C(128, 4) KVQ_C(128, 8)
    KVQ_C(64, 1) KVQ_C(64, 2) KVQ_C(64, 4) KVQ_C(64, 8)
#undef KVQ_C
  }
  return 0;
}

}  // namespace kvq
