// Content hashing and comparison of physical pages, for deduplicating full
// pages that hold the same bytes in every layer (the content hash of the
// KVBoost page, "KVBoost acelera inferencia de LLMs em 4,49x com cache
// reutilizavel", section "Contexto": cached chunks are found again by a hash of
// their content).
//
// A page's bytes in one layer are the n_kv_heads head blocks of that layer,
// which are contiguous.  The hash is 128 bits, four 32-bit lanes: 16-byte word
// group i of a layer region contributes word k of the group to lane k as
//   h_k += mix(w_k ^ (i * 0x9E3779B9 + layer * 0x85EBCA77))   (mod 2^32),
//   mix(x) = (x * 0x85EBCA6B) ^ ((x * 0x85EBCA6B) >> 13),
// a sum, so the order in which CTAs add their parts does not matter and the
// result is exact and deterministic.  The hash only proposes candidates: pages
// are merged after comparing their bytes (page_compare_kernel), so a collision
// can never merge different contents.
#include <cstdint>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kDedupThreads = 256;
constexpr int kDedupVecPerThread = 16;   // 16-byte loads per thread per CTA slice

__device__ __forceinline__ uint32_t dedup_mix(uint32_t x) {
  x *= 0x85EBCA6Bu;
  return x ^ (x >> 13);
}

// grid: (slices of one layer region, layer, page in the list); hashes[4 * i + k] += lane k.
__global__ void __launch_bounds__(kDedupThreads) page_hash_kernel(const __grid_constant__ PageList pl,
                                                                  uint32_t* __restrict__ hashes) {
  const int i = blockIdx.z, layer = blockIdx.y;
  const PageRegion& r = pl.layer[layer];
  const uint4* base = reinterpret_cast<const uint4*>(r.base + int64_t(pl.page[i]) * r.bytes);
  const int64_t n_vec = r.bytes / 16;
  const int64_t v0 = int64_t(blockIdx.x) * kDedupThreads * kDedupVecPerThread;
  uint32_t h[4] = {0u, 0u, 0u, 0u};
  const uint32_t lsalt = uint32_t(layer) * 0x85EBCA77u;
#pragma unroll 4
  for (int j = 0; j < kDedupVecPerThread; ++j) {
    const int64_t v = v0 + int64_t(j) * kDedupThreads + threadIdx.x;   // coalesced: consecutive threads, consecutive 16 B
    if (v < n_vec) {
      const uint4 w = __ldcs(base + v);
      const uint32_t salt = uint32_t(v) * 0x9E3779B9u + lsalt;
      h[0] += dedup_mix(w.x ^ salt);
      h[1] += dedup_mix(w.y ^ salt);
      h[2] += dedup_mix(w.z ^ salt);
      h[3] += dedup_mix(w.w ^ salt);
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) h[k] += __shfl_xor_sync(0xffffffffu, h[k], o);
  if ((threadIdx.x & 31) == 0)
#pragma unroll
    for (int k = 0; k < 4; ++k) atomicAdd(hashes + 4 * i + k, h[k]);
}

// grid: (slices, layer, pair in the list): diff[i] != 0 when page a[i] and page b[i] differ.
__global__ void __launch_bounds__(kDedupThreads) page_compare_kernel(const __grid_constant__ PagePairs pp,
                                                                     uint32_t* __restrict__ diff) {
  const int i = blockIdx.z, layer = blockIdx.y;
  const PageRegion& r = pp.layer[layer];
  const uint4* a = reinterpret_cast<const uint4*>(r.base + int64_t(pp.a[i]) * r.bytes);
  const uint4* b = reinterpret_cast<const uint4*>(r.base + int64_t(pp.b[i]) * r.bytes);
  const int64_t n_vec = r.bytes / 16;
  const int64_t v0 = int64_t(blockIdx.x) * kDedupThreads * kDedupVecPerThread;
  uint32_t d = 0;
#pragma unroll 4
  for (int j = 0; j < kDedupVecPerThread; ++j) {
    const int64_t v = v0 + int64_t(j) * kDedupThreads + threadIdx.x;
    if (v < n_vec) {
      const uint4 x = __ldcs(a + v), y = __ldcs(b + v);
      d |= (x.x ^ y.x) | (x.y ^ y.y) | (x.z ^ y.z) | (x.w ^ y.w);
    }
  }
  if (__any_sync(0xffffffffu, d != 0) && (threadIdx.x & 31) == 0) atomicOr(diff + i, 1u);
}

dim3 dedup_grid(const PageRegion* layers, int n_layers, int n) {
  int64_t most = 0;
  for (int l = 0; l < n_layers; ++l) most = layers[l].bytes > most ? layers[l].bytes : most;
  const int64_t per_cta = int64_t(kDedupThreads) * kDedupVecPerThread * 16;
  return dim3(unsigned((most + per_cta - 1) / per_cta), unsigned(n_layers), unsigned(n));
}

}  // namespace

cudaError_t launch_page_hash(const PageList& pl, int n_layers, uint32_t* hashes, bool zero_first, cudaStream_t s) {
  if (pl.n == 0) return cudaSuccess;
  if (zero_first) {
    const cudaError_t e = cudaMemsetAsync(hashes, 0, size_t(pl.n) * 4 * sizeof(uint32_t), s);
    if (e != cudaSuccess) return e;
  }
  page_hash_kernel<<<dedup_grid(pl.layer, n_layers, pl.n), kDedupThreads, 0, s>>>(pl, hashes);
  return cudaGetLastError();
}

cudaError_t launch_page_compare(const PagePairs& pp, int n_layers, uint32_t* diff, bool zero_first, cudaStream_t s) {
  if (pp.n == 0) return cudaSuccess;
  if (zero_first) {
    const cudaError_t e = cudaMemsetAsync(diff, 0, size_t(pp.n) * sizeof(uint32_t), s);
    if (e != cudaSuccess) return e;
  }
  page_compare_kernel<<<dedup_grid(pp.layer, n_layers, pp.n), kDedupThreads, 0, s>>>(pp, diff);
  return cudaGetLastError();
}

}  // namespace kvq
