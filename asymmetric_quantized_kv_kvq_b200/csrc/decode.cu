// Split-KV decode: dispatch over cache formats, and the log-sum-exp combine
// of partial results (O_s, m_s, l_s) written by the split kernel:
//   o = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s,  M = max_s m_s
// (m in the log2 domain of the scaled scores).
#include <cuda_fp16.h>

#include "kvq_internal.cuh"

namespace kvq {

template <int KB, int VB>
cudaError_t launch_decode_kv(const Layout&, int, const Batch&, const DecodePlan&, int, const void*, void*, const void*,
                             const void*, float, void*, cudaStream_t, bool*);
template <int KB, int VB>
int decode_chunk_tokens_kv(int D, int G, int page_tokens);

bool decode_tc_supported(const Layout& L, int G);
int decode_tc_tile_tokens();
cudaError_t launch_decode_tc(const Layout& L, int layer, const Batch& b, const DecodePlan& plan, int n_q_heads,
                             const void* q, void* out, float scale_log2, void* ws, cudaStream_t s);

namespace {

// One warp per (item, query head).  The lanes share the item's partial slots:
// each lane reads the (m, l) of slots lane, lane + 32, ... for the warp-wide max
// M and sum L, then the warp walks the slots once, every lane accumulating its
// D / 32 contiguous elements of O (one vector load per slot, weights broadcast
// by shuffle), so the loads of successive slots are independent.
template <int D>
__global__ void lse_combine_kernel(const __grid_constant__ Batch b, int H, int G, int n_q_heads, int64_t cpc,
                                   const float* __restrict__ ws_o, const float* __restrict__ ws_ml,
                                   __half* __restrict__ out) {
  constexpr int E = D / 32;   // elements per lane: 2 (D = 64) or 4 (D = 128)
  const int lane = threadIdx.x & 31;
  const int64_t wid = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (wid >= int64_t(b.n) * H * G) return;
  const int item = int(wid / G), g = int(wid % G);
  const int bi = item / H, h = item % H;
  const int nch = b.s[bi].c;
  const int64_t off = int64_t(b.s[bi].b) + int64_t(h) * nch;
  const int64_t c0 = off / cpc, c1 = (off + nch - 1) / cpc;
  if (c0 == c1) return;   // written directly by the split kernel
  const int n = int(c1 - c0 + 1);
  const float* ml = ws_ml + ((c0 + item) * G + g) * 2;          // slot c0 + i at ml[2 * G * i]
  float M = -INFINITY;
  for (int i = lane; i < n; i += 32) M = fmaxf(M, ml[int64_t(2) * G * i]);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float L = 0.f;
  for (int i = lane; i < n; i += 32) L += exp2f(ml[int64_t(2) * G * i] - M) * ml[int64_t(2) * G * i + 1];
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  const float* o0 = ws_o + ((c0 + item) * G + g) * D + E * lane;  // slot c0 + i at o0[G * D * i]
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    const float w = i < n ? exp2f(ml[int64_t(2) * G * i] - M) : 0.f;
    const int cnt = min(32, n - base);
#pragma unroll 4
    for (int k = 0; k < cnt; ++k) {
      const float wk = __shfl_sync(0xffffffffu, w, k);
      const float* src = o0 + int64_t(G) * D * (base + k);
      if constexpr (E == 4) {
        const float4 v = *reinterpret_cast<const float4*>(src);
        acc[0] = fmaf(wk, v.x, acc[0]); acc[1] = fmaf(wk, v.y, acc[1]);
        acc[2] = fmaf(wk, v.z, acc[2]); acc[3] = fmaf(wk, v.w, acc[3]);
      } else {
        const float2 v = *reinterpret_cast<const float2*>(src);
        acc[0] = fmaf(wk, v.x, acc[0]); acc[1] = fmaf(wk, v.y, acc[1]);
      }
    }
  }
  const float inv = 1.f / L;
  __half* dst = out + (int64_t(bi) * n_q_heads + h * G + g) * D + E * lane;
#pragma unroll
  for (int e = 0; e < E; e += 2) *reinterpret_cast<__half2*>(dst + e) = __floats2half2_rn(acc[e] * inv, acc[e + 1] * inv);
}

}  // namespace

int decode_max_ctas(int num_sms) { return num_sms < kMaxDecodeCtas ? num_sms : kMaxDecodeCtas; }

size_t decode_workspace_bytes(int n_items, int max_ctas, int G, int D) {
  const size_t slots = size_t(max_ctas) + size_t(n_items);
  return slots * G * (D + 2) * sizeof(float);
}

static int stage_tokens(const Layout& L, int G) {
  const int kb = L.k_bits, vb = L.v_bits, D = L.head_dim;
  if (decode_tc_supported(L, G)) return decode_tc_tile_tokens();
  if (kb == 16) return decode_chunk_tokens_kv<16, 16>(D, G, L.page_tokens);
  if (kb == 8 && vb == 8) return decode_chunk_tokens_kv<8, 8>(D, G, L.page_tokens);
  if (kb == 8 && vb == 4) return decode_chunk_tokens_kv<8, 4>(D, G, L.page_tokens);
  if (kb == 4 && vb == 4) return decode_chunk_tokens_kv<4, 4>(D, G, L.page_tokens);
  return decode_chunk_tokens_kv<4, 8>(D, G, L.page_tokens);
}

// Work chunk = gcd(stage capacity, page_tokens): both are multiples of 64, the
// chunk divides the page, so one chunk is one contiguous range of one page.
int decode_chunk_tokens(const Layout& L, int G) {
  int x = stage_tokens(L, G), y = L.page_tokens;
  while (y) {
    const int t = x % y;
    x = y;
    y = t;
  }
  return x;
}

cudaError_t launch_decode(const Layout& L, int layer, const Batch& b, const DecodePlan& plan, int n_q_heads,
                          const void* q, void* out, const void* k_new, const void* v_new, float scale_log2, void* ws,
                          cudaStream_t s) {
  const int kb = L.k_bits, vb = L.v_bits;
  cudaError_t e;
  bool combined = false;
  if (decode_tc_supported(L, n_q_heads / L.n_kv_heads))
    e = launch_decode_tc(L, layer, b, plan, n_q_heads, q, out, scale_log2, ws, s);
  else if (kb == 16)
    e = launch_decode_kv<16, 16>(L, layer, b, plan, n_q_heads, q, out, k_new, v_new, scale_log2, ws, s, &combined);
  else if (kb == 8 && vb == 8)
    e = launch_decode_kv<8, 8>(L, layer, b, plan, n_q_heads, q, out, k_new, v_new, scale_log2, ws, s, &combined);
  else if (kb == 8 && vb == 4)
    e = launch_decode_kv<8, 4>(L, layer, b, plan, n_q_heads, q, out, k_new, v_new, scale_log2, ws, s, &combined);
  else if (kb == 4 && vb == 4)
    e = launch_decode_kv<4, 4>(L, layer, b, plan, n_q_heads, q, out, k_new, v_new, scale_log2, ws, s, &combined);
  else
    e = launch_decode_kv<4, 8>(L, layer, b, plan, n_q_heads, q, out, k_new, v_new, scale_log2, ws, s, &combined);
  if (e != cudaSuccess) return e;
  // separate combine only for the kernels that leave split items' partials in the workspace
  if (!combined && (plan.n_cta > 1 || plan.n_items > 1)) {
    const int H = L.n_kv_heads, G = n_q_heads / H, D = L.head_dim;
    const int64_t slots = int64_t(plan.max_ctas) + plan.n_items;
    const float* ws_o = static_cast<const float*>(ws);
    const float* ws_ml = ws_o + slots * G * D;
    const int64_t warps = int64_t(plan.n_items) * G;
    const unsigned blocks = unsigned((warps + 7) / 8);
    if (D == 128)
      lse_combine_kernel<128><<<blocks, 256, 0, s>>>(b, H, G, n_q_heads, plan.chunks_per_cta, ws_o, ws_ml,
                                                     static_cast<__half*>(out));
    else
      lse_combine_kernel<64><<<blocks, 256, 0, s>>>(b, H, G, n_q_heads, plan.chunks_per_cta, ws_o, ws_ml,
                                                    static_cast<__half*>(out));
    e = cudaGetLastError();
  }
  return e;
}

// True when launch_decode quantises k_new / v_new itself (fused append).
bool decode_fuses_append(const Layout& L, int G) {
  return L.k_bits != 16 && L.v_bits != 16 && !decode_tc_supported(L, G);
}

}  // namespace kvq
