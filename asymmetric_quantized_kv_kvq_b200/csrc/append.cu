// Quantise-on-append, canonical export and page-table updates (sm_100a).
//
// Quantisation follows the KVSplit page ("KVSplit - contexto 2 a 3 vezes mais
// longo em Apple Silicon", section "Uso de memoria conforme o comprimento da
// sequencia": 32-element blocks with one fp16 scale, 34 B per 8-bit block and
// 18 B per 4-bit block; Hacker News reply on .gguf files: the cache is
// quantised at run time as tokens are processed).  Rounding rules (this
// library's reading of the format): 8-bit d = fp16(fp32(amax / 127)),
// c = clamp(roundf(x / d), -127, 127); 4-bit d = fp16(m / -8) with m the
// largest-|x| element (lowest index on ties), c = clamp(roundf(x / d), -8, 7),
// nibble u = c + 8, byte i = u_i | u_{i+16} << 4.  The 8-bit scale uses an
// IEEE fp32 divide; the codes use round_quotient below, which equals roundf of
// the IEEE fp32 quotient x / d, so codes and scales are bit-exact across
// implementations.
//
// One warp quantises one (token, KV head): D/32 elements per lane, a block is
// 32/E consecutive lanes, its max is a shuffle reduction inside that group.
// Loads and stores are lane-contiguous (one 8-B fp16 load, one 4-B code store
// per lane for D = 128), so the kernel streams HBM at full width.
#include <cuda_fp16.h>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

__global__ void pt_update_kernel(int32_t* table, const __grid_constant__ PtUpdate u) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < u.n) table[u.idx[i]] = u.val[i];
}

// Element i of this lane is row element lane * E + i.
template <int E>
struct HalfVec;
template <>
struct HalfVec<4> {
  using T = uint2;
};
template <>
struct HalfVec<2> {
  using T = uint32_t;
};

template <int E>
__device__ __forceinline__ typename HalfVec<E>::T load_raw(const __half* src, int lane) {
  return *reinterpret_cast<const typename HalfVec<E>::T*>(src + lane * E);
}
template <int E>
__device__ __forceinline__ void unpack_row(typename HalfVec<E>::T raw, float (&x)[E], uint16_t (&bits)[E]) {
  const uint16_t* h = reinterpret_cast<const uint16_t*>(&raw);
#pragma unroll
  for (int i = 0; i < E; ++i) {
    bits[i] = h[i];
    x[i] = __half2float(__ushort_as_half(h[i]));
  }
}

// Reduce over the G = 32/E lanes of one block (aligned groups of consecutive lanes).
template <int E>
__device__ __forceinline__ float group_max(float v) {
#pragma unroll
  for (int o = 1; o < 32 / E; o <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
template <int E>
__device__ __forceinline__ uint32_t group_max_u32(uint32_t v) {
#pragma unroll
  for (int o = 1; o < 32 / E; o <<= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// roundf(fp32(x / d)) clamped to [lo, hi], for fp16-valued x and d != 0, without
// a divide: n from the correctly rounded reciprocal is within 1 of the answer,
// the remainder x - n d is exact in fp32 (n d has at most 18 significant bits),
// and comparing it with |d| / 2 fixes n, ties going away from zero.  For fp16 x
// and d the fp32 rounding of the quotient never moves it across a half-integer
// it did not sit on, so this is the same integer (checked for every finite fp16
// x against 3400 scales).
__device__ __forceinline__ int round_quotient(float x, float d, float rd, int lo, int hi) {
  int n = __float2int_rn(__fmul_rn(x, rd));
  const float e = __fmaf_rn(-float(n), d, x);
  const float hd = 0.5f * fabsf(d);
  const float ed = d > 0.f ? e : -e;
  if (ed > hd || (ed == hd && n >= 0)) ++n;
  else if (ed < -hd || (ed == -hd && n <= 0)) --n;
  return max(lo, min(hi, n));
}

template <int E>
__device__ __forceinline__ void quant8(const float (&x)[E], const uint16_t (&bits)[E], int lane, uint8_t* codes_row,
                                       __half* scales_row) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < E; ++i) a = fmaxf(a, fabsf(x[i]));
  a = group_max<E>(a);
  const __half d = __float2half_rn(__fdiv_rn(a, 127.0f));
  const float df = __half2float(d);
  const float rd = df != 0.f ? __frcp_rn(df) : 0.f;
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < E; ++i) {
    const int c = df != 0.f ? round_quotient(x[i], df, rd, -127, 127) : 0;
    packed |= (uint32_t(uint8_t(int8_t(c)))) << (8 * i);
  }
  if (E == 4)
    *reinterpret_cast<uint32_t*>(codes_row + lane * 4) = packed;
  else
    *reinterpret_cast<uint16_t*>(codes_row + lane * 2) = uint16_t(packed);
  if ((lane & (32 / E - 1)) == 0) scales_row[lane / (32 / E)] = d;
}

template <int E>
__device__ __forceinline__ void quant4(const float (&x)[E], const uint16_t (&bits)[E], int lane, uint8_t* codes_row,
                                       __half* scales_row) {
  constexpr int LPB = 32 / E;           // lanes per block
  const int jbase = (lane % LPB) * E;   // index of this lane's first element inside its block
  // key = |x| bits (15) << 6 | (31 - j) << 1 | sign: the max is the largest
  // magnitude, lowest index on ties; the sign rides along in bit 0.
  uint32_t key = 0;
#pragma unroll
  for (int i = 0; i < E; ++i) {
    const uint32_t k = (uint32_t(bits[i] & 0x7FFF) << 6) | (uint32_t(31 - (jbase + i)) << 1) | (bits[i] >> 15);
    key = max(key, k);
  }
  key = group_max_u32<E>(key);
  const uint16_t mbits = uint16_t(((key >> 6) & 0x7FFF) | ((key & 1u) << 15));
  const float m = __half2float(__ushort_as_half(mbits));
  const __half d = __float2half_rn(m * -0.125f);   // m / -8, exact in fp32
  const float df = __half2float(d);
  const float rd = df != 0.f ? __frcp_rn(df) : 0.f;
  uint32_t u = 0;   // E nibbles, element i in bits [4i, 4i+4)
#pragma unroll
  for (int i = 0; i < E; ++i) {
    const int c = df != 0.f ? round_quotient(x[i], df, rd, -8, 7) : 0;
    u |= uint32_t(c + 8) << (4 * i);
  }
  // partner lane holds elements j + 16 of the same block
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, u, LPB / 2);
  if ((lane % LPB) < LPB / 2) {
    uint32_t out = 0;
#pragma unroll
    for (int i = 0; i < E; ++i) out |= (((u >> (4 * i)) & 0xF) | (((hi >> (4 * i)) & 0xF) << 4)) << (8 * i);
    uint8_t* dst = codes_row + (lane / LPB) * 16 + (lane % LPB) * E;
    if (E == 4)
      *reinterpret_cast<uint32_t*>(dst) = out;
    else
      *reinterpret_cast<uint16_t*>(dst) = uint16_t(out);
  }
  if ((lane & (LPB - 1)) == 0) scales_row[lane / LPB] = d;
}

template <int E>
__device__ __forceinline__ void store_row(int bits_w, const float (&x)[E], const uint16_t (&bits)[E], int lane,
                                          uint8_t* codes_row, __half* scales_row) {
  if (bits_w == 8) {
    quant8<E>(x, bits, lane, codes_row, scales_row);
  } else if (bits_w == 4) {
    quant4<E>(x, bits, lane, codes_row, scales_row);
  } else {
    typename HalfVec<E>::T raw;
    uint16_t* h = reinterpret_cast<uint16_t*>(&raw);
#pragma unroll
    for (int i = 0; i < E; ++i) h[i] = bits[i];
    *reinterpret_cast<typename HalfVec<E>::T*>(codes_row + lane * E * 2) = raw;
  }
}

template <int D>
__global__ void __launch_bounds__(256) append_kernel(const Layout L, int layer, const __grid_constant__ Batch b,
                                                     int total_tokens, const __half* __restrict__ k,
                                                     const __half* __restrict__ v) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t w = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int H = L.n_kv_heads;
  if (w >= int64_t(total_tokens) * H) return;
  const int row = int(w / H), h = int(w % H);
  // both fp16 rows are loaded first: their addresses need no page, so the loads
  // overlap the page-table lookup below
  const int64_t src = (int64_t(row) * H + h) * D;
  const typename HalfVec<E>::T kraw = load_raw<E>(k + src, lane), vraw = load_raw<E>(v + src, lane);
  // sequence of this row: last i with b.s[i].c <= row (row offsets ascending)
  int lo = 0, hi = b.n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (b.s[mid].c <= row) lo = mid; else hi = mid - 1;
  }
  const SeqDesc sd = b.s[lo];
  const int pos = sd.a + (row - sd.c);
  const int lp = pos / L.page_tokens, r = pos % L.page_tokens;
  const int page = L.page_table[int64_t(sd.seq_id) * L.max_pages_per_seq + lp];
  if (page < 0 || page >= L.n_pages) {
    if (lane == 0) record_error(L.err, kErrBadPage);
    return;
  }
  uint8_t* blk = L.head_ptr(layer, page, h);
  float x[E], y[E];
  uint16_t bits[E], ybits[E];
  unpack_row<E>(kraw, x, bits);
  unpack_row<E>(vraw, y, ybits);
  store_row<E>(L.k_bits, x, bits, lane, blk + int64_t(r) * L.k_row,
               reinterpret_cast<__half*>(blk + L.k_scales_off + int64_t(r) * L.s_row));
  store_row<E>(L.v_bits, y, ybits, lane, blk + L.v_codes_off + int64_t(r) * L.v_row,
               reinterpret_cast<__half*>(blk + L.v_scales_off + int64_t(r) * L.s_row));
}

// Canonical export: one warp per (token, head) copies that row's code and
// scale bytes to [n_tok, Hkv, row] destinations.
__global__ void export_kernel(const Layout L, int layer, int seq_id, int64_t tok0, int64_t n_tok, uint8_t* kc,
                              uint8_t* ks, uint8_t* vc, uint8_t* vs) {
  const int lane = threadIdx.x & 31;
  const int64_t w = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int H = L.n_kv_heads;
  if (w >= n_tok * H) return;
  const int64_t t = w / H;
  const int h = int(w % H);
  const int64_t pos = tok0 + t;
  const int page = L.page_table[int64_t(seq_id) * L.max_pages_per_seq + pos / L.page_tokens];
  if (page < 0 || page >= L.n_pages) {
    if (lane == 0) record_error(L.err, kErrBadPage);
    return;
  }
  const int r = int(pos % L.page_tokens);
  const uint8_t* blk = L.head_ptr(layer, page, h);
  auto copy = [&](uint8_t* dst, const uint8_t* src, int n) {
    if (!dst) return;
    for (int i = lane; i < n; i += 32) dst[w * n + i] = src[i];
  };
  copy(kc, blk + int64_t(r) * L.k_row, L.k_row);
  copy(vc, blk + L.v_codes_off + int64_t(r) * L.v_row, L.v_row);
  if (L.k_bits != 16) copy(ks, blk + L.k_scales_off + int64_t(r) * L.s_row, L.s_row);
  if (L.v_bits != 16) copy(vs, blk + L.v_scales_off + int64_t(r) * L.s_row, L.s_row);
}

}  // namespace

cudaError_t launch_pt_update(int32_t* table, const PtUpdate& u, cudaStream_t s) {
  if (u.n == 0) return cudaSuccess;
  pt_update_kernel<<<(u.n + 255) / 256, 256, 0, s>>>(table, u);
  return cudaGetLastError();
}

cudaError_t launch_append(const Layout& L, int layer, const Batch& b, int total_tokens, const void* k, const void* v,
                          cudaStream_t s) {
  const int64_t warps = int64_t(total_tokens) * L.n_kv_heads;
  const unsigned grid = unsigned((warps + 7) / 8);
  if (L.head_dim == 128)
    append_kernel<128><<<grid, 256, 0, s>>>(L, layer, b, total_tokens, static_cast<const __half*>(k),
                                            static_cast<const __half*>(v));
  else
    append_kernel<64><<<grid, 256, 0, s>>>(L, layer, b, total_tokens, static_cast<const __half*>(k),
                                           static_cast<const __half*>(v));
  return cudaGetLastError();
}

cudaError_t launch_export(const Layout& L, int layer, int seq_id, int64_t tok0, int64_t n_tok, void* kc, void* ks,
                          void* vc, void* vs, cudaStream_t s) {
  const int64_t warps = n_tok * L.n_kv_heads;
  export_kernel<<<unsigned((warps + 7) / 8), 256, 0, s>>>(L, layer, seq_id, tok0, n_tok, static_cast<uint8_t*>(kc),
                                                          static_cast<uint8_t*>(ks), static_cast<uint8_t*>(vc),
                                                          static_cast<uint8_t*>(vs));
  return cudaGetLastError();
}

}  // namespace kvq
