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
// IEEE fp32 divide; the codes use round_code below, which equals roundf of the
// IEEE fp32 quotient x / d, so codes and scales are bit-exact across
// implementations.
//
// One thread quantises one 32-element block of a K or V row (see
// append_kernel); a warp's loads and stores are contiguous 16-byte accesses.
#include <cuda_fp16.h>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

__global__ void pt_update_kernel(int32_t* table, const __grid_constant__ PtUpdate u) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < u.n) table[u.idx[i]] = u.val[i];
}

// Code rounding without a divide and without integer conversions, for
// fp16-valued x and d != 0: c = clamp(roundf(fp32(x / d)), -cn, cp) as an exact
// small integer in a float.  With t = |x| / |d|, n = rint(|x| * fp32(1/|d|)) (one
// FMA against 1.5 * 2^23) is within 1 of floor(t + 1/2); the remainder
// e = |x| - n |d| is exact in fp32 (n |d| has at most 18 significant bits) and
// moves n up when e >= |d|/2 and down when e < -|d|/2, ties going away from
// zero; the sign of x / d is applied last, then the clamp.  For fp16 x and d
// the fp32 rounding of the quotient never moves it across a half-integer it did
// not sit on, so this is the same integer as roundf of the IEEE quotient
// (checked for every finite fp16 x against 3400 scales, both clamp ranges).
struct RoundCtx {
  float ad, ra, hd;   // |d|, fp32(1 / |d|), |d| / 2
};
__device__ __forceinline__ RoundCtx round_ctx(float d) {
  RoundCtx r;
  r.ad = fabsf(d);
  r.ra = __frcp_rn(r.ad);
  r.hd = 0.5f * r.ad;
  return r;
}
__device__ __forceinline__ float round_mag(float x, const RoundCtx& r) {
  const float ax = fabsf(x);
  float n = __fadd_rn(__fmaf_rn(ax, r.ra, 12582912.0f), -12582912.0f);
  const float e = __fmaf_rn(-n, r.ad, ax);
  if (e >= r.hd) n += 1.f;           // rare: two compares and predicated adds
  if (e < -r.hd) n -= 1.f;
  return n;
}
// 4-bit (d of either sign): the sign of x / d set on the magnitude with one bit
// operation, then the asymmetric clamp to [-8, 7].
__device__ __forceinline__ float round_code4(float x, const RoundCtx& r, uint32_t dbits) {
  const float n = round_mag(x, r);
  const float c = __uint_as_float(__float_as_uint(n) | ((__float_as_uint(x) ^ dbits) & 0x80000000u));
  return fmaxf(fminf(c, 7.f), -8.f);
}
// 8-bit: d > 0, symmetric clamp
__device__ __forceinline__ float round_code8(float x, const RoundCtx& r) {
  return copysignf(fminf(round_mag(x, r), 127.f), x);
}
// max(a, b, c) and min(a, b, c) in one instruction each
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// Low byte of an exact integer v in [-128, 255] held in a float (two's complement for v < 0).
__device__ __forceinline__ uint32_t float_int_bits(float v) { return __float_as_uint(v + 12582912.0f); }
// Bytes 0 of a, b, c, e -> one word.
__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t e) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, e, 0x0040), 0x5410);
}

// One thread quantises one 32-element block of one K or V row: it loads the
// block's 64 bytes with four 16-byte loads, takes the block max in registers
// (no shuffles, one scale and one reciprocal per block), rounds the 32 codes on
// the FMA pipe and writes them with 16-byte stores.  A warp covers the 32
// consecutive blocks of 32 / (D / 32) rows of K only or of V only (warps
// alternate), so its loads and stores stay contiguous and its lanes never
// diverge between the 8-bit and the 4-bit code paths.
__device__ __forceinline__ void load_block(const __half* src, float (&x)[32]) {
  const uint4* p = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 w = p[c];
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ws[i]));
      x[8 * c + 2 * i] = f.x;
      x[8 * c + 2 * i + 1] = f.y;
    }
  }
}

// 8-bit: d = fp16(fp32(amax / 127)), c = clamp(roundf(x / d), -127, 127).
__device__ __forceinline__ void quant8_block(const float (&x)[32], uint8_t* codes, __half* scale) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < 32; i += 2) a = fmax3(a, fabsf(x[i]), fabsf(x[i + 1]));
  const __half d = __float2half_rn(__fdiv_rn(a, 127.0f));
  const float df = __half2float(d);
  uint32_t w[8];
  if (df != 0.f) {
    const RoundCtx r = round_ctx(df);
#pragma unroll
    for (int k = 0; k < 8; ++k)
      w[k] = pack_low_bytes(float_int_bits(round_code8(x[4 * k], r)), float_int_bits(round_code8(x[4 * k + 1], r)),
                            float_int_bits(round_code8(x[4 * k + 2], r)), float_int_bits(round_code8(x[4 * k + 3], r)));
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) w[k] = 0u;
  }
  reinterpret_cast<uint4*>(codes)[0] = make_uint4(w[0], w[1], w[2], w[3]);
  reinterpret_cast<uint4*>(codes)[1] = make_uint4(w[4], w[5], w[6], w[7]);
  *scale = d;
}

// 4-bit: m = the largest-|x| element (lowest index on ties), d = fp16(m / -8),
// c = clamp(roundf(x / d), -8, 7), u = c + 8, byte i = u_i | u_{i+16} << 4.
__device__ __forceinline__ void quant4_block(const float (&x)[32], uint8_t* codes, __half* scale) {
  // the largest-|x| element is max(x) or min(x); only when max(x) == -min(x) (a +- tie, or a zero
  // block) does the index decide, by a scan in which the lowest index wins
  float mx = x[0], mn = x[0];
#pragma unroll
  for (int i = 1; i < 31; i += 2) {
    mx = fmax3(mx, x[i], x[i + 1]);
    mn = fmin3(mn, x[i], x[i + 1]);
  }
  mx = fmaxf(mx, x[31]);
  mn = fminf(mn, x[31]);
  float m = mx > -mn ? mx : mn;
  if (mx == -mn) {
    m = x[0];
#pragma unroll                                               // registers only: no dynamic index into x
    for (int i = 1; i < 32; ++i)
      if (fabsf(x[i]) > fabsf(m)) m = x[i];                // strict: the lowest index wins ties
  }
  const __half d = __float2half_rn(m * -0.125f);            // m / -8, exact in fp32
  const float df = __half2float(d);
  uint32_t w[4];
  if (df != 0.f) {
    const RoundCtx r = round_ctx(df);
    const uint32_t dbits = __float_as_uint(df);
    uint32_t by[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      // u_j + 16 u_{j+16} = c_j + 16 c_{j+16} + 136, an exact integer in [0, 255]
      const float c0 = round_code4(x[j], r, dbits), c1 = round_code4(x[j + 16], r, dbits);
      by[j] = float_int_bits(__fmaf_rn(c1, 16.f, c0) + 136.f);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = pack_low_bytes(by[4 * k], by[4 * k + 1], by[4 * k + 2], by[4 * k + 3]);
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = 0x88888888u;         // all codes 0: u = 8 in both nibbles
  }
  reinterpret_cast<uint4*>(codes)[0] = make_uint4(w[0], w[1], w[2], w[3]);
  *scale = d;
}

template <int D>
__global__ void __launch_bounds__(256) append_kernel(const Layout L, int layer, const __grid_constant__ Batch b,
                                                     int total_tokens, const __half* __restrict__ k,
                                                     const __half* __restrict__ v) {
  constexpr int NB = D / 32;                       // blocks per row
  constexpr int RPW = 32 / NB;                     // rows per warp
  const int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int H = L.n_kv_heads;
  const int64_t n_rows = int64_t(total_tokens) * H;
  const int64_t gw = t >> 5;                       // warp pair gw / 2 covers rows [RPW (gw / 2), + RPW)
  const int lane = int(t & 31);
  const int kv = int(gw & 1), blk = lane % NB;
  const int64_t rr64 = (gw >> 1) * RPW + lane / NB;
  if (rr64 >= n_rows) return;
  const int rr = int(rr64);                        // (token, head) row; < 2^31 for any input that fits in HBM
  const __half* src = (kv ? v : k) + int64_t(rr) * D + blk * 32;
  float x[32];
  load_block(src, x);                              // issued before the page lookup it does not need
  const int row = rr / H, h = rr % H;
  // sequence of this row: last s with b.s[s].c <= row (row offsets ascending)
  int lo = 0, hi = b.n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (b.s[mid].c <= row) lo = mid; else hi = mid - 1;
  }
  const SeqDesc sd = b.s[lo];
  const int pos = sd.a + (row - sd.c);
  const int page = L.page_table[int64_t(sd.seq_id) * L.max_pages_per_seq + pos / L.page_tokens];
  if (page < 0 || page >= L.n_pages) {
    record_error(L.err, kErrBadPage);
    return;
  }
  const int r = pos % L.page_tokens;
  uint8_t* hb = L.head_ptr(layer, page, h);
  const int bitsw = kv ? L.v_bits : L.k_bits;
  uint8_t* codes_row = hb + (kv ? L.v_codes_off : 0) + int64_t(r) * (kv ? L.v_row : L.k_row);
  __half* scales_row = reinterpret_cast<__half*>(hb + (kv ? L.v_scales_off : L.k_scales_off) + int64_t(r) * L.s_row);
  if (bitsw == 8) {
    quant8_block(x, codes_row + blk * 32, scales_row + blk);
  } else if (bitsw == 4) {
    quant4_block(x, codes_row + blk * 16, scales_row + blk);
  } else {
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    uint4* d4 = reinterpret_cast<uint4*>(codes_row + blk * 64);
#pragma unroll
    for (int c = 0; c < 4; ++c) d4[c] = s4[c];
  }
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
  const int64_t rows = int64_t(total_tokens) * L.n_kv_heads, rpw = 32 / (L.head_dim / 32);
  const int64_t threads = (rows + rpw - 1) / rpw * 64;            // one K warp and one V warp per rpw rows
  const unsigned grid = unsigned((threads + 255) / 256);
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
