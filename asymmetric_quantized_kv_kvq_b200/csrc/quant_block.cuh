// Quantisation of one 32-element block (8-bit or 4-bit codes and one fp16
// scale), shared by the append kernel and the decode kernel's fused append, so
// both write the same bits.
//
// Format (KVSplit page, "KVSplit - contexto 2 a 3 vezes mais longo em Apple
// Silicon", section "Uso de memoria conforme o comprimento da sequencia":
// 32-element blocks with one fp16 scale, 34 B per 8-bit block and 18 B per
// 4-bit block), with this library's reading of the rounding: 8-bit
// d = fp16(fp32(amax / 127)), c = clamp(roundf(x / d), -127, 127); 4-bit
// d = fp16(m / -8) with m the largest-|x| element (lowest index on ties),
// c = clamp(roundf(x / d), -8, 7), nibble u = c + 8, byte i = u_i | u_{i+16} << 4.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

namespace kvq {

// Code rounding without a divide and without integer conversions, for
// fp16-valued x and d != 0: c = clamp(roundf(fp32(x / d)), -cn, cp) as an exact
// small integer in a float.  With t = |x| / |d| <= 128.5 and ra = 1 / |d| rounded
// up to fp32, round(t) (halves away from zero) is floor(|x| ra + 1/2) with that FMA
// rounded down to fp32.  ra >= 1 / |d| keeps the exact |x| ra + 1/2 at or above
// t + 1/2, so an exact tie t = k + 1/2 reaches k + 1; |x| ra exceeds t by at most
// t 2^-23 < 2^-16, and a quotient of two fp16 values that is not a half-integer
// lies at least 2^-15 from one, so neither that excess nor the downward rounding
// of the FMA (less than one fp32 ulp, 2^-16 below 256) moves the sum across an
// integer that t + 1/2 does not reach.  The floor is one more addition, of
// 1.5 * 2^23 rounded down, which leaves M + n (M = 1.5 * 2^23).  The sign of x / d
// is applied afterwards, then the clamp.  This is the same integer as roundf of the
// IEEE fp32 quotient for every fp16 magnitude against every positive fp16 scale
// with t <= 128.5 (checked exhaustively: 7.0e8 pairs).
constexpr float kRoundBias = 12582912.0f;   // M = 1.5 * 2^23: M + v holds the integer v in its low bits
struct RoundCtx {
  float ra;   // 1 / |d|, rounded up to fp32
};
__device__ __forceinline__ RoundCtx round_ctx(float d) {
  RoundCtx r;
  r.ra = __frcp_ru(fabsf(d));
  return r;
}
// M + round(|x| / |d|)
__device__ __forceinline__ float round_mag_biased(float x, const RoundCtx& r) {
  return __fadd_rd(__fmaf_rd(fabsf(x), r.ra, 0.5f), kRoundBias);
}
__device__ __forceinline__ float round_mag(float x, const RoundCtx& r) { return round_mag_biased(x, r) - kRoundBias; }
// The clamps only matter for subnormal scales.  With a normal fp16 scale (|d| >= 2^-14) the
// largest |x| / |d| of a block is below 127.06 for 8 bits (d = fp16(amax / 127)) and exactly 8
// for 4 bits (d = m / -8 is exact), so no 8-bit code passes 127 and no 4-bit code falls below -8;
// a subnormal scale rounds with a coarser step (up to 190 and 11).  Checked for every fp16 amax
// and m.
constexpr float kMinNormalHalf = 6.103515625e-05f;   // 2^-14
// 4-bit (d of either sign): the sign of x / d set on the magnitude with one bit
// operation, then the asymmetric clamp to [-8, 7] (LOW: the lower bound too).
template <bool LOW = true>
__device__ __forceinline__ float round_code4(float x, const RoundCtx& r, uint32_t dbits) {
  const float n = round_mag(x, r);
  const float c = __uint_as_float(__float_as_uint(n) | ((__float_as_uint(x) ^ dbits) & 0x80000000u));
  return LOW ? fmaxf(fminf(c, 7.f), -8.f) : fminf(c, 7.f);
}
// 8-bit: d > 0, symmetric clamp (applied to M + n, which is exact; CLAMP = false for a normal d)
template <bool CLAMP = true>
__device__ __forceinline__ float round_code8(float x, const RoundCtx& r) {
  if constexpr (CLAMP) return copysignf(fminf(round_mag_biased(x, r), kRoundBias + 127.f) - kRoundBias, x);
  return copysignf(round_mag(x, r), x);
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
__device__ __forceinline__ uint32_t float_int_bits(float v) { return __float_as_uint(v + kRoundBias); }
// Bytes 0 of a, b, c, e -> one word.
__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t e) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, e, 0x0040), 0x5410);
}

// The block's 32 fp16 values (64 bytes, 16-byte aligned) as fp32.
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

// 8-bit: d = fp16(fp32(amax / 127)), c = clamp(roundf(x / d), -127, 127).  The codes as 8 words
// (byte i of the block in byte i % 4 of word i / 4); returns d.
__device__ __forceinline__ __half quant8_words(const float (&x)[32], uint32_t (&w)[8]) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < 32; i += 2) a = fmax3(a, fabsf(x[i]), fabsf(x[i + 1]));
  const __half d = __float2half_rn(__fdiv_rn(a, 127.0f));
  const float df = __half2float(d);
  if (df >= kMinNormalHalf) {
    const RoundCtx r = round_ctx(df);
#pragma unroll
    for (int k = 0; k < 8; ++k)
      w[k] = pack_low_bytes(float_int_bits(round_code8<false>(x[4 * k], r)),
                            float_int_bits(round_code8<false>(x[4 * k + 1], r)),
                            float_int_bits(round_code8<false>(x[4 * k + 2], r)),
                            float_int_bits(round_code8<false>(x[4 * k + 3], r)));
  } else if (df != 0.f) {
    const RoundCtx r = round_ctx(df);
#pragma unroll
    for (int k = 0; k < 8; ++k)
      w[k] = pack_low_bytes(float_int_bits(round_code8(x[4 * k], r)), float_int_bits(round_code8(x[4 * k + 1], r)),
                            float_int_bits(round_code8(x[4 * k + 2], r)), float_int_bits(round_code8(x[4 * k + 3], r)));
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) w[k] = 0u;
  }
  return d;
}
__device__ __forceinline__ void quant8_block(const float (&x)[32], uint8_t* codes, __half* scale) {
  uint32_t w[8];
  const __half d = quant8_words(x, w);
  reinterpret_cast<uint4*>(codes)[0] = make_uint4(w[0], w[1], w[2], w[3]);
  reinterpret_cast<uint4*>(codes)[1] = make_uint4(w[4], w[5], w[6], w[7]);
  *scale = d;
}

// 4-bit: m = the largest-|x| element (lowest index on ties), d = fp16(m / -8),
// c = clamp(roundf(x / d), -8, 7), u = c + 8, byte i = u_i | u_{i+16} << 4.  The 16 bytes as 4
// words; returns d.
__device__ __forceinline__ __half quant4_words(const float (&x)[32], uint32_t (&w)[4]) {
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
  if (df != 0.f) {
    const RoundCtx r = round_ctx(df);
    const uint32_t dbits = __float_as_uint(df);
    uint32_t by[16];
    if (fabsf(df) >= kMinNormalHalf) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        // u_j + 16 u_{j+16} = c_j + 16 c_{j+16} + 136, an exact integer in [0, 255]
        const float c0 = round_code4<false>(x[j], r, dbits), c1 = round_code4<false>(x[j + 16], r, dbits);
        by[j] = __float_as_uint(__fmaf_rn(c1, 16.f, c0) + (kRoundBias + 136.f));   // exact integers throughout
      }
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float c0 = round_code4(x[j], r, dbits), c1 = round_code4(x[j + 16], r, dbits);
        by[j] = __float_as_uint(__fmaf_rn(c1, 16.f, c0) + (kRoundBias + 136.f));
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = pack_low_bytes(by[4 * k], by[4 * k + 1], by[4 * k + 2], by[4 * k + 3]);
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = 0x88888888u;         // all codes 0: u = 8 in both nibbles
  }
  return d;
}
__device__ __forceinline__ void quant4_block(const float (&x)[32], uint8_t* codes, __half* scale) {
  uint32_t w[4];
  const __half d = quant4_words(x, w);
  reinterpret_cast<uint4*>(codes)[0] = make_uint4(w[0], w[1], w[2], w[3]);
  *scale = d;
}

}  // namespace kvq
