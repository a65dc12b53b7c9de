// Split-KV flash-decoding over a quantized paged cache (8- or 4-bit keys and
// values) on CUDA cores, sm_100a.
//
// Computes, for each sequence b, KV head h and query head g of its GQA group,
//   o = sum_t p_t v^_t / sum_t p_t,  p_t = 2^(s_t - m),  s_t = (sigma log2 e) q . k^_t
// over cache positions t < len: exact softmax attention read "through the
// flash-attention path" (KVSplit page, "KVSplit - contexto 2 a 3 vezes mais
// longo em Apple Silicon", section "Exemplos de uso e opcoes de CLI"), with
// k^ = d_k c_k and v^ = d_v c_v dequantised in registers from the stored codes.
//
// Work decomposition: the flat list of (sequence, KV head, chunk) units is cut
// into equal contiguous ranges, one per CTA ("stream-K"), so every SM streams
// the same number of bytes whatever the length mix.  A CTA writes one partial
// (O, m, l) per item it touches; an item inside one CTA is normalised and
// written directly, the partials of an item spread over several CTAs are merged
// by the last of those CTAs to finish (a counter per item; no CTA ever waits
// for another): o = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.
//
// CTA = 8 consumer warps + 1 producer warp:
//  - producer: streams each chunk's K codes, K scales, V codes and V scales
//    (four contiguous ranges of one page's head block) into a ring of shared-
//    memory stages with 1-D TMA bulk copies; with a fused append it first
//    quantises the new token's K and V row into the page (same block
//    quantiser as the append kernel), for the one chunk that holds it;
//  - a stage holds one chunk: 256 tokens on pages of a multiple of 256 tokens
//    when three such stages fit and the step gives every CTA at least two of
//    them (fewer, larger stages halve the per-stage control work per token),
//    else 128 (the stage size is the template parameter CT); its tokens are
//    split into partitions, one per consumer warp (at 8 query heads per KV
//    head two warps share a partition, 4 heads each); a
//    warp keeps its own running softmax (m, l per head) and accumulators O, so
//    consumer warps never wait for one another inside an item;
//  - a warp is software-pipelined by one stage: the score passes of stage k and
//    the value passes of stage k - 1 form one straight-line block, so the long
//    dependency chains of the scores (shared-memory loads, dp4a chains,
//    shuffles) are filled with the independent FMAs of the values;
//  - scores: a lane owns one 32-element key block of one token and holds the
//    query as two int8 digits per element (15 bits: q ~= s (256 hi + lo),
//    s = max|q| / 32512 per head) for the warp's heads; dp4a on the stored key
//    codes (4-bit codes unpacked to bytes, their +8 offset folded into the
//    accumulator's start) gives exact integer dot products, then one int->float
//    conversion and one multiply by d_k per (token, block, head); a
//    reduce-scatter over the token's lanes (query register slots permuted per
//    lane, so that it needs no selects) leaves each lane its own heads' scores;
//  - online softmax with a lazily moved maximum (moved only when a score passes
//    it by 2^8); p' = p d_v per (token, value block, head) goes to a
//    warp-private buffer;
//  - values: a lane owns E elements of one token; each code is converted to
//    fp32 exactly once (a byte placed in the mantissa of 2^23, then one
//    subtraction per pair) and feeds all of the warp's heads; the FMAs are
//    packed two elements at a time (fma.rn.f32x2).
// Every wait is bounded: on expiry the kernel records an error code, raises a
// CTA-wide abort flag, drains its own copies and returns.
#pragma once

#include <cuda_fp16.h>

#include "decode_common.cuh"
#include "kvq_internal.cuh"
#include "quant_block.cuh"
#include "sm100_util.cuh"

namespace kvq {

struct DecodeQArgs {
  Layout L;
  int layer;
  int n_q_heads;
  const __half* q;
  __half* out;
  const __half* k_new;   // fused append: fp16 [B, Hkv, D] K / V of position len - 1 (nullptr: none)
  const __half* v_new;
  float* ws_o;           // [slots][G][D]
  float* ws_ml;          // [slots][G][2]
  int32_t* counters;     // [items], zero between launches
  float scale_log2;      // sigma * log2(e)
  int64_t total_chunks;
  int64_t cpc;           // chunks per CTA
  int chunk;             // tokens per work chunk (divides page_tokens, <= C)
};

template <int KB, int VB, int D, int G, int CT>
struct QDec {
  static constexpr int C = CT;                       // tokens per stage (128, or 256 on 256-token pages)
  static constexpr int NB = D / 32;                  // 32-element blocks per row
  static constexpr int GW = G > 4 ? 4 : G;           // query heads per consumer warp
  static constexpr int NHG = G / GW;                 // warps sharing one partition (head groups)
  static constexpr int NW = 8;                       // consumer warps
  static constexpr int NPART = NW / NHG;             // token partitions of a stage
  static constexpr int W = C / NPART;                // tokens per partition
  static constexpr int LPT = NB;                     // score lanes per token: one key block each
  static constexpr int TPP = 32 / LPT;               // tokens per score pass
  static constexpr int NPASS = W / TPP;              // score passes per stage
  static constexpr int NF = GW > LPT ? GW / LPT : 1; // heads a score lane owns after the reduce-scatter
  static constexpr int E = 32 / GW;                  // value elements per lane (E x GW = 32 accumulators)
  static constexpr int LPV = D / E;                  // value lanes per token
  static constexpr int TPV = 32 / LPV;               // tokens per value pass
  static constexpr int NPV = W / TPV;                // value passes per stage
  static constexpr int NT = (NW + 4) * 32;
  static constexpr int REG_L = 168, REG_C = 216, REG_P = 72;
  // setmaxnreg moves registers between warpgroups of this block only: the split must fit in what
  // the block was launched with, or a warpgroup's increase would never be granted
  static_assert(NW * 32 * REG_C + 4 * 32 * REG_P <= NT * REG_L, "register split exceeds the launch allocation");
  static constexpr int K_ROW = KB == 8 ? D : D / 2;
  static constexpr int V_ROW = VB == 8 ? D : D / 2;
  static constexpr int KBLK = K_ROW / NB;            // code bytes of one key block
  static constexpr int S_ROW = NB * 2;               // fp16 scales per row
  static constexpr int TOK_BYTES = K_ROW + S_ROW + V_ROW + S_ROW;
  static constexpr int BPL = VB == 8 ? E : E / 2;    // value code bytes per lane
  static constexpr int VBLK = VB == 8 ? 32 : 16;     // code bytes per value block
  static constexpr int OFF_KS = C * K_ROW;
  static constexpr int OFF_VC = OFF_KS + C * S_ROW;
  static constexpr int OFF_VS = OFF_VC + C * V_ROW;
  static constexpr int STAGE = OFF_VS + C * S_ROW;
  // per warp: p' [W][NB][GW] during the stages; at an item's start the query digits of the
  // warp's heads (hi and lo words [GW][D / 4] each, 4-bit-key corrections [GW][NB], max|q| [GW])
  static constexpr int QD_BYTES = GW * D * 2 + GW * NB * 4 + GW * 4;
  static constexpr int PB_WARP = ((W * NB * GW * 4 > QD_BYTES ? W * NB * GW * 4 : QD_BYTES) + 15) / 16 * 16;
  static constexpr int PBUF = NW * PB_WARP;
  // partial O per partition; the last CTA of a split item reuses it for one weight per CTA and head
  static constexpr int MRG_O_F = NPART * G * D > (kMaxDecodeCtas + 1) * G ? NPART * G * D : (kMaxDecodeCtas + 1) * G;
  static constexpr int MRG_O = (MRG_O_F * 4 + 15) / 16 * 16;
  static constexpr int MRG_ML = (NPART * G * 2 * 4 + 15) / 16 * 16;
  static constexpr int QBUF = NW * GW * D * 2;       // each warp's query rows (fp16)
  static constexpr int BARS = 256;
  static constexpr int FIXED = PBUF + MRG_O + MRG_ML + QBUF + BARS;
  static constexpr int SMEM_LIMIT = 227 * 1024;
  static constexpr int S_FIT = (SMEM_LIMIT - FIXED) / STAGE;
  static constexpr int S = S_FIT > 8 ? 8 : S_FIT;    // stages in the ring
  static constexpr int SMEM = S * STAGE + FIXED;
  static constexpr bool FITS = S_FIT >= 3;           // three stages of C tokens fit (checked by the kernel)
  static_assert(W % TPP == 0 && NPASS >= 1 && W % TPV == 0 && NPV >= 1, "tiling");
  static_assert(BPL % 4 == 0 && BPL <= VBLK, "a value lane's codes lie in one value block");
  static_assert(STAGE % 16 == 0 && OFF_KS % 16 == 0 && OFF_VC % 16 == 0 && OFF_VS % 16 == 0, "alignment");
  static_assert(PBUF % 16 == 0 && QBUF % 16 == 0, "alignment");
  static_assert((2 * S + 6) * 8 + 8 <= BARS, "barrier area");
};

// ---- the permuted reduce-scatter of the score lanes ------------------------------
// Slot j of lane L holds query head j ^ f(L), where f maps the lane's block
// bits (high to low) onto the head bits (high to low).  Then at every exchange
// level each lane keeps its low slots and adds the partner's high slots, which
// hold the same heads: no lane-dependent selects.
template <int LPT, int GW>
__host__ __device__ constexpr int rs_map(int blk) {
  int f = 0, lb = LPT / 2, hb = GW / 2;
  while (lb >= 1 && hb >= 1) {
    if (blk & lb) f |= hb;
    lb >>= 1;
    hb >>= 1;
  }
  return f;
}
// The block lane (within its token) that owns head g after the reduce-scatter; slot g % NF.
template <int LPT, int GW>
__host__ __device__ constexpr int rs_lane_of(int g) {
  int l = 0, lb = LPT / 2, hb = GW / 2;
  while (lb >= 1 && hb >= 1) {
    if (g & hb) l |= lb;
    lb >>= 1;
    hb >>= 1;
  }
  return l;
}
template <int LPT, int GW>
__device__ __forceinline__ void reduce_scatter_perm(float (&v)[GW]) {
  int n = GW;
#pragma unroll
  for (int o = LPT / 2; o >= 1; o >>= 1) {
    if (n > 1) {
#pragma unroll
      for (int j = 0; j < GW / 2; ++j)
        if (j < n / 2) v[j] += __shfl_xor_sync(0xffffffffu, v[j + n / 2], o);
      n >>= 1;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
  }
}

// 2^x on the SFU (ex2.approx.ftz: results below 2^-126 flush to 0, which a
// softmax weight that small never notices; 2^-inf = 0).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---- stored codes -------------------------------------------------------------
// A score lane reads the codes of its key block: 8-bit codes as two 16-byte
// chunks, chunk c ^ x at load step c (x depends on the lane's token, so that
// the 16-byte loads of a warp spread over all shared-memory banks); 4-bit codes
// as one 16-byte chunk, unpacked to one byte per code (0..15: words 0..3 the low
// nibbles, 4..7 the high nibbles).  Byte e of word w is then element
// kq_elem(w, e, x) of the block.
template <int KB>
__host__ __device__ constexpr int kq_elem(int w, int e, int x) {
  if (KB == 8) return 16 * ((w >> 2) ^ x) + 4 * (w & 3) + e;
  return w < 4 ? 4 * w + e : 16 + 4 * (w - 4) + e;   // byte j of a 4-bit block: elements j (low), j + 16 (high)
}
// Chunk rotation of a score lane of token tl: rows 128 bytes apart share banks.
template <int KB, int D>
__device__ __forceinline__ int kq_rot(int tl) {
  return KB == 8 ? ((tl * D) / 128) & 1 : 0;
}

// Value lane's codes of one 4-byte word -> 8 exact values (u - 8 or c) as fp32,
// in the order: 4-bit: low nibbles of bytes 0..3, then high nibbles;
// 8-bit: bytes 0..3 (and the next word's bytes are the next call).
__device__ __forceinline__ void cvt_v4_word(uint32_t w, float (&f)[8]) {
  const uint32_t lo = w & 0x0F0F0F0Fu, hi = w & 0xF0F0F0F0u;
  const float2 blo = make_float2(-(kTwo23 + 8.f), -(kTwo23 + 8.f));
  // high nibble byte reads 2^23 + 16 u: (x / 16) - (2^19 + 8) = u - 8 exactly
  const float2 m16 = make_float2(0.0625f, 0.0625f), bhi = make_float2(-(524288.f + 8.f), -(524288.f + 8.f));
  float2 a = fadd2(bytes01_f(lo), blo), b = fadd2(bytes23_f(lo), blo);
  float2 c = ffma2(bytes01_f(hi), m16, bhi), d = ffma2(bytes23_f(hi), m16, bhi);
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
  f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}
__device__ __forceinline__ void cvt_v8_word(uint32_t w, float (&f)[4]) {
  const uint32_t u = w ^ 0x80808080u;
  const float2 off = make_float2(-(kTwo23 + 128.f), -(kTwo23 + 128.f));
  const float2 a = fadd2(bytes01_f(u), off), b = fadd2(bytes23_f(u), off);
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
}

// Head-dim element of value i (0 .. E-1) of the value lane with slot `sl`.
template <int VB, int E>
__host__ __device__ constexpr int v_elem_of(int sl, int i) {
  if (VB == 8) return sl * E + i;
  const int o = sl * (E / 2) + 4 * (i / 8) + (i % 4);   // byte of the value
  return 32 * (o / 16) + (o % 16) + ((i % 8) >= 4 ? 16 : 0);
}

// Shared-memory carve-up and barriers of one CTA.
template <int KB, int VB, int D, int G, int CT>
struct QDecSmem {
  using T = QDec<KB, VB, D, G, CT>;
  uint8_t* stages;
  float* pbuf;          // [warp][PB_WARP bytes]  p' = p d_v [W][NB][GW], or the query digits
  float* mrg_o;         // [part][G][D]
  float* mrg_ml;        // [part][G][2]
  __half* qbuf;         // [warp][GW][D]
  uint32_t full0, empty0, mfull, mfree, mws, mlast, mcomb, abar;
  volatile int* abort_flag;
  volatile int* last_flag;

  __device__ __forceinline__ explicit QDecSmem(uint8_t* smem) {
    stages = smem;
    uint8_t* p = smem + T::S * T::STAGE;
    pbuf = reinterpret_cast<float*>(p);
    mrg_o = reinterpret_cast<float*>(p + T::PBUF);
    mrg_ml = reinterpret_cast<float*>(p + T::PBUF + T::MRG_O);
    qbuf = reinterpret_cast<__half*>(p + T::PBUF + T::MRG_O + T::MRG_ML);
    uint64_t* bars = reinterpret_cast<uint64_t*>(p + T::FIXED - T::BARS);
    full0 = smem_u32(bars);                              // [S]: stage filled (tx bytes)
    empty0 = full0 + 8 * T::S;                           // [S]: stage released by every consumer warp
    mfull = empty0 + 8 * T::S;                           // merge data written
    mfree = mfull + 8;                                   // merge data consumed
    mws = mfull + 16;                                    // partial written to the workspace
    mlast = mfull + 24;                                  // "last CTA of the item" decided
    mcomb = mfull + 32;                                  // merge weights of a split item written
    abar = mfull + 40;                                   // fused append: the chunk's copies landed
    abort_flag = reinterpret_cast<volatile int*>(bars + 2 * T::S + 6);
    last_flag = abort_flag + 1;
  }
};

// End of an item segment, run by every consumer warp after it published its
// (m, l) and O into the merge area: combine the partitions, write the output
// (item inside this CTA) or this CTA's partial, and let the last CTA of a
// split item merge all partials.  Returns false when a wait gave up.
template <int KB, int VB, int D, int G, int CT>
__device__ __forceinline__ bool merge_item(const DecodeQArgs& a, const QDecSmem<KB, VB, D, G, CT>& sm,
                                           const DecodeSeg& sg, const SeqDesc& sd, uint32_t& itm,
                                           uint32_t& itw, uint32_t& itc) {
  using T = QDec<KB, VB, D, G, CT>;
  constexpr int NPART = T::NPART, NW = T::NW;
  const int lane = threadIdx.x & 31;
  const int H = a.L.n_kv_heads;
  const int item = sg.bi * H + sg.h;
  __syncwarp();
  mbar_arrive_if(sm.mfull, lane == 0);
  if (!mbar_wait(sm.mfull, itm & 1, sm.abort_flag, a.L.wait_ns)) {
    if (lane == 0) record_error(a.L.err, kErrWaitTimeout | 6);
    *sm.abort_flag = 1;
    return false;
  }
  const int nch = sd.c;
  const int64_t off = int64_t(sd.b) + int64_t(sg.h) * nch;
  const int64_t c0 = off / a.cpc, c1 = (off + nch - 1) / a.cpc;
  const int ct = threadIdx.x;                          // consumer threads are 0 .. NW * 32 - 1
  for (int e = ct; e < G * D; e += NW * 32) {
    const int g = e / D, d = e % D;
    float M = -INFINITY;
#pragma unroll
    for (int pt = 0; pt < NPART; ++pt) M = fmaxf(M, sm.mrg_ml[(pt * G + g) * 2]);
    float acc = 0.f, L = 0.f;
#pragma unroll
    for (int pt = 0; pt < NPART; ++pt) {
      const float f = exp2f(sm.mrg_ml[(pt * G + g) * 2] - M);   // 0 for a partition without tokens
      acc = fmaf(f, sm.mrg_o[(pt * G + g) * D + d], acc);
      L = fmaf(f, sm.mrg_ml[(pt * G + g) * 2 + 1], L);
    }
    if (c0 == c1) {
      a.out[(int64_t(sg.bi) * a.n_q_heads + sg.h * G + g) * D + d] = __float2half_rn(acc / L);
    } else {
      const int64_t slot = int64_t(blockIdx.x) + item;
      a.ws_o[(slot * G + g) * D + d] = acc;
      if (d == 0) {
        a.ws_ml[(slot * G + g) * 2] = M;
        a.ws_ml[(slot * G + g) * 2 + 1] = L;
      }
    }
  }
  if (c0 != c1) {
    // the last CTA of the item to finish merges every CTA's partial (fixed slot order)
    __threadfence();
    __syncwarp();
    mbar_arrive_if(sm.mws, lane == 0);
    if (ct == 0) {
      const bool ok = mbar_wait(sm.mws, itw & 1, sm.abort_flag, a.L.wait_ns);
      int last = 0;
      if (ok) {
        __threadfence();
        const int old = atomicAdd(a.counters + item, 1);
        last = old == int(c1 - c0);
        if (last) a.counters[item] = 0;                // ready for the next launch
      } else {
        record_error(a.L.err, kErrWaitTimeout | 7);
        *sm.abort_flag = 1;
      }
      *sm.last_flag = last;
      mbar_arrive(sm.mlast);
    }
    if (!mbar_wait(sm.mlast, itw & 1, sm.abort_flag, a.L.wait_ns)) {
      if (lane == 0) record_error(a.L.err, kErrWaitTimeout | 8);
      *sm.abort_flag = 1;
      return false;
    }
    ++itw;
    if (*sm.last_flag) {
      __threadfence();
      const int n = int(c1 - c0 + 1);                  // <= grid size <= kMaxDecodeCtas
      // weights 2^(m_i - M) of every partial slot i and 1 / L per head, one warp per head: the
      // (m, l) pairs of all slots are loaded at once (a lane holds slots lane + 32 q), into the
      // merge area, which this CTA's own merge no longer reads
      float* wts = sm.mrg_o;                             // [n][G]
      float* linv = sm.mrg_o + n * G;                    // [G]
      constexpr int QS = kMaxDecodeCtas / 32;
      for (int g = ct >> 5; g < G; g += NW) {
        const float2* ml = reinterpret_cast<const float2*>(a.ws_ml) + (c0 + item) * G + g;   // slot i: ml[G i]
        float2 v[QS];
        float M = -INFINITY;
#pragma unroll
        for (int q = 0; q < QS; ++q) {
          const int i = lane + 32 * q;
          v[q] = i < n ? __ldcg(ml + int64_t(G) * i) : make_float2(-INFINITY, 0.f);
          M = fmaxf(M, v[q].x);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float L = 0.f;
#pragma unroll
        for (int q = 0; q < QS; ++q) {
          const int i = lane + 32 * q;
          if (i < n) {
            const float w = exp2f(v[q].x - M);         // 0 for a slot without tokens
            wts[i * G + g] = w;
            L = fmaf(w, v[q].y, L);
          }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
        if (lane == 0) linv[g] = 1.f / L;
      }
      __syncwarp();
      mbar_arrive_if(sm.mcomb, lane == 0);
      if (!mbar_wait(sm.mcomb, itc & 1, sm.abort_flag, a.L.wait_ns)) {
        if (lane == 0) record_error(a.L.err, kErrWaitTimeout | 9);
        *sm.abort_flag = 1;
        return false;
      }
      ++itc;
      // every output element: the weighted sum of its slots.  A thread takes 4 consecutive
      // elements (16-byte loads) and every SG-th slot, loads up to 16 slots at once, and the SG
      // threads of a column (adjacent lanes) add their sums in a fixed order
      constexpr int NCOL = G * D / 4;
      constexpr int SG = NCOL >= NW * 32 ? 1 : NW * 32 / NCOL;
      static_assert(NCOL * SG == NW * 32 || SG == 1, "one column per thread");
      for (int cb = ct / SG; cb < NCOL; cb += NW * 32 / SG) {
        const int sgi = ct % SG;
        const int g = (cb * 4) / D, d0 = (cb * 4) % D;
        const float4* o0 = reinterpret_cast<const float4*>(a.ws_o + ((c0 + item) * G + g) * D + d0);   // slot i: o0[NCOL i]
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int i0 = sgi; i0 < n; i0 += 16 * SG) {
          float4 t[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const int i = i0 + q * SG;
            t[q] = i < n ? __ldcg(o0 + int64_t(NCOL) * i) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const int i = i0 + q * SG;
            const float wgt = i < n ? wts[i * G + g] : 0.f;
            acc.x = fmaf(wgt, t[q].x, acc.x);
            acc.y = fmaf(wgt, t[q].y, acc.y);
            acc.z = fmaf(wgt, t[q].z, acc.z);
            acc.w = fmaf(wgt, t[q].w, acc.w);
          }
        }
#pragma unroll
        for (int o = 1; o < SG; o <<= 1) {
          acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o);
          acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o);
          acc.z += __shfl_xor_sync(0xffffffffu, acc.z, o);
          acc.w += __shfl_xor_sync(0xffffffffu, acc.w, o);
        }
        if (sgi == 0) {
          const float li = linv[g];
          __half2* dst = reinterpret_cast<__half2*>(a.out + (int64_t(sg.bi) * a.n_q_heads + sg.h * G + g) * D + d0);
          dst[0] = __floats2half2_rn(acc.x * li, acc.y * li);
          dst[1] = __floats2half2_rn(acc.z * li, acc.w * li);
        }
      }
    }
  }
  __syncwarp();
  mbar_arrive_if(sm.mfree, lane == 0);
  ++itm;
  return true;
}

// Page of the chunk at flat position xl of a CTA range ending at x1 (-1 outside it or for a chunk
// that holds no tokens).
__device__ __forceinline__ int chunk_page(const DecodeQArgs& a, const Batch& b, int64_t xl, int64_t x1) {
  if (xl >= x1) return -1;
  const DecodeSeg gl = decode_find_seg(b, xl, x1);
  if (gl.n <= 0) return -1;
  const SeqDesc dl = b.s[gl.bi];
  const int t0 = dl.lo / a.chunk * a.chunk + gl.k0 * a.chunk;
  return a.L.page_table[int64_t(dl.seq_id) * a.L.max_pages_per_seq + page_slot(t0 / a.L.page_tokens, dl.ring)];
}

// Fused append, quantised by the whole producer warp: the row's 2 NB blocks (K blocks, then V
// blocks), LB lanes per block, EQ consecutive elements per lane.  Same arithmetic as the block
// quantiser of the append kernel, element for element, so the bytes are the same.
template <int D>
struct NewRow {
  static constexpr int NB = D / 32, LB = 32 / (2 * NB), EQ = 32 / LB;   // D 128: 4 lanes x 8; D 64: 8 x 4
  uint32_t raw[EQ / 2];                                                 // the lane's EQ fp16 values
};
template <int D>
__device__ __forceinline__ void new_row_load(NewRow<D>& nr, const DecodeQArgs& a, int bi, int h, int lane) {
  using R = NewRow<D>;
  const int blk = lane / R::LB, l = lane % R::LB;
  const bool is_v = blk >= R::NB;
  const __half* src = (is_v ? a.v_new : a.k_new) + (int64_t(bi) * a.L.n_kv_heads + h) * D + 32 * (blk % R::NB) + R::EQ * l;
  if constexpr (R::EQ == 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(src);
    nr.raw[0] = v.x; nr.raw[1] = v.y; nr.raw[2] = v.z; nr.raw[3] = v.w;
  } else {
    const uint2 v = *reinterpret_cast<const uint2*>(src);
    nr.raw[0] = v.x; nr.raw[1] = v.y;
  }
}
// Codes of the lane's part (cw: its EQ bytes for 8 bits; for 4 bits the lanes of the block's
// first 16 elements hold the EQ packed bytes j | j + 16 << 4, the others nothing) and the
// block's scale.  The warp's blocks mix 8- and 4-bit codes (K8V4, K4V8), so every shuffle sits
// on the path that all 32 lanes take: both reductions run in every lane, and each lane picks
// its own afterwards.
template <int D>
__device__ __forceinline__ __half new_row_quant(const NewRow<D>& nr, bool q8, int lane, uint32_t (&cw)[2]) {
  using R = NewRow<D>;
  constexpr int LB = R::LB, EQ = R::EQ;
  constexpr uint32_t FULL = 0xffffffffu;
  const int l = lane % LB;
  float x[EQ];
#pragma unroll
  for (int i = 0; i < EQ / 2; ++i) {
    const float2 f = h2_to_f2(nr.raw[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
  // 8 bits: amax over the block; 4 bits: m = the element of largest |x|, the lowest index on ties
  float am = fabsf(x[0]), m = x[0];
  int mi = EQ * l;
#pragma unroll
  for (int i = 1; i < EQ; ++i)
    if (fabsf(x[i]) > am) {
      am = fabsf(x[i]);
      m = x[i];
      mi = EQ * l + i;
    }
#pragma unroll
  for (int o = 1; o < LB; o <<= 1) {
    const float am2 = __shfl_xor_sync(FULL, am, o), m2 = __shfl_xor_sync(FULL, m, o);
    const int mi2 = __shfl_xor_sync(FULL, mi, o);
    if (am2 > am || (am2 == am && mi2 < mi)) {
      am = am2;
      m = m2;
      mi = mi2;
    }
  }
  const __half d = q8 ? __float2half_rn(__fdiv_rn(am, 127.0f)) : __float2half_rn(m * -0.125f);   // m / -8 exact
  const float df = __half2float(d);
  float c[EQ];                                           // 4-bit codes (unused by 8-bit lanes)
  cw[0] = cw[1] = 0u;
  if (df != 0.f) {
    const RoundCtx r = round_ctx(df);
    if (q8) {
#pragma unroll
      for (int k = 0; k < EQ / 4; ++k)
        cw[k] = pack_low_bytes(float_int_bits(round_code8(x[4 * k], r)), float_int_bits(round_code8(x[4 * k + 1], r)),
                               float_int_bits(round_code8(x[4 * k + 2], r)), float_int_bits(round_code8(x[4 * k + 3], r)));
    }
    const uint32_t dbits = __float_as_uint(df);
#pragma unroll
    for (int i = 0; i < EQ; ++i) c[i] = q8 ? 0.f : round_code4(x[i], r, dbits);
  } else {
#pragma unroll
    for (int i = 0; i < EQ; ++i) c[i] = 0.f;
  }
  // element j + 16 lies LB / 2 lanes further on (all lanes shuffle)
  float ch[EQ];
#pragma unroll
  for (int i = 0; i < EQ; ++i) ch[i] = __shfl_xor_sync(FULL, c[i], LB / 2);
  if (!q8) {
    uint32_t by[EQ];
#pragma unroll
    for (int i = 0; i < EQ; ++i) by[i] = __float_as_uint(__fmaf_rn(ch[i], 16.f, c[i]) + (kRoundBias + 136.f));   // u_j + 16 u_{j+16}
#pragma unroll
    for (int k = 0; k < EQ / 4; ++k) cw[k] = pack_low_bytes(by[4 * k], by[4 * k + 1], by[4 * k + 2], by[4 * k + 3]);
  }
  return d;
}
// Store the lane's part of the row: codes at `codes` (the block's first byte), the scale at `scale`.
template <int D>
__device__ __forceinline__ void new_row_store(uint8_t* codes, __half* scale, bool q8, int lane, const uint32_t (&cw)[2],
                                              __half d) {
  using R = NewRow<D>;
  constexpr int LB = R::LB, EQ = R::EQ;
  const int l = lane % LB;
  if (q8 || l < LB / 2) {
    uint8_t* dst = codes + EQ * l;
    if constexpr (EQ == 8) *reinterpret_cast<uint2*>(dst) = make_uint2(cw[0], cw[1]);
    else *reinterpret_cast<uint32_t*>(dst) = cw[0];
  }
  if (l == 0) *scale = d;
}

// Producer warp: streams the CTA's chunks into the stage ring (and, with a fused
// append, quantises each item's new token into its page and the stage).
template <int KB, int VB, int D, int G, int CT>
__device__ __forceinline__ void producer_role(const DecodeQArgs& a, const Batch& b,
                                              const QDecSmem<KB, VB, D, G, CT>& sm, int64_t x0, int64_t x1, int page0) {
  using T = QDec<KB, VB, D, G, CT>;
  constexpr int S = T::S, NB = T::NB;
  const int lane = threadIdx.x & 31;
  const uint64_t pol = l2_evict_first_policy();
  uint32_t it = 0;
  int s = 0;                                           // ring slot of stage `it` and its fill parity
  uint32_t ph = 0, aph = 0;                            // aph: phase of abar
  bool ok = true;
  // Page ids of the next 32 chunks, one per lane, loaded together once every 32 chunks: the
  // page-table read (a global load, ~1 us) would otherwise sit in front of every stage's copies
  // (the first 32 were loaded at the kernel's start: page0).
  int my_page = page0;
  NewRow<D> nr;
  for (int64_t x = x0; x < x1 && ok;) {
    const DecodeSeg sg = decode_find_seg(b, x, x1);
    const SeqDesc sd = b.s[sg.bi];
    // fused append: the new token's K and V, loaded as soon as the segment's last chunk is the
    // item's last (the one that holds the token)
    if (a.k_new != nullptr && sg.n > 0 && sg.k0 + sg.n == (sd.cr > 0 ? sd.cr : sd.c)) new_row_load<D>(nr, a, sg.bi, sg.h, lane);
    for (int k = sg.k0; k < sg.k0 + sg.n; ++k) {
      if ((it & 31) == 0 && it > 0) my_page = chunk_page(a, b, x0 + it + lane, x1);
      const int page = __shfl_sync(0xffffffffu, my_page, it & 31);
      if (!mbar_wait(sm.empty0 + 8 * s, ph ^ 1, sm.abort_flag, a.L.wait_ns)) {
        if (lane == 0) record_error(a.L.err, kErrWaitTimeout | 1);
        *sm.abort_flag = 1;
        ok = false;
        break;
      }
      const int tok0 = sd.lo / a.chunk * a.chunk + k * a.chunk;   // chunks start at the window's first chunk
      const int ntok = min(a.chunk, sd.a - tok0);
      const int ncopy = min(a.chunk, (ntok + 15) & ~15);
      if (page < 0 || page >= a.L.n_pages) {
        if (lane == 0) record_error(a.L.err, kErrBadPage);
        *sm.abort_flag = 1;
        ok = false;
        break;
      }
      const int r = tok0 % a.L.page_tokens;
      uint8_t* hb = a.L.head_ptr(a.layer + sd.l, page, sg.h);
      // fused append: this chunk holds the new token (position len - 1, chunk row ntok - 1)
      const bool app = a.k_new != nullptr && tok0 + ntok == sd.a;
      // test hook (cache created with KVQ_TEST_WITHHOLD_ARRIVAL set): CTA 0 never fills its
      // first stage, so its consumers' bounded waits run out and report kErrWaitTimeout
      const bool withhold = a.L.test_withhold && blockIdx.x == 0 && it == 0;
      if (lane == 0 && !withhold) {
        // an appending chunk's copies complete on abar: the stage is released to the consumers
        // only after the new row has been written into it
        const uint32_t bar = app ? sm.abar : sm.full0 + 8 * s;
        const uint32_t dst = smem_u32(sm.stages + s * T::STAGE);
        mbar_arrive_expect_tx(bar, uint32_t(ncopy * T::TOK_BYTES));
        bulk_g2s(dst, hb + int64_t(r) * T::K_ROW, ncopy * T::K_ROW, bar, pol);
        bulk_g2s(dst + T::OFF_KS, hb + a.L.k_scales_off + int64_t(r) * T::S_ROW, ncopy * T::S_ROW, bar, pol);
        bulk_g2s(dst + T::OFF_VC, hb + a.L.v_codes_off + int64_t(r) * T::V_ROW, ncopy * T::V_ROW, bar, pol);
        bulk_g2s(dst + T::OFF_VS, hb + a.L.v_scales_off + int64_t(r) * T::S_ROW, ncopy * T::S_ROW, bar, pol);
      }
      if (app) {
        // quantise the new K and V row into registers while the copies are in flight; once they
        // landed, write it over the copied (stale) row and release the stage, and only then store
        // it into the page (so that the release does not wait for those global stores)
        const int rl = ntok - 1;
        const int blk = lane / NewRow<D>::LB;
        const bool is_v = blk >= NB;
        const bool q8 = (is_v ? VB : KB) == 8;
        const int cb = q8 ? 32 : 16;                       // code bytes of one block
        const int row_b = is_v ? T::V_ROW : T::K_ROW;
        uint32_t cw[2];
        const __half d = new_row_quant<D>(nr, q8, lane, cw);
        if (!mbar_wait(sm.abar, aph, sm.abort_flag, a.L.wait_ns)) {
          if (lane == 0) record_error(a.L.err, kErrWaitTimeout | 10);
          *sm.abort_flag = 1;
          ok = false;
          break;
        }
        aph ^= 1;
        uint8_t* st = sm.stages + s * T::STAGE;
        new_row_store<D>(st + (is_v ? T::OFF_VC : 0) + rl * row_b + cb * (blk % NB),
                         reinterpret_cast<__half*>(st + (is_v ? T::OFF_VS : T::OFF_KS) + rl * T::S_ROW) + blk % NB, q8,
                         lane, cw, d);
        __syncwarp();
        mbar_arrive_if(sm.full0 + 8 * s, lane == 0);       // release: the row is visible to the consumers
        new_row_store<D>(hb + (is_v ? a.L.v_codes_off : 0) + int64_t(r + rl) * row_b + cb * (blk % NB),
                         reinterpret_cast<__half*>(hb + (is_v ? a.L.v_scales_off : a.L.k_scales_off) +
                                                   int64_t(r + rl) * T::S_ROW) + blk % NB,
                         q8, lane, cw, d);
      }
      ++it;
      if (++s == S) {
        s = 0;
        ph ^= 1;
      }
    }
    x += sg.adv;
  }
  // no copy may outlive the CTA: wait (bounded) for the last fills to land
  if (lane == 0)
    for (uint32_t j = it > uint32_t(S) ? it - S : 0; j < it; ++j) mbar_wait(sm.full0 + 8 * (j % S), (j / S) & 1, nullptr, a.L.wait_ns);
}

// A consumer warp's state for one item segment: the query digits of its heads,
// its running softmax and its accumulators.
template <int KB, int VB, int D, int G, int CT>
struct QWarp {
  using T = QDec<KB, VB, D, G, CT>;
  uint32_t qh[T::GW][8], ql[T::GW][8];   // query digits of the lane's key block, slot j = head j ^ fmap
  int qcorr[T::GW];                      // 4-bit keys: -8 * sum of the digits (codes are read as c + 8)
  float qsc[T::NF], m[T::NF], l[T::NF];  // per owned head: digit scale, running max and sum
  float O[T::GW][T::E];                  // value lane's accumulators, all of the warp's heads
};

// Per-lane byte offsets (pass 0) inside a stage and inside the warp's p' buffer; the other
// passes add compile-time constants, so every shared-memory access is one 32-bit register plus
// an immediate.
struct QLaneOff {
  uint32_t kc0, kc1;   // key codes of the lane's block: its first and second 16-byte chunk (8-bit keys)
  uint32_t ks, vs;     // K and V scale of the lane's block (score-lane layout)
  uint32_t vc;         // V codes of the value lane
  uint32_t pst, pld;   // p' store (score-lane layout) and load (value-lane layout)
};

// Score passes of one stage: sc[pass][j] for the lane's token and owned heads (-inf outside
// the valid rows [rv0, rv1) of the chunk; row0 = the lane's row in pass 0).
template <int KB, int VB, int D, int G, int CT, bool MASK = true>
__device__ __forceinline__ void qk_stage(const QWarp<KB, VB, D, G, CT>& w, uint32_t u_st, const QLaneOff& lo, int row0,
                                         bool masked, int rv0, int rv1,
                                         float (&sc)[QDec<KB, VB, D, G, CT>::NPASS][QDec<KB, VB, D, G, CT>::NF]) {
  using T = QDec<KB, VB, D, G, CT>;
  constexpr int GW = T::GW, NF = T::NF;
#pragma unroll
  for (int ps = 0; ps < T::NPASS; ++ps) {
    uint32_t cw[8];
    if constexpr (KB == 8) {
      const uint4 c0 = lds_v4(u_st + lo.kc0 + ps * T::TPP * T::K_ROW);
      const uint4 c1 = lds_v4(u_st + lo.kc1 + ps * T::TPP * T::K_ROW);
      cw[0] = c0.x; cw[1] = c0.y; cw[2] = c0.z; cw[3] = c0.w;
      cw[4] = c1.x; cw[5] = c1.y; cw[6] = c1.z; cw[7] = c1.w;
    } else {
      const uint4 c = lds_v4(u_st + lo.kc0 + ps * T::TPP * T::K_ROW);
      cw[0] = c.x & 0x0F0F0F0Fu; cw[1] = c.y & 0x0F0F0F0Fu; cw[2] = c.z & 0x0F0F0F0Fu; cw[3] = c.w & 0x0F0F0F0Fu;
      cw[4] = (c.x >> 4) & 0x0F0F0F0Fu; cw[5] = (c.y >> 4) & 0x0F0F0F0Fu;
      cw[6] = (c.z >> 4) & 0x0F0F0F0Fu; cw[7] = (c.w >> 4) & 0x0F0F0F0Fu;
    }
    const float dk = h_bits_to_f(lds_u16(u_st + lo.ks + ps * T::TPP * T::S_ROW));
    int hs[GW], ls[GW];
#pragma unroll
    for (int j = 0; j < GW; ++j) {
      hs[j] = 0;
      ls[j] = w.qcorr[j];
    }
#pragma unroll
    for (int k = 0; k < 8; ++k)
#pragma unroll
      for (int j = 0; j < GW; ++j) {
        hs[j] = __dp4a(int(cw[k]), int(w.qh[j][k]), hs[j]);
        ls[j] = __dp4a(int(cw[k]), int(w.ql[j][k]), ls[j]);
      }
    float ps_[GW];
#pragma unroll
    for (int j = 0; j < GW; ++j) ps_[j] = __int2float_rn(hs[j] * 256 + ls[j]) * dk;
    reduce_scatter_perm<T::LPT, GW>(ps_);
    const int row = row0 + ps * T::TPP;
#pragma unroll
    for (int j = 0; j < NF; ++j) {
      const float v = ps_[j] * w.qsc[j];
      if constexpr (MASK)
        sc[ps][j] = (!masked || (row >= rv0 && row < rv1)) ? v : -INFINITY;
      else
        sc[ps][j] = v;
    }
  }
}

// (o0, o1) += p (x0, x1) as one packed fp32 FMA (two correctly rounded FMAs: the same result as
// two scalar ones, in half the issue slots).
__device__ __forceinline__ void fma_pair(float& o0, float& o1, float p, float x0, float x1) {
  const float2 r = ffma2(make_float2(p, p), make_float2(x0, x1), make_float2(o0, o1));
  o0 = r.x;
  o1 = r.y;
}

// Value passes of one stage: O += p' c over the lane's tokens of the partition.
template <int KB, int VB, int D, int G, int CT>
__device__ __forceinline__ void pv_stage(QWarp<KB, VB, D, G, CT>& w, uint32_t u_st, uint32_t u_pb, const QLaneOff& lo) {
  using T = QDec<KB, VB, D, G, CT>;
  constexpr int GW = T::GW, NB = T::NB;
#pragma unroll
  for (int pv = 0; pv < T::NPV; ++pv) {
    const uint32_t va = u_st + lo.vc + pv * T::TPV * T::V_ROW;
    uint32_t vw[T::BPL / 4];
    if constexpr (T::BPL == 4) {
      vw[0] = lds_u32(va);
    } else if constexpr (T::BPL == 8) {
      const uint2 u = lds_v2(va);
      vw[0] = u.x;
      vw[1] = u.y;
    } else {
#pragma unroll
      for (int c = 0; c < T::BPL / 16; ++c) {
        const uint4 u = lds_v4(va + 16 * c);
        vw[4 * c] = u.x; vw[4 * c + 1] = u.y; vw[4 * c + 2] = u.z; vw[4 * c + 3] = u.w;
      }
    }
    const uint32_t pa = u_pb + lo.pld + pv * T::TPV * NB * GW * 4;
    float pg[GW];
    if constexpr (GW == 4) {
      const float4 f = lds_f4(pa);
      pg[0] = f.x; pg[1] = f.y; pg[2] = f.z; pg[3] = f.w;
    } else if constexpr (GW == 2) {
      const float2 f = lds_f2(pa);
      pg[0] = f.x;
      pg[1] = f.y;
    } else {
      pg[0] = lds_f32(pa);
    }
#pragma unroll
    for (int wi = 0; wi < T::BPL / 4; ++wi) {
      if constexpr (VB == 4) {
        float f[8];
        cvt_v4_word(vw[wi], f);
#pragma unroll
        for (int g = 0; g < GW; ++g)
#pragma unroll
          for (int e = 0; e < 8; e += 2) fma_pair(w.O[g][8 * wi + e], w.O[g][8 * wi + e + 1], pg[g], f[e], f[e + 1]);
      } else {
        float f[4];
        cvt_v8_word(vw[wi], f);
#pragma unroll
        for (int g = 0; g < GW; ++g)
#pragma unroll
          for (int e = 0; e < 4; e += 2) fma_pair(w.O[g][4 * wi + e], w.O[g][4 * wi + e + 1], pg[g], f[e], f[e + 1]);
      }
    }
  }
}

// Online softmax of one stage's scores, then p' = p d_v into the warp's buffer (which the
// warp's value passes of the previous stage have finished reading).
template <int KB, int VB, int D, int G, int CT, bool MASK = true>
__device__ __forceinline__ void softmax_stage(QWarp<KB, VB, D, G, CT>& w,
                                              const float (&sc)[QDec<KB, VB, D, G, CT>::NPASS][QDec<KB, VB, D, G, CT>::NF],
                                              uint32_t u_st, uint32_t u_pb, const QLaneOff& lo, int row0, bool masked,
                                              int rv0, int rv1) {
  using T = QDec<KB, VB, D, G, CT>;
  constexpr int GW = T::GW, NF = T::NF, LPT = T::LPT, NB = T::NB;
  constexpr uint32_t FULL = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  // lazy maximum: moved only when a score passes it by 2^8
  bool need = false;
#pragma unroll
  for (int ps = 0; ps < T::NPASS; ++ps)
#pragma unroll
    for (int j = 0; j < NF; ++j) need |= sc[ps][j] > w.m[j] + 8.f;
  if (__any_sync(FULL, need)) {
    float alpha[NF];
#pragma unroll
    for (int j = 0; j < NF; ++j) {
      float mx = sc[0][j];
#pragma unroll
      for (int ps = 1; ps < T::NPASS; ++ps) mx = fmaxf(mx, sc[ps][j]);
#pragma unroll
      for (int o = LPT; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
      const float mn = fmaxf(w.m[j], mx);
      alpha[j] = fast_exp2(w.m[j] - mn);               // 0 while m is -inf
      w.m[j] = mn;
      w.l[j] *= alpha[j];
    }
    // rescale the accumulators of every head: head g's factor is held by the lane of token 0
    // that owns g after the reduce-scatter (all tokens hold the same maximum)
#pragma unroll
    for (int g = 0; g < GW; ++g) {
      const float al = __shfl_sync(FULL, alpha[g % NF], rs_lane_of<LPT, GW>(g));
#pragma unroll
      for (int i = 0; i < T::E; ++i) w.O[g][i] *= al;
    }
  }
  __syncwarp();                                        // the previous stage's p' has been read
#pragma unroll
  for (int ps = 0; ps < T::NPASS; ++ps) {
    const int row = row0 + ps * T::TPP;
    const bool valid = !MASK || !masked || (row >= rv0 && row < rv1);
    float p[NF];
#pragma unroll
    for (int j = 0; j < NF; ++j) {
      const float e2 = fast_exp2(sc[ps][j] - w.m[j]);
      p[j] = valid ? e2 : 0.f;
      w.l[j] += p[j];
    }
    float pa[GW];
#pragma unroll
    for (int g = 0; g < GW; ++g) pa[g] = __shfl_sync(FULL, p[g % NF], (lane & ~(LPT - 1)) | rs_lane_of<LPT, GW>(g));
    const float dv0 = h_bits_to_f(lds_u16(u_st + lo.vs + ps * T::TPP * T::S_ROW));
    const float dv = valid ? dv0 : 0.f;
    const uint32_t dst = u_pb + lo.pst + ps * T::TPP * NB * GW * 4;
    if constexpr (GW == 4) {
      sts_f4(dst, pa[0] * dv, pa[1] * dv, pa[2] * dv, pa[3] * dv);
    } else if constexpr (GW == 2) {
      sts_f2(dst, pa[0] * dv, pa[1] * dv);
    } else {
      sts_f32(dst, pa[0] * dv);
    }
  }
  __syncwarp();
}

// Consumer warp: for each item segment of the CTA's range, the query digits, then the
// stage pipeline (scores of stage k with the values of stage k - 1), then the merge.
template <int KB, int VB, int D, int G, int CT>
__device__ __forceinline__ void consumer_role(const DecodeQArgs& a, const Batch& b, const QDecSmem<KB, VB, D, G, CT>& sm,
                                              int64_t x0, int64_t x1) {
  using T = QDec<KB, VB, D, G, CT>;
  constexpr int S = T::S, GW = T::GW, NF = T::NF, LPT = T::LPT, NHG = T::NHG, E = T::E;
  constexpr uint32_t FULL = 0xffffffffu;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int part = warp / NHG, hg = warp % NHG;
  const int prow0 = part * T::W;
  const int tl = lane / LPT, blk = lane % LPT;         // score lane: token tl of a pass, key block blk
  const int tv = lane / T::LPV, sl = lane % T::LPV;    // value lane: token tv of a pass, element slot sl
  const int fmap = rs_map<LPT, GW>(blk);
  const int xr = kq_rot<KB, D>(tl);
  const uint32_t u_stages = smem_u32(sm.stages);
  const uint32_t u_pb = smem_u32(sm.pbuf) + warp * T::PB_WARP;
  QLaneOff lo;
  {
    const int row = prow0 + tl;                        // score lane's row in pass 0
    const int vrow = prow0 + tv;                       // value lane's row in pass 0
    lo.kc0 = uint32_t(row * T::K_ROW + blk * T::KBLK + 16 * xr);
    lo.kc1 = uint32_t(row * T::K_ROW + blk * T::KBLK + 16 * (xr ^ 1));
    lo.ks = uint32_t(T::OFF_KS + row * T::S_ROW + 2 * blk);
    lo.vs = uint32_t(T::OFF_VS + row * T::S_ROW + 2 * blk);
    lo.vc = uint32_t(T::OFF_VC + vrow * T::V_ROW + sl * T::BPL);
    lo.pst = uint32_t((tl * T::NB + blk) * GW * 4);
    lo.pld = uint32_t((tv * T::NB + (sl * T::BPL) / T::VBLK) * GW * 4);
  }
  const int row0 = prow0 + tl;
  QWarp<KB, VB, D, G, CT> w;
  uint32_t itm = 0, itw = 0, itc = 0;
  int s = 0;                                           // ring slot of the next stage and its fill parity
  uint32_t ph = 0;
  for (int64_t x = x0; x < x1;) {
    const DecodeSeg sg = decode_find_seg(b, x, x1);
    const SeqDesc sd = b.s[sg.bi];
    // ---- query digits in permuted slots: slot j <-> head hg * GW + (j ^ fmap), this lane's block.
    // The warp's GW query rows are staged in shared memory with 16-byte loads, then each lane reads
    // its elements in its own (bank-rotated) word order from there.
    __half* qs = sm.qbuf + warp * GW * D;
    {
      const uint4* src = reinterpret_cast<const uint4*>(a.q + (int64_t(sg.bi) * a.n_q_heads + sg.h * G + hg * GW) * D);
      for (int i = lane; i < GW * D / 8; i += 32) reinterpret_cast<uint4*>(qs)[i] = src[i];
      __syncwarp();
    }
    // The digits are computed once per warp: lane (head j, slice u) takes EPL consecutive elements
    // of head row j, finds max|q| with its head's other lanes, and writes the packed hi and lo
    // words of its elements (and, for 4-bit keys, the sum of the digits of each key block) into
    // the warp's p' buffer, which is idle at an item's start.  Each lane then loads the words of
    // its own key block in its own word order.
    {
      constexpr int LH = 32 / GW < D / 4 ? 32 / GW : D / 4;   // lanes per head
      constexpr int EPL = D / LH;                              // elements per lane (4, 8 or 16)
      constexpr int WPL = EPL / 4;                             // digit words per lane
      const uint32_t qd_hi = u_pb, qd_lo = u_pb + GW * D;      // [GW][D / 4] words each
      const uint32_t qd_corr = u_pb + 2 * GW * D, qd_amax = qd_corr + GW * T::NB * 4;
      const int j = lane / LH, u = lane % LH;
      const bool act = j < GW;
      const __half* qe = qs + (act ? j : 0) * D + u * EPL;
      uint32_t hw[EPL / 2];
      if constexpr (EPL == 16) {
        const uint4 a0 = reinterpret_cast<const uint4*>(qe)[0], a1 = reinterpret_cast<const uint4*>(qe)[1];
        hw[0] = a0.x; hw[1] = a0.y; hw[2] = a0.z; hw[3] = a0.w; hw[4] = a1.x; hw[5] = a1.y; hw[6] = a1.z; hw[7] = a1.w;
      } else if constexpr (EPL == 8) {
        const uint4 a0 = reinterpret_cast<const uint4*>(qe)[0];
        hw[0] = a0.x; hw[1] = a0.y; hw[2] = a0.z; hw[3] = a0.w;
      } else {
        const uint2 a0 = reinterpret_cast<const uint2*>(qe)[0];
        hw[0] = a0.x; hw[1] = a0.y;
      }
      float mx = 0.f;
#pragma unroll
      for (int i = 0; i < EPL / 2; ++i) {
        const float2 f = h2_to_f2(hw[i]);
        mx = fmax3(mx, fabsf(f.x), fabsf(f.y));
      }
#pragma unroll
      for (int o = 1; o < LH; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
      const float amax = mx * fabsf(a.scale_log2);
      // n = rint(q / s) with s = max|q| / 32512 (|n| <= 32512), as hi = (n + 128) >> 8 and the low byte
      // lo = n mod 256 read as int8, so that n = 256 hi + lo
      const float mul = amax > 0.f ? a.scale_log2 * (32512.f / amax) : 0.f;
      int corr = 0;
#pragma unroll
      for (int k = 0; k < WPL; ++k) {
        const float2 f01 = h2_to_f2(hw[2 * k]), f23 = h2_to_f2(hw[2 * k + 1]);
        int n[4];
        n[0] = __float_as_int(fmaf(f01.x, mul, 12582912.f)) - 0x4B400000;   // round to nearest
        n[1] = __float_as_int(fmaf(f01.y, mul, 12582912.f)) - 0x4B400000;
        n[2] = __float_as_int(fmaf(f23.x, mul, 12582912.f)) - 0x4B400000;
        n[3] = __float_as_int(fmaf(f23.y, mul, 12582912.f)) - 0x4B400000;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          n[e] = max(-32512, min(32512, n[e]));
          corr += n[e];
        }
        const uint32_t lo = __byte_perm(__byte_perm(n[0], n[1], 0x0040), __byte_perm(n[2], n[3], 0x0040), 0x5410);
        const int h0 = (n[0] + 128) >> 8, h1 = (n[1] + 128) >> 8, h2 = (n[2] + 128) >> 8, h3 = (n[3] + 128) >> 8;
        const uint32_t hi = __byte_perm(__byte_perm(h0, h1, 0x0040), __byte_perm(h2, h3, 0x0040), 0x5410);
        if (act) {
          const uint32_t wo = 4 * uint32_t(j * (D / 4) + u * WPL + k);
          asm volatile("st.shared.u32 [%0], %1;" ::"r"(qd_hi + wo), "r"(hi) : "memory");
          asm volatile("st.shared.u32 [%0], %1;" ::"r"(qd_lo + wo), "r"(lo) : "memory");
        }
      }
      // digit sum of each 32-element block: the block's 32 / EPL lanes are adjacent
#pragma unroll
      for (int o = 1; o < 32 / EPL; o <<= 1) corr += __shfl_xor_sync(FULL, corr, o);
      if (act && u % (32 / EPL) == 0)
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(qd_corr + 4 * uint32_t(j * T::NB + u * EPL / 32)), "r"(corr) : "memory");
      if (act && u == 0) sts_f32(qd_amax + 4 * j, amax);
      __syncwarp();
      // this lane's words: slot j holds head j ^ fmap; word w of its order is natural word
      // 4 ((w >> 2) ^ xr) + (w & 3) of its block (xr = 0 for 4-bit keys)
#pragma unroll
      for (int jj = 0; jj < GW; ++jj) {
        const uint32_t base = 4 * uint32_t((jj ^ fmap) * (D / 4) + blk * 8);
        const uint4 h0 = lds_v4(qd_hi + base + 16 * xr), h1 = lds_v4(qd_hi + base + 16 * (xr ^ 1));
        const uint4 l0 = lds_v4(qd_lo + base + 16 * xr), l1 = lds_v4(qd_lo + base + 16 * (xr ^ 1));
        w.qh[jj][0] = h0.x; w.qh[jj][1] = h0.y; w.qh[jj][2] = h0.z; w.qh[jj][3] = h0.w;
        w.qh[jj][4] = h1.x; w.qh[jj][5] = h1.y; w.qh[jj][6] = h1.z; w.qh[jj][7] = h1.w;
        w.ql[jj][0] = l0.x; w.ql[jj][1] = l0.y; w.ql[jj][2] = l0.z; w.ql[jj][3] = l0.w;
        w.ql[jj][4] = l1.x; w.ql[jj][5] = l1.y; w.ql[jj][6] = l1.z; w.ql[jj][7] = l1.w;
        w.qcorr[jj] = KB == 4 ? -8 * int(lds_u32(qd_corr + 4 * uint32_t((jj ^ fmap) * T::NB + blk))) : 0;
      }
#pragma unroll
      for (int jj = 0; jj < NF; ++jj) {                        // slot jj < NF ends with head jj ^ fmap
        w.qsc[jj] = lds_f32(qd_amax + 4 * (jj ^ fmap)) * (1.f / 32512.f);
        w.m[jj] = -INFINITY;
        w.l[jj] = 0.f;
      }
      __syncwarp();                                            // the p' stores may now reuse the area
    }
#pragma unroll
    for (int g = 0; g < GW; ++g)
#pragma unroll
      for (int i = 0; i < E; ++i) w.O[g][i] = 0.f;

    // ---- stage pipeline: chunk k's scores together with chunk k - 1's values
    const int base_tok = sd.lo / a.chunk * a.chunk;        // chunks start at the window's first chunk
    uint32_t u_prev = u_stages;
    int s_prev = 0;
    for (int k = sg.k0; k < sg.k0 + sg.n; ++k) {
      if (!mbar_wait(sm.full0 + 8 * s, ph, sm.abort_flag, a.L.wait_ns)) {
        if (lane == 0) record_error(a.L.err, kErrWaitTimeout | 2);
        *sm.abort_flag = 1;
        return;
      }
      const uint32_t u_st = u_stages + s * T::STAGE;
      const int tok0 = base_tok + k * a.chunk;
      const int rv0 = max(0, sd.lo - tok0), rv1 = min(a.chunk, sd.a - tok0);   // valid rows [rv0, rv1)
      const bool masked = rv0 > prow0 || rv1 < prow0 + T::W;
      float sc[T::NPASS][NF];
      // the steady state (a full stage after the first) in a copy without the row mask, whose selects
      // the compiler would otherwise run on every stage; at G = 8 the doubled block costs more than it saves
      bool steady = false;
      if constexpr (T::NHG == 1) steady = k != sg.k0 && !masked;
      if (steady) {
        qk_stage<KB, VB, D, G, CT, false>(w, u_st, lo, row0, false, rv0, rv1, sc);
        pv_stage<KB, VB, D, G, CT>(w, u_prev, u_pb, lo);
        __syncwarp();
        mbar_arrive_if(sm.empty0 + 8 * s_prev, lane == 0);
        softmax_stage<KB, VB, D, G, CT, false>(w, sc, u_st, u_pb, lo, row0, false, rv0, rv1);
      } else {
        if (k == sg.k0) {
          qk_stage<KB, VB, D, G, CT>(w, u_st, lo, row0, masked, rv0, rv1, sc);
        } else {
          // one straight-line block: the previous stage's values and this stage's scores
          qk_stage<KB, VB, D, G, CT>(w, u_st, lo, row0, masked, rv0, rv1, sc);
          pv_stage<KB, VB, D, G, CT>(w, u_prev, u_pb, lo);
          __syncwarp();
          mbar_arrive_if(sm.empty0 + 8 * s_prev, lane == 0);
        }
        softmax_stage<KB, VB, D, G, CT>(w, sc, u_st, u_pb, lo, row0, masked, rv0, rv1);
      }
      u_prev = u_st;
      s_prev = s;
      if (++s == S) {
        s = 0;
        ph ^= 1;
      }
    }
    pv_stage<KB, VB, D, G, CT>(w, u_prev, u_pb, lo);
    __syncwarp();
    mbar_arrive_if(sm.empty0 + 8 * s_prev, lane == 0);

    // ---- publish (m, l) of the owned heads and O of all the warp's heads, then merge
    if (!mbar_wait(sm.mfree, (itm & 1) ^ 1, sm.abort_flag, a.L.wait_ns)) {
      if (lane == 0) record_error(a.L.err, kErrWaitTimeout | 5);
      *sm.abort_flag = 1;
      return;
    }
#pragma unroll
    for (int j = 0; j < NF; ++j)
#pragma unroll
      for (int o = LPT; o < 32; o <<= 1) w.l[j] += __shfl_xor_sync(FULL, w.l[j], o);
    if (tl == 0) {
#pragma unroll
      for (int j = 0; j < NF; ++j) {
        const int g = hg * GW + (j ^ fmap);
        sm.mrg_ml[(part * G + g) * 2] = w.m[j];
        sm.mrg_ml[(part * G + g) * 2 + 1] = w.l[j];
      }
    }
#pragma unroll
    for (int o = T::LPV; o < 32; o <<= 1)
#pragma unroll
      for (int g = 0; g < GW; ++g)
#pragma unroll
        for (int i = 0; i < E; ++i) w.O[g][i] += __shfl_xor_sync(FULL, w.O[g][i], o);
    if (tv == 0) {
      float* mo = sm.mrg_o + (part * G + hg * GW) * D;
#pragma unroll
      for (int g = 0; g < GW; ++g)
#pragma unroll
        for (int i = 0; i < E; ++i) mo[g * D + v_elem_of<VB, E>(sl, i)] = w.O[g][i];
    }
    if (!merge_item<KB, VB, D, G, CT>(a, sm, sg, sd, itm, itw, itc)) return;
    x += sg.adv;
  }
}

// Per-warpgroup register count after launch: setmaxnreg.inc to grow, .dec to shrink (the
// direction must match, and every warp of the warpgroup executes it).
template <int R, int R_LAUNCH>
__device__ __forceinline__ void set_max_regs() {
  static_assert(R % 8 == 0 && R >= 24 && R <= 256, "setmaxnreg range");
  if constexpr (R > R_LAUNCH) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R));
  else if constexpr (R < R_LAUNCH) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R));
}

template <int KB, int VB, int D, int G, int CT>
__global__ void __launch_bounds__(QDec<KB, VB, D, G, CT>::NT, 1)
    decode_q_kernel(const DecodeQArgs a, const __grid_constant__ Batch b) {
  using T = QDec<KB, VB, D, G, CT>;
  static_assert(T::FITS, "stage ring does not fit");
  extern __shared__ __align__(128) uint8_t smem[];
  const QDecSmem<KB, VB, D, G, CT> sm(smem);
  const int warp = threadIdx.x >> 5;
  const int64_t x0 = int64_t(blockIdx.x) * a.cpc;
  const int64_t x1 = min(a.total_chunks, x0 + a.cpc);
  // the producer's first 32 page ids, read while the barriers are set up
  const int page0 = warp == T::NW ? chunk_page(a, b, x0 + (threadIdx.x & 31), x1) : -1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < T::S; ++s) {
      mbar_init(sm.full0 + 8 * s, 1);
      mbar_init(sm.empty0 + 8 * s, T::NW);
    }
    mbar_init(sm.mfull, T::NW);
    mbar_init(sm.mfree, T::NW);
    mbar_init(sm.mws, T::NW);
    mbar_init(sm.mlast, 1);
    mbar_init(sm.mcomb, T::NW);
    mbar_init(sm.abar, 1);
    *sm.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (warp >= T::NW) {
    set_max_regs<T::REG_P, T::REG_L>();
    if (warp == T::NW) producer_role<KB, VB, D, G, CT>(a, b, sm, x0, x1, page0);
    return;                                                 // the group's other 3 warps have no role
  }
  set_max_regs<T::REG_C, T::REG_L>();
  consumer_role<KB, VB, D, G, CT>(a, b, sm, x0, x1);
}

}  // namespace kvq
