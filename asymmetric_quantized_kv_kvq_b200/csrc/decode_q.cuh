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
// CTA = 4 warpgroups: score warps (4), value warps (8), the producer warp (+3
// idle warps); after launch the producer group gives registers back
// (setmaxnreg) and the score group, whose query digits live in registers, takes
// them (208 per thread; value warps 120, producer 64):
//  - producer: streams each chunk's K codes, K scales, V codes and V scales
//    (four contiguous ranges of one page's head block) into a ring of shared-
//    memory stages with 1-D TMA bulk copies; with a fused append it first
//    quantises the new token's K and V row into the page (same block
//    quantiser as the append kernel), for the one chunk that holds it;
//  - a stage's tokens are split into NPART partitions; each partition has its
//    own running softmax state (m, l per head) kept by its score warp(s) and
//    its own accumulators O kept by its value warps;
//  - score warps hold the query as two int8 digits per element (15 bits:
//    q ~= s (256 hi + lo), s = max|q| / 32512 per head) and take dot products
//    with dp4a directly on the stored key codes (4-bit codes unpacked to
//    bytes, their +8 offset folded into the accumulator's start); a lane sums
//    two 32-element blocks of one token for GW heads (16 independent dp4a
//    chains), and one exchange with the token's other lane (head_dim 128; none
//    at 64) leaves each lane the full scores of its own heads (the query's
//    register slots are permuted per lane so the exchange needs no selects);
//    online softmax with a lazily moved maximum (moved only when a score passes
//    it by 2^8); each lane then publishes p' = p d_v for its two value blocks
//    and all GW heads (16-byte stores);
//  - value warps convert each value code once (a byte placed in the mantissa
//    of 2^23, then one subtraction per pair) and accumulate O += p' c with one
//    scalar FMA per element and head; a lane owns E elements of one token, so
//    one converted code feeds all G heads.
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

template <int KB, int VB, int D, int G>
struct QDec {
  static constexpr int NB = D / 32;                  // 32-element blocks per row
  static constexpr int SBL = 2;                      // key blocks per score lane
  static constexpr int LPT = NB / SBL;               // score lanes per token
  static constexpr int TPP = 32 / LPT;               // tokens per score pass
  static constexpr int GW = G > 4 ? 4 : G;           // query heads per score warp
  static constexpr int NHG = G / GW;                 // score warps per partition (head groups)
  static constexpr int NF = GW > LPT ? GW / LPT : 1; // heads a score lane owns after the reduce-scatter
  static constexpr int NS = 4;                       // score warps
  static constexpr int NP = 8;                       // value warps
  static constexpr int NPART = NS / NHG;             // token partitions of a stage
  static constexpr int NPP = NP / NPART;             // value warps per partition (split its tokens)
  static constexpr int NCW = NS + NP;                // consumer warps
  static constexpr int NT = 16 * 32;                 // 4 warpgroups: score, value, value, producer (+3 idle)
  // registers per thread after the split (setmaxnreg; the block launches with 128 each):
  // 128 * (REG_S + 2 REG_V + REG_P) <= 65536
  static constexpr int REG_S = 208, REG_V = 120, REG_P = 64;
  static_assert(REG_S + 2 * REG_V + REG_P <= 512, "register split");
  static_assert(NS == 4 && NP == 8, "warp roles are whole warpgroups");
  static constexpr int C = 128;                      // tokens per stage
  static constexpr int W = C / NPART;                // tokens per partition
  static constexpr int NPASS = W / TPP;              // score passes per stage
  static constexpr int WP = W / NPP;                 // tokens per value warp per stage
  static constexpr int E = G >= 4 ? 64 / G : 16;    // value elements per lane (E x G <= 64 accumulators)
  static constexpr int LPV = D / E;                  // value lanes per token
  static constexpr int TPV = 32 / LPV;               // tokens per value pass
  static constexpr int NPV = WP / TPV;               // value passes per stage
  static constexpr int K_ROW = KB == 8 ? D : D / 2;
  static constexpr int V_ROW = VB == 8 ? D : D / 2;
  static constexpr int S_ROW = NB * 2;               // fp16 scales per row
  static constexpr int TOK_BYTES = K_ROW + S_ROW + V_ROW + S_ROW;
  static constexpr int BPL = VB == 8 ? E : E / 2;    // value code bytes per lane
  static constexpr int VBLK = VB == 8 ? 32 : 16;     // code bytes per value block
  static constexpr int NBL = BPL > VBLK ? BPL / VBLK : 1;   // value blocks per lane
  static constexpr int OFF_KS = C * K_ROW;
  static constexpr int OFF_VC = OFF_KS + C * S_ROW;
  static constexpr int OFF_VS = OFF_VC + C * V_ROW;
  static constexpr int STAGE = OFF_VS + C * S_ROW;
  static constexpr int PBUF = NPART * 2 * W * NB * G * 4;        // p', two buffers per partition
  static constexpr int ALPHA = (NPART * 2 * (G + NHG) * 4 + 15) / 16 * 16;   // rescale factors + flags
  static constexpr int MRG_O = NP * G * D * 4;                   // one partial O per value warp
  static constexpr int MRG_ML = NPART * G * 2 * 4;
  static constexpr int QBUF = NS * GW * D * 2;                   // each score warp's query rows (fp16)
  static constexpr int BARS = 512;
  static constexpr int FIXED = PBUF + ALPHA + MRG_O + MRG_ML + QBUF + BARS;
  static constexpr int SMEM_LIMIT = 227 * 1024;
  static constexpr int S_FIT = (SMEM_LIMIT - FIXED) / STAGE;
  static constexpr int S = S_FIT > 8 ? 8 : S_FIT;    // stages in the ring
  static constexpr int SMEM = S * STAGE + FIXED;
  static_assert(S >= 3, "stage ring does not fit");
  static_assert(W % TPP == 0 && WP % TPV == 0 && NPV >= 1 && NPASS >= 1, "tiling");
  static_assert(E * G <= 64 && BPL % 4 == 0, "value lane");
  static_assert(STAGE % 16 == 0 && OFF_KS % 16 == 0 && OFF_VC % 16 == 0 && OFF_VS % 16 == 0, "alignment");
  static_assert(S * STAGE % 16 == 0 && PBUF % 16 == 0 && ALPHA % 16 == 0 && MRG_O % 16 == 0, "alignment");
  static_assert(MRG_ML % 16 == 0 && QBUF % 16 == 0, "alignment");
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
// A score lane reads the codes of its token's two key blocks (64 bytes of 8-bit
// codes in four 16-byte chunks, or 32 bytes of 4-bit codes in two), chunk
// c ^ x at load step c, x depending on the lane's token, so that the 16-byte
// loads of a warp spread over all shared-memory banks.  The words land in two
// slots of 8: slot sp holds the lane's key block sp ^ bswap (bswap = x >> 1 for
// 8-bit, x for 4-bit), words in this order: 8-bit: element
// 16 ((w >> 2) ^ (x & 1)) + 4 (w & 3) + e of the block for byte e of word w;
// 4-bit: words 0..3 the low nibbles (elements 4w + e), 4..7 the high nibbles
// (elements 16 + 4 (w - 4) + e), unpacked to one byte each (0..15).
template <int KB>
__device__ __forceinline__ void load_kq2(const uint8_t* span, int x, uint32_t (&cw)[16]) {
  if constexpr (KB == 8) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 a = *reinterpret_cast<const uint4*>(span + 16 * (c ^ x));
      cw[4 * c] = a.x; cw[4 * c + 1] = a.y; cw[4 * c + 2] = a.z; cw[4 * c + 3] = a.w;
    }
  } else {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const uint4 a = *reinterpret_cast<const uint4*>(span + 16 * (c ^ x));
      cw[8 * c] = a.x & 0x0F0F0F0Fu; cw[8 * c + 1] = a.y & 0x0F0F0F0Fu;
      cw[8 * c + 2] = a.z & 0x0F0F0F0Fu; cw[8 * c + 3] = a.w & 0x0F0F0F0Fu;
      cw[8 * c + 4] = (a.x >> 4) & 0x0F0F0F0Fu; cw[8 * c + 5] = (a.y >> 4) & 0x0F0F0F0Fu;
      cw[8 * c + 6] = (a.z >> 4) & 0x0F0F0F0Fu; cw[8 * c + 7] = (a.w >> 4) & 0x0F0F0F0Fu;
    }
  }
}
// Element (within its block) of byte e of word w of a slot, for the load order above.
template <int KB>
__host__ __device__ constexpr int kq2_elem(int w, int e, int x) {
  if (KB == 8) return 16 * ((w >> 2) ^ (x & 1)) + 4 * (w & 3) + e;
  return w < 4 ? 4 * w + e : 16 + 4 * (w - 4) + e;
}
// Chunk rotation x of a score lane of token tl (see load_kq2) and the block swap it implies.
template <int KB, int D>
__device__ __forceinline__ int kq2_rot(int tl) {
  if (KB == 8) return D == 128 ? (tl & 3) : ((tl >> 1) & 3);
  return D == 128 ? ((tl >> 1) & 1) : ((tl >> 2) & 1);
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
template <int KB, int VB, int D, int G>
struct QDecSmem {
  using T = QDec<KB, VB, D, G>;
  uint8_t* stages;
  float* pbuf;          // [part][parity][W][NB][G]  p' = p d_v
  float* palpha;        // [part][parity][G]         O rescale factors
  int* pflag;           // [part][parity][NHG]       1 when the head group moved its maximum
  float* mrg_o;         // [value warp][G][D]
  float* mrg_ml;        // [part][G][2]
  __half* qbuf;         // [score warp][GW][D]
  uint32_t full0, empty0, ready0, free0, mfull, mfree, mws, mlast, mcomb;
  volatile int* abort_flag;
  volatile int* last_flag;

  __device__ __forceinline__ explicit QDecSmem(uint8_t* smem) {
    stages = smem;
    pbuf = reinterpret_cast<float*>(smem + T::S * T::STAGE);
    palpha = reinterpret_cast<float*>(smem + T::S * T::STAGE + T::PBUF);
    pflag = reinterpret_cast<int*>(palpha + T::NPART * 2 * G);
    mrg_o = reinterpret_cast<float*>(smem + T::S * T::STAGE + T::PBUF + T::ALPHA);
    mrg_ml = mrg_o + T::NP * G * D;
    qbuf = reinterpret_cast<__half*>(mrg_ml + T::NPART * G * 2);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::S * T::STAGE + T::FIXED - T::BARS);
    full0 = smem_u32(bars);                              // [S]: stage filled (tx bytes)
    empty0 = full0 + 8 * T::S;                           // [S]: stage released by every consumer warp
    ready0 = empty0 + 8 * T::S;                          // [part][parity]: p' published by the score warps
    free0 = ready0 + 16 * T::NPART;                      // [part][parity]: p' consumed by the value warps
    mfull = free0 + 16 * T::NPART;                       // merge data written
    mfree = mfull + 8;                                   // merge data consumed
    mws = mfull + 16;                                    // partial written to the workspace
    mlast = mfull + 24;                                  // "last CTA of the item" decided
    mcomb = mfull + 32;                                  // merge weights of a split item written
    abort_flag = reinterpret_cast<volatile int*>(bars + 2 * T::S + 4 * T::NPART + 5);
    last_flag = abort_flag + 1;
  }
};

// End of an item segment, run by every consumer warp after it published its
// part (m, l or O) into the merge area: combine the partitions, write the
// output (item inside this CTA) or this CTA's partial, and let the last CTA of
// a split item merge all partials.  Returns false when a wait gave up.
template <int KB, int VB, int D, int G>
__device__ __forceinline__ bool merge_item(const DecodeQArgs& a, const QDecSmem<KB, VB, D, G>& sm,
                                           const DecodeSeg& sg, const SeqDesc& sd, uint32_t& itm,
                                           uint32_t& itw, uint32_t& itc) {
  using T = QDec<KB, VB, D, G>;
  constexpr int NPART = T::NPART, NPP = T::NPP, NCW = T::NCW;
  const int lane = threadIdx.x & 31;
  const int H = a.L.n_kv_heads;
  const int item = sg.bi * H + sg.h;
  __syncwarp();
  if (lane == 0) mbar_arrive(sm.mfull);
  if (!mbar_wait(sm.mfull, itm & 1, sm.abort_flag, a.L.wait_ns)) {
    if (lane == 0) record_error(a.L.err, kErrWaitTimeout | 6);
    *sm.abort_flag = 1;
    return false;
  }
  const int nch = sd.c;
  const int64_t off = int64_t(sd.b) + int64_t(sg.h) * nch;
  const int64_t c0 = off / a.cpc, c1 = (off + nch - 1) / a.cpc;
  const int ct = threadIdx.x;                          // consumer threads are 0 .. NCW * 32 - 1
  for (int e = ct; e < G * D; e += NCW * 32) {
    const int g = e / D, d = e % D;
    float M = -INFINITY;
#pragma unroll
    for (int pt = 0; pt < NPART; ++pt) M = fmaxf(M, sm.mrg_ml[(pt * G + g) * 2]);
    float acc = 0.f, L = 0.f;
#pragma unroll
    for (int pt = 0; pt < NPART; ++pt) {
      const float f = exp2f(sm.mrg_ml[(pt * G + g) * 2] - M);   // 0 for a partition without tokens
      float o = 0.f;
#pragma unroll
      for (int q2 = 0; q2 < NPP; ++q2) o += sm.mrg_o[((pt * NPP + q2) * G + g) * D + d];
      acc = fmaf(f, o, acc);
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
    if (lane == 0) mbar_arrive(sm.mws);
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
      const int n = int(c1 - c0 + 1);
      // weights 2^(m_i - M) of every partial slot i and 1 / L per head, one warp per head (lanes
      // share the slots), into the merge area, which this CTA's own merge no longer reads
      float* wts = sm.mrg_o;                             // [n][G]
      float* linv = sm.mrg_o + n * G;                    // [G]
      for (int g = ct >> 5; g < G; g += NCW) {
        const float* ml = a.ws_ml + ((c0 + item) * G + g) * 2;
        float M = -INFINITY;
        for (int i = lane; i < n; i += 32) M = fmaxf(M, __ldcg(ml + int64_t(2) * G * i));
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float L = 0.f;
        for (int i = lane; i < n; i += 32) {
          const float w = exp2f(__ldcg(ml + int64_t(2) * G * i) - M);   // 0 for a slot without tokens
          wts[i * G + g] = w;
          L = fmaf(w, __ldcg(ml + int64_t(2) * G * i + 1), L);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
        if (lane == 0) linv[g] = 1.f / L;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.mcomb);
      if (!mbar_wait(sm.mcomb, itc & 1, sm.abort_flag, a.L.wait_ns)) {
        if (lane == 0) record_error(a.L.err, kErrWaitTimeout | 9);
        *sm.abort_flag = 1;
        return false;
      }
      ++itc;
      // every output element: the weighted sum of its slots, slots in a fixed order (loads unrolled)
      for (int e = ct; e < G * D; e += NCW * 32) {
        const int g = e / D, d = e % D;
        const float* o0 = a.ws_o + ((c0 + item) * G + g) * D + d;
        float acc = 0.f;
#pragma unroll 8
        for (int i = 0; i < n; ++i) acc = fmaf(wts[i * G + g], __ldcg(o0 + int64_t(G) * D * i), acc);
        a.out[(int64_t(sg.bi) * a.n_q_heads + sg.h * G + g) * D + d] = __float2half_rn(acc * linv[g]);
      }
    }
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(sm.mfree);
  ++itm;
  return true;
}

// Producer warp: streams the CTA's chunks into the stage ring (and, with a fused
// append, quantises each item's new token into its page first).
template <int KB, int VB, int D, int G>
__device__ __forceinline__ void producer_role(const DecodeQArgs& a, const Batch& b,
                                              const QDecSmem<KB, VB, D, G>& sm, int64_t x0, int64_t x1) {
  using T = QDec<KB, VB, D, G>;
  constexpr int S = T::S, NB = T::NB;
  const int lane = threadIdx.x & 31;
  const int H = a.L.n_kv_heads;
  const uint64_t pol = l2_evict_first_policy();
  uint32_t it = 0;
  bool ok = true;
  // Page ids of the next 32 chunks, one per lane, loaded together once every 32 chunks: the
  // page-table read (a global load, ~1 us) would otherwise sit in front of every stage's copies.
  int my_page = -1;
  for (int64_t x = x0; x < x1 && ok;) {
    const DecodeSeg sg = decode_find_seg(b, x, x1);
    const SeqDesc sd = b.s[sg.bi];
    for (int k = sg.k0; k < sg.k0 + sg.n; ++k) {
      const int s = it % S;
      if ((it & 31) == 0) {
        const int64_t xl = x0 + it + lane;                  // this lane's chunk of the flat list
        my_page = -1;
        if (xl < x1) {
          const DecodeSeg gl = decode_find_seg(b, xl, x1);
          const SeqDesc dl = b.s[gl.bi];
          const int t0 = dl.lo / a.chunk * a.chunk + gl.k0 * a.chunk;
          my_page = a.L.page_table[int64_t(dl.seq_id) * a.L.max_pages_per_seq + page_slot(t0 / a.L.page_tokens, dl.ring)];
        }
      }
      const int page = __shfl_sync(0xffffffffu, my_page, it & 31);
      if (!mbar_wait(sm.empty0 + 8 * s, ((it / S) & 1) ^ 1, sm.abort_flag, a.L.wait_ns)) {
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
      uint8_t* hb = a.L.head_ptr(a.layer, page, sg.h);
      if (a.k_new != nullptr && tok0 + ntok == sd.a) {
        // fused append: quantise the new token (position len - 1 = page row r + ntok - 1)
        // before the copy that reads it; lane i < NB takes K block i, NB <= i < 2 NB a V block
        const int rn = r + ntok - 1;
        if (lane < 2 * NB) {
          const bool is_v = lane >= NB;
          const int blk = lane % NB;
          const __half* src = (is_v ? a.v_new : a.k_new) + (int64_t(sg.bi) * H + sg.h) * D + 32 * blk;
          float xv[32];
          load_block(src, xv);
          uint8_t* codes = hb + (is_v ? a.L.v_codes_off : 0) + int64_t(rn) * (is_v ? T::V_ROW : T::K_ROW);
          __half* scales =
              reinterpret_cast<__half*>(hb + (is_v ? a.L.v_scales_off : a.L.k_scales_off) + int64_t(rn) * T::S_ROW);
          if ((is_v ? VB : KB) == 8) quant8_block(xv, codes + 32 * blk, scales + blk);
          else quant4_block(xv, codes + 16 * blk, scales + blk);
          // the bulk copy below reads these bytes through the async proxy
          asm volatile("fence.proxy.async.global;" ::: "memory");
        }
        __syncwarp();
      }
      // test hook (cache created with KVQ_TEST_WITHHOLD_ARRIVAL set): CTA 0 never fills its
      // first stage, so its consumers' bounded waits run out and report kErrWaitTimeout
      const bool withhold = a.L.test_withhold && blockIdx.x == 0 && it == 0;
      if (lane == 0 && !withhold) {
        const uint32_t bar = sm.full0 + 8 * s;
        const uint32_t dst = smem_u32(sm.stages + s * T::STAGE);
        mbar_arrive_expect_tx(bar, uint32_t(ncopy * T::TOK_BYTES));
        bulk_g2s(dst, hb + int64_t(r) * T::K_ROW, ncopy * T::K_ROW, bar, pol);
        bulk_g2s(dst + T::OFF_KS, hb + a.L.k_scales_off + int64_t(r) * T::S_ROW, ncopy * T::S_ROW, bar, pol);
        bulk_g2s(dst + T::OFF_VC, hb + a.L.v_codes_off + int64_t(r) * T::V_ROW, ncopy * T::V_ROW, bar, pol);
        bulk_g2s(dst + T::OFF_VS, hb + a.L.v_scales_off + int64_t(r) * T::S_ROW, ncopy * T::S_ROW, bar, pol);
      }
      ++it;
    }
    x += sg.n;
  }
  // no copy may outlive the CTA: wait (bounded) for the last fills to land
  if (lane == 0)
    for (uint32_t j = it > uint32_t(S) ? it - S : 0; j < it; ++j) mbar_wait(sm.full0 + 8 * (j % S), (j / S) & 1, nullptr, a.L.wait_ns);
}

// Score warp: q . k over its partition's tokens, online softmax, p' = p d_v.
template <int KB, int VB, int D, int G>
__device__ __forceinline__ void score_role(const DecodeQArgs& a, const Batch& b, const QDecSmem<KB, VB, D, G>& sm,
                                           int64_t x0, int64_t x1) {
  using T = QDec<KB, VB, D, G>;
  constexpr int S = T::S, W = T::W, NB = T::NB, GW = T::GW, NF = T::NF, LPT = T::LPT, NHG = T::NHG;
  constexpr int KSPAN = 2 * (T::K_ROW / NB);           // code bytes of the lane's two key blocks
  constexpr uint32_t FULL = 0xffffffffu;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int part = warp / NHG, hg = warp % NHG;
  const int tl = lane / LPT, half = lane % LPT;        // lane = tl * LPT + half: blocks 2 half, 2 half + 1
  const int fmap = rs_map<LPT, GW>(half);
  const int xr = kq2_rot<KB, D>(tl);
  const int bswap = KB == 8 ? (xr >> 1) : xr;          // slot sp holds block 2 half + (sp ^ bswap)
  uint32_t it = 0, itm = 0, itw = 0, itc = 0;
  for (int64_t x = x0; x < x1;) {
    const DecodeSeg sg = decode_find_seg(b, x, x1);
    const SeqDesc sd = b.s[sg.bi];
    // ---- query digits in permuted slots: slot j <-> head hg * GW + (j ^ fmap), this lane's two blocks.
    // The warp's GW query rows are staged in shared memory with 16-byte loads, then each lane reads its
    // elements in its own (bank-rotated) word order from there.
    __half* qs = sm.qbuf + warp * GW * D;
    {
      const uint4* src = reinterpret_cast<const uint4*>(a.q + (int64_t(sg.bi) * a.n_q_heads + sg.h * G + hg * GW) * D);
      for (int i = lane; i < GW * D / 8; i += 32) reinterpret_cast<uint4*>(qs)[i] = src[i];
      __syncwarp();
    }
    float amax[GW];
#pragma unroll
    for (int j = 0; j < GW; ++j) {
      const uint4* qr = reinterpret_cast<const uint4*>(qs + (j ^ fmap) * D + 64 * half);
      float mx = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 w4 = qr[c];
        const uint32_t ws[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = h2_to_f2(ws[i]);
          mx = fmax3(mx, fabsf(f.x), fabsf(f.y));
        }
      }
      amax[j] = mx * fabsf(a.scale_log2);
    }
    // per-head max over the token's lanes: the lane at lane ^ o holds this lane's slot-j head in
    // its slot j ^ rs_map(o)
#pragma unroll
    for (int o = 1; o < LPT; o <<= 1) {
      float t[GW];
#pragma unroll
      for (int j = 0; j < GW; ++j) t[j] = __shfl_xor_sync(FULL, amax[j ^ rs_map<LPT, GW>(o)], o);
#pragma unroll
      for (int j = 0; j < GW; ++j) amax[j] = fmaxf(amax[j], t[j]);
    }
    // n = rint(q / s) with s = max|q| / 32512 (|n| <= 32512), as hi = (n + 128) >> 8 and the low byte
    // lo = n mod 256 read as int8, so that n = 256 hi + lo
    uint32_t qh[GW][16], ql[GW][16];
    int qcorr[GW][2];
#pragma unroll
    for (int j = 0; j < GW; ++j) {
      const __half* qr = qs + (j ^ fmap) * D + 64 * half;
      const float mul = amax[j] > 0.f ? a.scale_log2 * (32512.f / amax[j]) : 0.f;
#pragma unroll
      for (int sp = 0; sp < 2; ++sp) {
        const __half* qb = qr + 32 * (sp ^ bswap);
        int corr = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          // the word's 4 elements are consecutive in the row
          const uint2 h4 = *reinterpret_cast<const uint2*>(qb + kq2_elem<KB>(w, 0, xr));
          const float2 f01 = h2_to_f2(h4.x), f23 = h2_to_f2(h4.y);
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
          ql[j][8 * sp + w] = __byte_perm(__byte_perm(n[0], n[1], 0x0040), __byte_perm(n[2], n[3], 0x0040), 0x5410);
          const int h0 = (n[0] + 128) >> 8, h1 = (n[1] + 128) >> 8, h2 = (n[2] + 128) >> 8, h3 = (n[3] + 128) >> 8;
          qh[j][8 * sp + w] = __byte_perm(__byte_perm(h0, h1, 0x0040), __byte_perm(h2, h3, 0x0040), 0x5410);
        }
        qcorr[j][sp] = KB == 4 ? -8 * corr : 0;          // 4-bit codes are read as u = c + 8
      }
    }
    float qsc[NF], m_own[NF], l_own[NF];
#pragma unroll
    for (int j = 0; j < NF; ++j) {                         // slot j < NF ends with head j ^ fmap
      qsc[j] = amax[j] * (1.f / 32512.f);
      m_own[j] = -INFINITY;
      l_own[j] = 0.f;
    }

    for (int k = sg.k0; k < sg.k0 + sg.n; ++k) {
      const int s = it % S, par = it & 1;
      const uint32_t pph = (it >> 1) & 1;
      if (!mbar_wait(sm.full0 + 8 * s, (it / S) & 1, sm.abort_flag, a.L.wait_ns)) {
        if (lane == 0) record_error(a.L.err, kErrWaitTimeout | 2);
        *sm.abort_flag = 1;
        return;
      }
      const uint8_t* st = sm.stages + s * T::STAGE;
      const int tok0 = sd.lo / a.chunk * a.chunk + k * a.chunk;
      const int rv0 = max(0, sd.lo - tok0), rv1 = min(a.chunk, sd.a - tok0);   // valid rows [rv0, rv1)
      const int row0 = part * W;
      const bool masked = rv0 > row0 || rv1 < row0 + W;
      float sc[T::NPASS][NF];
#pragma unroll
      for (int ps = 0; ps < T::NPASS; ++ps) {
        const int row = row0 + ps * T::TPP + tl;
        uint32_t cw[16];
        load_kq2<KB>(st + row * T::K_ROW + half * KSPAN, xr, cw);
        const float2 dk2 = h2_to_f2(*reinterpret_cast<const uint32_t*>(st + T::OFF_KS + row * T::S_ROW + 4 * half));
        const float dks0 = bswap ? dk2.y : dk2.x, dks1 = bswap ? dk2.x : dk2.y;
        int hs[GW][2], ls[GW][2];
#pragma unroll
        for (int j = 0; j < GW; ++j) {
          hs[j][0] = hs[j][1] = 0;
          ls[j][0] = qcorr[j][0];
          ls[j][1] = qcorr[j][1];
        }
#pragma unroll
        for (int w = 0; w < 8; ++w)
#pragma unroll
          for (int sp = 0; sp < 2; ++sp)
#pragma unroll
            for (int j = 0; j < GW; ++j) {
              hs[j][sp] = __dp4a(int(cw[8 * sp + w]), int(qh[j][8 * sp + w]), hs[j][sp]);
              ls[j][sp] = __dp4a(int(cw[8 * sp + w]), int(ql[j][8 * sp + w]), ls[j][sp]);
            }
        float ps_[GW];
#pragma unroll
        for (int j = 0; j < GW; ++j)
          ps_[j] = fmaf(__int2float_rn(hs[j][1] * 256 + ls[j][1]), dks1,
                        __int2float_rn(hs[j][0] * 256 + ls[j][0]) * dks0);
        reduce_scatter_perm<LPT, GW>(ps_);
#pragma unroll
        for (int j = 0; j < NF; ++j) {
          const float v = ps_[j] * qsc[j];
          sc[ps][j] = (!masked || (row >= rv0 && row < rv1)) ? v : -INFINITY;
        }
      }
      // lazy maximum: moved only when a score passes it by 2^8
      bool need = false;
#pragma unroll
      for (int ps = 0; ps < T::NPASS; ++ps)
#pragma unroll
        for (int j = 0; j < NF; ++j) need |= sc[ps][j] > m_own[j] + 8.f;
      const bool any = __any_sync(FULL, need);
      // the value warps must be done with this buffer (two stages back) before it is rewritten
      if (!mbar_wait(sm.free0 + 8 * (part * 2 + par), pph ^ 1, sm.abort_flag, a.L.wait_ns)) {
        if (lane == 0) record_error(a.L.err, kErrWaitTimeout | 3);
        *sm.abort_flag = 1;
        return;
      }
      if (any) {
        float alpha[NF];
#pragma unroll
        for (int j = 0; j < NF; ++j) {
          float mx = sc[0][j];
#pragma unroll
          for (int ps = 1; ps < T::NPASS; ++ps) mx = fmaxf(mx, sc[ps][j]);
#pragma unroll
          for (int o = LPT; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
          const float mn = fmaxf(m_own[j], mx);
          alpha[j] = fast_exp2(m_own[j] - mn);           // 0 while m_own is -inf
          m_own[j] = mn;
          l_own[j] *= alpha[j];
        }
        if (tl == 0) {
#pragma unroll
          for (int j = 0; j < NF; ++j) sm.palpha[(part * 2 + par) * G + hg * GW + (j ^ fmap)] = alpha[j];
        }
      }
      if (lane == 0) sm.pflag[(part * 2 + par) * NHG + hg] = any ? 1 : 0;
      // p, and p' = p d_v of this lane's two value blocks for the group's GW heads
      float* pb = sm.pbuf + (part * 2 + par) * (W * NB * G);
#pragma unroll
      for (int ps = 0; ps < T::NPASS; ++ps) {
        const int t = ps * T::TPP + tl;
        const bool valid = !masked || (row0 + t >= rv0 && row0 + t < rv1);
        float p[NF];
#pragma unroll
        for (int j = 0; j < NF; ++j) {
          const float e2 = fast_exp2(sc[ps][j] - m_own[j]);
          p[j] = valid ? e2 : 0.f;
          l_own[j] += p[j];
        }
        float pa[GW];
#pragma unroll
        for (int g = 0; g < GW; ++g) {
          if constexpr (LPT == 1) pa[g] = p[g];           // this lane holds every head (slot g = head g)
          else pa[g] = __shfl_sync(FULL, p[g % NF], (lane & ~(LPT - 1)) | rs_lane_of<LPT, GW>(g));
        }
        float2 dv2 = h2_to_f2(*reinterpret_cast<const uint32_t*>(st + T::OFF_VS + (row0 + t) * T::S_ROW + 4 * half));
        if (!valid) dv2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
          const float dv = bb ? dv2.y : dv2.x;
          float* dst = pb + (t * NB + 2 * half + bb) * G + hg * GW;
          if constexpr (GW == 4) {
            *reinterpret_cast<float4*>(dst) = make_float4(pa[0] * dv, pa[1] * dv, pa[2] * dv, pa[3] * dv);
          } else if constexpr (GW == 2) {
            *reinterpret_cast<float2*>(dst) = make_float2(pa[0] * dv, pa[1] * dv);
          } else {
            *dst = pa[0] * dv;
          }
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(sm.ready0 + 8 * (part * 2 + par));
        mbar_arrive(sm.empty0 + 8 * s);
      }
      ++it;
    }
    // ---- publish (m, l) of this partition's heads, then merge
    if (!mbar_wait(sm.mfree, (itm & 1) ^ 1, sm.abort_flag, a.L.wait_ns)) {
      if (lane == 0) record_error(a.L.err, kErrWaitTimeout | 5);
      *sm.abort_flag = 1;
      return;
    }
#pragma unroll
    for (int j = 0; j < NF; ++j)
#pragma unroll
      for (int o = LPT; o < 32; o <<= 1) l_own[j] += __shfl_xor_sync(FULL, l_own[j], o);
    if (tl == 0) {
#pragma unroll
      for (int j = 0; j < NF; ++j) {
        const int g = hg * GW + (j ^ fmap);
        sm.mrg_ml[(part * G + g) * 2] = m_own[j];
        sm.mrg_ml[(part * G + g) * 2 + 1] = l_own[j];
      }
    }
    if (!merge_item<KB, VB, D, G>(a, sm, sg, sd, itm, itw, itc)) return;
    x += sg.n;
  }
}

// Value warp: O += p' c over its share of the partition's tokens.
template <int KB, int VB, int D, int G>
__device__ __forceinline__ void value_role(const DecodeQArgs& a, const Batch& b, const QDecSmem<KB, VB, D, G>& sm,
                                           int64_t x0, int64_t x1) {
  using T = QDec<KB, VB, D, G>;
  constexpr int S = T::S, W = T::W, NB = T::NB, GW = T::GW, NHG = T::NHG, E = T::E;
  constexpr uint32_t FULL = 0xffffffffu;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int vw_ = warp - T::NS;
  const int part = vw_ / T::NPP, pw = vw_ % T::NPP;
  const int tv = lane / T::LPV, sl = lane % T::LPV;    // lane = tv * LPV + sl
  uint32_t it = 0, itm = 0, itw = 0, itc = 0;
  for (int64_t x = x0; x < x1;) {
    const DecodeSeg sg = decode_find_seg(b, x, x1);
    const SeqDesc sd = b.s[sg.bi];
    float O[G][E];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int i = 0; i < E; ++i) O[g][i] = 0.f;
    for (int k = sg.k0; k < sg.k0 + sg.n; ++k) {
      const int s = it % S, par = it & 1;
      const uint32_t pph = (it >> 1) & 1;
      if (!mbar_wait(sm.full0 + 8 * s, (it / S) & 1, sm.abort_flag, a.L.wait_ns) ||
          !mbar_wait(sm.ready0 + 8 * (part * 2 + par), pph, sm.abort_flag, a.L.wait_ns)) {
        if (lane == 0) record_error(a.L.err, kErrWaitTimeout | 4);
        *sm.abort_flag = 1;
        return;
      }
      const uint8_t* st = sm.stages + s * T::STAGE;
      const float* pb = sm.pbuf + (part * 2 + par) * (W * NB * G);
#pragma unroll
      for (int h2 = 0; h2 < NHG; ++h2) {
        if (sm.pflag[(part * 2 + par) * NHG + h2]) {       // that head group moved its maximum
#pragma unroll
          for (int g = 0; g < GW; ++g) {
            const float al = sm.palpha[(part * 2 + par) * G + h2 * GW + g];
#pragma unroll
            for (int i = 0; i < E; ++i) O[h2 * GW + g][i] *= al;
          }
        }
      }
      const int t0 = pw * T::WP;                            // this warp's first token in the partition
#pragma unroll 2
      for (int pv = 0; pv < T::NPV; ++pv) {
        const int tloc = t0 + pv * T::TPV + tv;
        const uint8_t* vrow = st + T::OFF_VC + (part * W + tloc) * T::V_ROW + sl * T::BPL;
        uint32_t vw[T::BPL / 4];
        if constexpr (T::BPL == 4) {
          vw[0] = *reinterpret_cast<const uint32_t*>(vrow);
        } else if constexpr (T::BPL == 8) {
          const uint2 u = *reinterpret_cast<const uint2*>(vrow);
          vw[0] = u.x;
          vw[1] = u.y;
        } else {
#pragma unroll
          for (int c = 0; c < T::BPL / 16; ++c) {
            const uint4 u = reinterpret_cast<const uint4*>(vrow)[c];
            vw[4 * c] = u.x; vw[4 * c + 1] = u.y; vw[4 * c + 2] = u.z; vw[4 * c + 3] = u.w;
          }
        }
#pragma unroll
        for (int bl = 0; bl < T::NBL; ++bl) {
          const int vblk = (sl * T::BPL) / T::VBLK + bl;
          const float* pp = pb + (tloc * NB + vblk) * G;
          float pg[G];
          if constexpr (G >= 4) {
#pragma unroll
            for (int c = 0; c < G / 4; ++c) {
              const float4 f = reinterpret_cast<const float4*>(pp)[c];
              pg[4 * c] = f.x; pg[4 * c + 1] = f.y; pg[4 * c + 2] = f.z; pg[4 * c + 3] = f.w;
            }
          } else if constexpr (G == 2) {
            const float2 f = *reinterpret_cast<const float2*>(pp);
            pg[0] = f.x;
            pg[1] = f.y;
          } else {
            pg[0] = *pp;
          }
          constexpr int WPB = (T::BPL / T::NBL) / 4;      // code words of one value block in this lane
#pragma unroll
          for (int wq = 0; wq < WPB; ++wq) {
            const int wi = bl * WPB + wq;
            if constexpr (VB == 4) {
              float f[8];
              cvt_v4_word(vw[wi], f);
#pragma unroll
              for (int g = 0; g < G; ++g)
#pragma unroll
                for (int e = 0; e < 8; ++e) O[g][8 * wi + e] = fmaf(pg[g], f[e], O[g][8 * wi + e]);
            } else {
              float f[4];
              cvt_v8_word(vw[wi], f);
#pragma unroll
              for (int g = 0; g < G; ++g)
#pragma unroll
                for (int e = 0; e < 4; ++e) O[g][4 * wi + e] = fmaf(pg[g], f[e], O[g][4 * wi + e]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(sm.free0 + 8 * (part * 2 + par));
        mbar_arrive(sm.empty0 + 8 * s);
      }
      ++it;
    }
    // ---- publish this warp's O (summed over its token lanes), then merge
    if (!mbar_wait(sm.mfree, (itm & 1) ^ 1, sm.abort_flag, a.L.wait_ns)) {
      if (lane == 0) record_error(a.L.err, kErrWaitTimeout | 5);
      *sm.abort_flag = 1;
      return;
    }
#pragma unroll
    for (int o = T::LPV; o < 32; o <<= 1)
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int i = 0; i < E; ++i) O[g][i] += __shfl_xor_sync(FULL, O[g][i], o);
    if (tv == 0) {
      float* mo = sm.mrg_o + vw_ * G * D;
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int i = 0; i < E; ++i) mo[g * D + v_elem_of<VB, E>(sl, i)] = O[g][i];
    }
    if (!merge_item<KB, VB, D, G>(a, sm, sg, sd, itm, itw, itc)) return;
    x += sg.n;
  }
}

template <int KB, int VB, int D, int G>
__global__ void __launch_bounds__(QDec<KB, VB, D, G>::NT, 1)
    decode_q_kernel(const DecodeQArgs a, const __grid_constant__ Batch b) {
  using T = QDec<KB, VB, D, G>;
  extern __shared__ __align__(128) uint8_t smem[];
  const QDecSmem<KB, VB, D, G> sm(smem);
  if (threadIdx.x == 0) {
    for (int s = 0; s < T::S; ++s) {
      mbar_init(sm.full0 + 8 * s, 1);
      mbar_init(sm.empty0 + 8 * s, T::NCW);
    }
    for (int i = 0; i < 2 * T::NPART; ++i) {
      mbar_init(sm.ready0 + 8 * i, T::NHG);
      mbar_init(sm.free0 + 8 * i, T::NPP);
    }
    mbar_init(sm.mfull, T::NCW);
    mbar_init(sm.mfree, T::NCW);
    mbar_init(sm.mws, T::NCW);
    mbar_init(sm.mlast, 1);
    mbar_init(sm.mcomb, T::NCW);
    *sm.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  const int64_t x0 = int64_t(blockIdx.x) * a.cpc;
  const int64_t x1 = min(a.total_chunks, x0 + a.cpc);
  // register split by warpgroup: the producer group gives registers back first, then the
  // score group (query digits in registers) takes more; the value groups keep theirs
  if (warp >= T::NCW) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(T::REG_P));
    if (warp == T::NCW) producer_role<KB, VB, D, G>(a, b, sm, x0, x1);
    return;                                                 // the group's other 3 warps have no role
  }
  if (warp < T::NS) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(T::REG_S));
    score_role<KB, VB, D, G>(a, b, sm, x0, x1);
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(T::REG_V));
    value_role<KB, VB, D, G>(a, b, sm, x0, x1);
  }
}

}  // namespace kvq
