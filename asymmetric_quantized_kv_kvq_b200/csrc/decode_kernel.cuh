// Split-KV flash-decoding over the quantized paged cache (sm_100a, CUDA cores).
//
// Computes, for each sequence b, KV head h and query head g of its GQA group,
//   o = sum_t p_t v^_t / sum_t p_t,  p_t = 2^(s_t - m),  s_t = (sigma log2 e) q . k^_t
// over cache positions t < len (exact softmax attention read "through the
// flash-attention path", KVSplit page, section "Exemplos de uso e opcoes de
// CLI"), with k^ = d_k * c_k and v^ = d_v * c_v dequantised in registers from
// the stored 8-bit / 4-bit codes (or read as fp16).
//
// Work decomposition ("stream-K" over the flat list of (sequence, KV head,
// chunk) units): CTA c owns chunks [c * cpc, (c+1) * cpc) of that list, so
// every SM streams the same number of bytes whatever the length mix.  A CTA
// writes one partial (O, m, l) per item it touches; an item covered by one CTA
// is normalised and written to `out` directly, the others are merged by the
// log-sum-exp combine kernel.
//
// CTA = 1 producer warp + NW consumer warps, one CTA per SM (persistent):
//  - producer: lane 0 streams each chunk's K codes, K scales, V codes and V
//    scales (four contiguous ranges of one page's head block) into a ring of S
//    shared-memory stages with 1-D TMA bulk copies (cp.async.bulk, L2
//    evict-first) completing on the stage's "full" mbarrier;
//  - consumers: the NW warps form NG = G / GW head groups of NTW warps; a
//    warp holds the state of GW <= 4 query heads (more would not fit its
//    registers) and takes tokens [tw*W, tw*W + W) of each stage, tw being its
//    slot in the group, so with 8 query heads per KV head two warps read every
//    token, each for its 4 heads.
//      QK on quantized keys: integer dot products.  Each lane owns a whole
//      32-element block of every query head of the warp.  The query, pre-scaled by sigma log2 e, is held as two int8
//      digits per element against one fp32 scale per (head, lane slice):
//      q ~= s * (256 hi + lo), |q - s (256 hi + lo)| <= s / 2 with
//      s = max|q| / 32512, i.e. 15-bit precision.  dp4a multiplies the stored
//      int8 codes (4-bit codes unpacked to bytes, offset -8 folded into a
//      per-head correction) by both digit words with exact int32
//      accumulation; the block's scales (s * d_k) are applied once per
//      (token, head, slice).  No code is converted to floating point.
//      QK on fp16 keys: f32x2 FMAs on converted halves.
//      A reduce-scatter across the token's lanes then leaves each lane the
//      full score of its own head(s).
//      Softmax: online, per warp, with lazy rescaling (the running max is only
//      moved when a score exceeds it by more than 2^8).
//      PV: 8 head_dim elements per lane; p' = p * d_v is precomputed per
//      (token, block, head) into a warp-private buffer (stored twice, so two
//      heads' values arrive in one 16-byte load), and the inner loop is one
//      scalar FMA per element and head: scalar FMAs overlap with the byte
//      permutes of the V conversion, f32x2 FMAs do not.
//  - every wait is bounded (2 s); on expiry the kernel records an error code,
//    raises a CTA-wide abort flag, drains its own copies and returns.
#pragma once

#include <cuda_fp16.h>

#include "decode_common.cuh"
#include "kvq_internal.cuh"
#include "sm100_util.cuh"

namespace kvq {

template <int KB, int VB, int D, int G>
struct DecodeTraits {
  static constexpr bool INT_QK = KB != 16;              // dp4a path for quantized keys
  static constexpr int GW = G > 4 ? 4 : G;               // query heads whose state one warp holds
  static constexpr int NG = G / GW;                      // head groups (warps of different groups read the same tokens)
  static constexpr int NW = 8;                           // consumer warps
  static constexpr int NTW = NW / NG;                    // warps that split the tokens of a stage
  static constexpr int NT = (NW + 1) * 32;
  static constexpr int NB = D / 32;
  static constexpr int K_ROW = KB == 16 ? 2 * D : KB == 8 ? D : D / 2;
  static constexpr int V_ROW = VB == 16 ? 2 * D : VB == 8 ? D : D / 2;
  static constexpr int KS_ROW = KB == 16 ? 0 : NB * 2;
  static constexpr int VS_ROW = VB == 16 ? 0 : NB * 2;
  static constexpr int TOK_BYTES = K_ROW + KS_ROW + V_ROW + VS_ROW;
  static constexpr int C = TOK_BYTES <= 320 ? 256 / NG : 64;   // tokens per stage (W = C / NTW per warp)
  static constexpr int W = C / NTW;
  static constexpr int J = INT_QK ? 32 : 16;             // head_dim elements per lane in QK
  static constexpr int LPT = D / J;
  static constexpr int TPS = 32 / LPT;
  static constexpr int NJ = W / TPS;
  static constexpr int GPL = GW > LPT ? GW / LPT : 1;
  static constexpr int REP = GW < LPT ? LPT / GW : 1;
  static constexpr int LPV = D / 8;
  static constexpr int TPV = 32 / LPV;
  static constexpr int NPV = W / TPV;
  static constexpr int NBP = VB == 16 ? 1 : NB;
  static constexpr int OFF_KS = C * K_ROW;
  static constexpr int OFF_VC = OFF_KS + C * KS_ROW;
  static constexpr int OFF_VS = OFF_VC + C * V_ROW;
  static constexpr int STAGE_BYTES = OFF_VS + C * VS_ROW;
  static constexpr int PBUF_BYTES = NW * W * NBP * GW * 8;
  static constexpr int MRG_O_BYTES = NTW * G * D * 4;
  static constexpr int MRG_ML_BYTES = NTW * G * 2 * 4;
  static constexpr int BAR_BYTES = 256;
  static constexpr int FIXED = PBUF_BYTES + MRG_O_BYTES + MRG_ML_BYTES + BAR_BYTES;
  static constexpr int SMEM_LIMIT = 227 * 1024;
  static constexpr int S_FIT = (SMEM_LIMIT - FIXED) / STAGE_BYTES;
  static constexpr int S = S_FIT > 6 ? 6 : S_FIT;
  static constexpr int SMEM = S * STAGE_BYTES + FIXED;
  static_assert(S >= 2, "stage ring does not fit in shared memory");
  static_assert(W % TPS == 0 && W % TPV == 0 && NJ >= 1, "warp tile");
  static_assert(2 * S + 4 <= BAR_BYTES / 8, "barrier area");
  static_assert(STAGE_BYTES % 16 == 0 && OFF_KS % 16 == 0 && OFF_VC % 16 == 0 && OFF_VS % 16 == 0, "alignment");
};

// ---- per-format element maps ----------------------------------------------------
// QK lane `slice` owns 16 elements of the row; element index of its i-th value.
template <int KB, int D>
__device__ __forceinline__ int k_elem(int slice, int i) {
  if (KB == 8) return 16 * slice + i;
  if (KB == 4) return 32 * (slice >> 1) + 8 * (slice & 1) + (i < 8 ? i : i + 8);
  return i < 8 ? 8 * slice + i : D / 2 + 8 * slice + (i - 8);
}

// Integer QK path: element index of digit i (0 .. J-1) of lane `slice`, and the
// lane's code words in the same order (4-bit codes unpacked to one byte each,
// values 0..15, read as non-negative int8 by dp4a).
template <int KB, int J>
__device__ __forceinline__ int kq_elem(int slice, int i) {
  if (KB == 8) return J * slice + i;
  if (J == 32) return 32 * slice + i;          // whole block: low nibbles 0..15, high nibbles 16..31
  return 32 * (slice >> 1) + 8 * (slice & 1) + (i < 8 ? i : i + 8);
}
template <int KB, int J>
__device__ __forceinline__ void load_kcodes(const uint8_t* row, int slice, uint32_t (&cw)[J / 4]) {
  if (KB == 8) {
    const uint4 a = *reinterpret_cast<const uint4*>(row + J * slice);
    cw[0] = a.x; cw[1] = a.y; cw[2] = a.z; cw[3] = a.w;
    if constexpr (J == 32) {
      const uint4 c = *reinterpret_cast<const uint4*>(row + J * slice + 16);
      cw[4] = c.x; cw[5] = c.y; cw[6] = c.z; cw[7] = c.w;
    }
  } else if constexpr (J == 32) {
    const uint4 a = *reinterpret_cast<const uint4*>(row + 16 * slice);
    cw[0] = a.x & 0x0F0F0F0Fu; cw[1] = a.y & 0x0F0F0F0Fu; cw[2] = a.z & 0x0F0F0F0Fu; cw[3] = a.w & 0x0F0F0F0Fu;
    cw[4] = (a.x >> 4) & 0x0F0F0F0Fu; cw[5] = (a.y >> 4) & 0x0F0F0F0Fu;
    cw[6] = (a.z >> 4) & 0x0F0F0F0Fu; cw[7] = (a.w >> 4) & 0x0F0F0F0Fu;
  } else {
    const uint2 a = *reinterpret_cast<const uint2*>(row + 16 * (slice >> 1) + 8 * (slice & 1));
    cw[0] = a.x & 0x0F0F0F0Fu; cw[1] = a.y & 0x0F0F0F0Fu;
    cw[2] = (a.x >> 4) & 0x0F0F0F0Fu; cw[3] = (a.y >> 4) & 0x0F0F0F0Fu;
  }
}

// Load and convert the lane's 16 K values of one row (exact integers or fp16 values).
template <int KB, int D>
__device__ __forceinline__ void load_k16(const uint8_t* row, int slice, float2 (&kf)[8]) {
  if (KB == 8) {
    const uint4 w = *reinterpret_cast<const uint4*>(row + 16 * slice);
    cvt_s8x4(w.x, kf[0], kf[1]);
    cvt_s8x4(w.y, kf[2], kf[3]);
    cvt_s8x4(w.z, kf[4], kf[5]);
    cvt_s8x4(w.w, kf[6], kf[7]);
  } else if (KB == 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(row + 8 * slice);
    cvt_u4x4(w.x & 0x0F0F0F0Fu, kf[0], kf[1]);
    cvt_u4x4(w.y & 0x0F0F0F0Fu, kf[2], kf[3]);
    cvt_u4x4((w.x >> 4) & 0x0F0F0F0Fu, kf[4], kf[5]);
    cvt_u4x4((w.y >> 4) & 0x0F0F0F0Fu, kf[6], kf[7]);
  } else {
    const uint4 a = *reinterpret_cast<const uint4*>(row + 16 * slice);
    const uint4 c = *reinterpret_cast<const uint4*>(row + D + 16 * slice);
    kf[0] = h2_to_f2(a.x); kf[1] = h2_to_f2(a.y); kf[2] = h2_to_f2(a.z); kf[3] = h2_to_f2(a.w);
    kf[4] = h2_to_f2(c.x); kf[5] = h2_to_f2(c.y); kf[6] = h2_to_f2(c.z); kf[7] = h2_to_f2(c.w);
  }
}

// Index of the (token, V block) group of G p' pairs in a warp's buffer: the
// block index is XOR-swizzled by the token so that the p' stores of the tokens
// of a step fall in different banks.
template <int NBP>
__device__ __forceinline__ int pgroup(int t, int blk) {
  return t * NBP + (blk ^ (t & (NBP - 1)));
}

// o += p * v for the two elements of a pair, as two scalar FMAs.
__device__ __forceinline__ void fma_pair(float p, float2 v, float2& o) {
  o.x = fmaf(p, v.x, o.x);
  o.y = fmaf(p, v.y, o.y);
}

// Reduce-scatter of G partial sums over the LPT lanes of one token (lanes
// differing in bits below LPT): afterwards this lane holds the full sums of
// heads g0 .. g0 + GPL - 1 in v[0 .. GPL-1].
template <int G, int LPT>
__device__ __forceinline__ void reduce_scatter(float (&v)[G], int lane) {
  int n = G;
#pragma unroll
  for (int o = LPT / 2; o >= 1; o >>= 1) {
    if (n > 1) {
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < G / 2; ++i) {
        if (i < n / 2) {
          const float send = upper ? v[i] : v[i + n / 2];
          const float keep = upper ? v[i + n / 2] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      n >>= 1;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
  }
}

template <int KB, int VB, int D, int G>
__global__ void __launch_bounds__(DecodeTraits<KB, VB, D, G>::NT, 1)
    decode_split_kernel(const DecodeArgs a, const __grid_constant__ Batch b) {
  using T = DecodeTraits<KB, VB, D, G>;
  constexpr int S = T::S, W = T::W, NW = T::NW, GW = T::GW, NTW = T::NTW;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* stages = smem;
  float2* pbuf = reinterpret_cast<float2*>(smem + S * T::STAGE_BYTES);
  float* mrg_o = reinterpret_cast<float*>(smem + S * T::STAGE_BYTES + T::PBUF_BYTES);
  float* mrg_ml = mrg_o + NTW * G * D;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * T::STAGE_BYTES + T::PBUF_BYTES + T::MRG_O_BYTES +
                                               T::MRG_ML_BYTES);
  // bars[0..S) full, [S..2S) empty, [2S] merge-full, [2S+1] merge-free, then the abort flag
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * S + 2);
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + S);
  const uint32_t mfull = smem_u32(bars + 2 * S), mfree = smem_u32(bars + 2 * S + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = a.L.n_kv_heads;
  const int64_t x0 = int64_t(blockIdx.x) * a.cpc;
  const int64_t x1 = min(a.total_chunks, x0 + a.cpc);

  // the stage ring is not cleared: rows past a sequence's end (never copied, or
  // stale) only reach scores that are replaced by -inf with a select, and the PV
  // loop skips them, so their contents never matter
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, NW);
    }
    mbar_init(mfull, NW);
    mbar_init(mfree, NW);
    *abort_flag = 0;
    fence_mbar_init();
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();

  // ------------------------------------------------------------------ producer
  if (warp == NW) {
    const uint64_t pol = l2_evict_first_policy();
    uint32_t it = 0;
    bool ok = true;
    // page ids of the next 32 chunks, one per lane, loaded together once every 32 chunks (a
    // page-table read in front of every stage would cap the stage rate); lane 0 issues the copies
    int my_page = -1;
    for (int64_t x = x0; x < x1 && ok;) {
      const DecodeSeg sg = decode_find_seg(b, x, x1);
      const SeqDesc sd = b.s[sg.bi];
      for (int k = sg.k0; k < sg.k0 + sg.n; ++k) {
        const int s = it % S;
        if ((it & 31) == 0) {
          const int64_t xl = x0 + it + lane;
          my_page = -1;
          const DecodeSeg gl = xl < x1 ? decode_find_seg(b, xl, x1) : DecodeSeg{0, 0, 0, 0, 0};
          if (gl.n > 0) {                                   // a chunk that holds tokens
            const SeqDesc dl = b.s[gl.bi];
            const int t0 = dl.lo / a.chunk * a.chunk + gl.k0 * a.chunk;
            my_page = a.L.page_table[int64_t(dl.seq_id) * a.L.max_pages_per_seq + page_slot(t0 / a.L.page_tokens, dl.ring)];
          }
        }
        const int page = __shfl_sync(0xffffffffu, my_page, it & 31);
        if (!mbar_wait(empty0 + 8 * s, ((it / S) & 1) ^ 1, abort_flag)) {
          if (lane == 0) record_error(a.L.err, kErrWaitTimeout | 1);
          *abort_flag = 1;
          ok = false;
          break;
        }
        const int tok0 = sd.lo / a.chunk * a.chunk + k * a.chunk;   // chunks start at the window's first chunk
        const int ntok = min(a.chunk, sd.a - tok0);
        const int ncopy = min(a.chunk, (ntok + 15) & ~15);
        if (page < 0 || page >= a.L.n_pages) {
          if (lane == 0) record_error(a.L.err, kErrBadPage);
          *abort_flag = 1;
          ok = false;
          break;
        }
        if (lane == 0) {
          const int r = tok0 % a.L.page_tokens;
          const uint8_t* hb = a.L.head_ptr(a.layer + sd.l, page, sg.h);
          const uint32_t bar = full0 + 8 * s;
          const uint32_t dst = smem_u32(stages + s * T::STAGE_BYTES);
          mbar_arrive_expect_tx(bar, uint32_t(ncopy * T::TOK_BYTES));
          bulk_g2s(dst, hb + int64_t(r) * T::K_ROW, ncopy * T::K_ROW, bar, pol);
          if (T::KS_ROW) bulk_g2s(dst + T::OFF_KS, hb + a.L.k_scales_off + int64_t(r) * T::KS_ROW, ncopy * T::KS_ROW, bar, pol);
          bulk_g2s(dst + T::OFF_VC, hb + a.L.v_codes_off + int64_t(r) * T::V_ROW, ncopy * T::V_ROW, bar, pol);
          if (T::VS_ROW) bulk_g2s(dst + T::OFF_VS, hb + a.L.v_scales_off + int64_t(r) * T::VS_ROW, ncopy * T::VS_ROW, bar, pol);
        }
        ++it;
      }
      x += sg.adv;
    }
    // no copy may outlive the CTA: wait (bounded) for the last fills to land
    if (lane == 0)
      for (uint32_t j = it > uint32_t(S) ? it - S : 0; j < it; ++j) mbar_wait(full0 + 8 * (j % S), (j / S) & 1, nullptr);
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int slice = lane % T::LPT, tis = lane / T::LPT;
  const int vsl = lane % T::LPV, tslot = lane / T::LPV;
  const int hg = warp / NTW, tw = warp % NTW;     // head group, token slot of this warp
  const int gb = hg * GW;                          // first query head of the group
  const int g0 = (slice / T::REP) * T::GPL;
  const int rep = slice % T::REP;
  const int ct = warp * 32 + lane;
  uint32_t it = 0, itm = 0;

  for (int64_t x = x0; x < x1;) {
    const DecodeSeg sg = decode_find_seg(b, x, x1);
    const SeqDesc sd = b.s[sg.bi];
    const int item = sg.bi * H + sg.h;

    // q slice in registers, pre-scaled by sigma * log2(e)
    float2 qp[T::INT_QK ? 1 : GW][8];          // fp16-key path: fp32 pairs
    uint32_t qh[T::INT_QK ? GW : 1][T::J / 4], ql[T::INT_QK ? GW : 1][T::J / 4];   // integer path: digit words
    float qsc[GW];
    int qcorr[GW];
#pragma unroll
    for (int g = 0; g < GW; ++g) {
      const __half* qrow = a.q + (int64_t(sg.bi) * a.n_q_heads + sg.h * G + gb + g) * D;
      if constexpr (T::INT_QK) {
        float qv[T::J];
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < T::J; ++i) {
          qv[i] = __half2float(qrow[kq_elem<KB, T::J>(slice, i)]) * a.scale_log2;
          amax = fmaxf(amax, fabsf(qv[i]));
        }
        const float inv = amax > 0.f ? 32512.f / amax : 0.f;
        qsc[g] = amax * (1.f / 32512.f);
        int corr = 0;
#pragma unroll
        for (int k = 0; k < T::J / 4; ++k) {
          uint32_t hw = 0, lw = 0;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            int n = __float2int_rn(qv[4 * k + e] * inv);
            n = max(-32512, min(32512, n));
            const int lo = ((n + 128) & 255) - 128;
            const int hi = (n - lo) >> 8;
            hw |= uint32_t(hi & 255) << (8 * e);
            lw |= uint32_t(lo & 255) << (8 * e);
            corr += n;
          }
          qh[g][k] = hw;
          ql[g][k] = lw;
        }
        qcorr[g] = KB == 4 ? 8 * corr : 0;
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float e0 = __half2float(qrow[k_elem<KB, D>(slice, 2 * i)]);
          const float e1 = __half2float(qrow[k_elem<KB, D>(slice, 2 * i + 1)]);
          qp[g][i] = make_float2(e0 * a.scale_log2, e1 * a.scale_log2);
        }
        qsc[g] = 1.f;
        qcorr[g] = 0;
      }
    }
    float2 O[GW][4];
#pragma unroll
    for (int g = 0; g < GW; ++g)
#pragma unroll
      for (int k = 0; k < 4; ++k) O[g][k] = make_float2(0.f, 0.f);
    float m_own[T::GPL], l_own[T::GPL];
#pragma unroll
    for (int gi = 0; gi < T::GPL; ++gi) {
      m_own[gi] = -INFINITY;
      l_own[gi] = 0.f;
    }

    for (int k = sg.k0; k < sg.k0 + sg.n; ++k) {
      const int s = it % S;
      if (!mbar_wait(full0 + 8 * s, (it / S) & 1, abort_flag)) {
        if (lane == 0) record_error(a.L.err, kErrWaitTimeout | 2);
        *abort_flag = 1;
        return;
      }
      ++it;
      // valid rows of the stage: [rv0, rv1) (rv0 > 0 only in the first chunk of a rotating window);
      // of this warp's W rows: [lo_w, nv_w)
      const int tok0 = sd.lo / a.chunk * a.chunk + k * a.chunk;
      const int rv0 = max(0, sd.lo - tok0), rv1 = min(a.chunk, sd.a - tok0);
      const int nv_w = min(W, max(0, rv1 - tw * W));
      const int lo_w = max(0, rv0 - tw * W);
      if (nv_w > lo_w) {
        const uint8_t* st = stages + s * T::STAGE_BYTES;
        const int row0 = tw * W;
        // ---- scores
        float sc[T::NJ][T::GPL];
#pragma unroll
        for (int j = 0; j < T::NJ; ++j) {
          const int t = j * T::TPS + tis;
          const int row = row0 + t;
          float part[GW];
          if constexpr (T::INT_QK) {
            uint32_t cw[T::J / 4];
            load_kcodes<KB, T::J>(st + row * T::K_ROW, slice, cw);
            const float dk = __half2float(
                reinterpret_cast<const __half*>(st + T::OFF_KS + row * T::KS_ROW)[(slice * T::J) >> 5]);
            int hs[GW], ls[GW];
#pragma unroll
            for (int g = 0; g < GW; ++g) hs[g] = ls[g] = 0;
#pragma unroll
            for (int q = 0; q < T::J / 4; ++q) {        // 2 GW independent dp4a chains, interleaved
#pragma unroll
              for (int g = 0; g < GW; ++g) {
                hs[g] = __dp4a(int(cw[q]), int(qh[g][q]), hs[g]);
                ls[g] = __dp4a(int(cw[q]), int(ql[g][q]), ls[g]);
              }
            }
#pragma unroll
            for (int g = 0; g < GW; ++g) part[g] = __int2float_rn(hs[g] * 256 + ls[g] - qcorr[g]) * (qsc[g] * dk);
          } else {
            float2 kf[8];
            load_k16<KB, D>(st + row * T::K_ROW, slice, kf);
#pragma unroll
            for (int g = 0; g < GW; ++g) {
              float2 acc = make_float2(0.f, 0.f);
#pragma unroll
              for (int i = 0; i < 8; ++i) acc = ffma2(qp[g][i], kf[i], acc);
              part[g] = acc.x + acc.y;
            }
          }
          reduce_scatter<GW, T::LPT>(part, lane);
#pragma unroll
          for (int gi = 0; gi < T::GPL; ++gi) sc[j][gi] = (t >= lo_w && t < nv_w) ? part[gi] : -INFINITY;
        }
        // ---- online softmax, max moved lazily: a vote decides whether any score
        //      exceeds the running max by more than 2^8; only then is the exact
        //      tile max reduced across lanes and O, l rescaled
        bool need = false;
#pragma unroll
        for (int gi = 0; gi < T::GPL; ++gi)
#pragma unroll
          for (int j = 0; j < T::NJ; ++j) need |= sc[j][gi] > m_own[gi] + 8.f;
        if (__any_sync(0xffffffffu, need)) {
          float alpha[T::GPL];
#pragma unroll
          for (int gi = 0; gi < T::GPL; ++gi) {
            float mx = sc[0][gi];
#pragma unroll
            for (int j = 1; j < T::NJ; ++j) mx = fmaxf(mx, sc[j][gi]);
#pragma unroll
            for (int o = T::LPT; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float mn = fmaxf(m_own[gi], mx);
            alpha[gi] = exp2f(m_own[gi] - mn);
            m_own[gi] = mn;
            l_own[gi] *= alpha[gi];
          }
#pragma unroll
          for (int g = 0; g < GW; ++g) {
            const float al = __shfl_sync(0xffffffffu, alpha[g % T::GPL], (g / T::GPL) * T::REP);
#pragma unroll
            for (int k = 0; k < 4; ++k) O[g][k] = fmul2(O[g][k], make_float2(al, al));
          }
        }
        // ---- p and p' = p * d_v (duplicated pairs) into the warp's buffer
        float2* pw = pbuf + size_t(warp) * W * T::NBP * GW;
#pragma unroll
        for (int j = 0; j < T::NJ; ++j) {
          const int t = j * T::TPS + tis;
          const int row = row0 + t;
          float dv[T::NBP];
          if constexpr (VB != 16) {
            const __half* vs = reinterpret_cast<const __half*>(st + T::OFF_VS + row * T::VS_ROW);
            if constexpr (T::NBP == 4) {
              const uint2 w = *reinterpret_cast<const uint2*>(vs);
              const float2 a0 = h2_to_f2(w.x), a1 = h2_to_f2(w.y);
              dv[0] = a0.x; dv[1] = a0.y; dv[2] = a1.x; dv[3] = a1.y;
            } else {
              const float2 a0 = h2_to_f2(*reinterpret_cast<const uint32_t*>(vs));
              dv[0] = a0.x; dv[1] = a0.y;
            }
          }
#pragma unroll
          for (int gi = 0; gi < T::GPL; ++gi) {
            const float p = exp2f(sc[j][gi] - m_own[gi]);   // 0 for masked tokens
            l_own[gi] += p;
            if (VB == 16) {
              if (rep == 0) pw[t * GW + g0 + gi] = make_float2(p, p);
            } else {
#pragma unroll
              for (int bb = 0; bb < T::NBP; bb += T::REP) {
                const int blk = bb + rep;
                if (blk < T::NBP) {
                  const float pv = p * dv[blk < T::NBP ? blk : 0];
                  pw[pgroup<T::NBP>(t, blk) * GW + g0 + gi] = make_float2(pv, pv);
                }
              }
            }
          }
        }
        __syncwarp();
        // ---- O += p' v
#pragma unroll 4
        for (int j2 = 0; j2 < T::NPV; ++j2) {
          const int t = j2 * T::TPV + tslot;
          if (t >= lo_w && t < nv_w) {
            float2 vf[4];
            load_v8<VB>(st + T::OFF_VC + (row0 + t) * T::V_ROW, vsl, vf);
            const float2* pp = pw + pgroup<T::NBP>(t, v_block<VB>(vsl)) * GW;
#pragma unroll
            for (int g = 0; g < GW; g += 2) {
              float2 p0, p1;
              (void)p1;
              if constexpr (GW >= 2) {
                const float4 pq = *reinterpret_cast<const float4*>(pp + g);
                p0 = make_float2(pq.x, pq.y);
                p1 = make_float2(pq.z, pq.w);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) fma_pair(p0.x, vf[kk], O[g][kk]);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) fma_pair(p1.x, vf[kk], O[g + 1][kk]);
              } else {
                p0 = pp[g];
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) fma_pair(p0.x, vf[kk], O[g][kk]);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * s);
    }

    // ---- merge token slots inside the warp, then the warps of the CTA
#pragma unroll
    for (int o = T::LPV; o < 32; o <<= 1)
#pragma unroll
      for (int g = 0; g < GW; ++g)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          O[g][k].x += __shfl_xor_sync(0xffffffffu, O[g][k].x, o);
          O[g][k].y += __shfl_xor_sync(0xffffffffu, O[g][k].y, o);
        }
#pragma unroll
    for (int gi = 0; gi < T::GPL; ++gi)
#pragma unroll
      for (int o = T::LPT; o < 32; o <<= 1) l_own[gi] += __shfl_xor_sync(0xffffffffu, l_own[gi], o);

    if (!mbar_wait(mfree, (itm & 1) ^ 1, abort_flag)) {
      if (lane == 0) record_error(a.L.err, kErrWaitTimeout | 3);
      *abort_flag = 1;
      return;
    }
    if (tslot == 0) {
#pragma unroll
      for (int g = 0; g < GW; ++g)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          mrg_o[(tw * G + gb + g) * D + v_elem<VB>(vsl, 2 * k)] = O[g][k].x;
          mrg_o[(tw * G + gb + g) * D + v_elem<VB>(vsl, 2 * k + 1)] = O[g][k].y;
        }
    }
    if (tis == 0 && rep == 0) {
#pragma unroll
      for (int gi = 0; gi < T::GPL; ++gi) {
        mrg_ml[(tw * G + gb + g0 + gi) * 2] = m_own[gi];
        mrg_ml[(tw * G + gb + g0 + gi) * 2 + 1] = l_own[gi];
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(mfull);
    if (!mbar_wait(mfull, itm & 1, abort_flag)) {
      if (lane == 0) record_error(a.L.err, kErrWaitTimeout | 4);
      *abort_flag = 1;
      return;
    }
    const int nch = sd.c;
    const int64_t off = int64_t(sd.b) + int64_t(sg.h) * nch;
    const bool single = (off / a.cpc) == ((off + nch - 1) / a.cpc);
    for (int e = ct; e < G * D; e += NW * 32) {
      const int g = e / D, d = e % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NTW; ++w) M = fmaxf(M, mrg_ml[(w * G + g) * 2]);
      float acc = 0.f, L = 0.f;
#pragma unroll
      for (int w = 0; w < NTW; ++w) {
        const float f = exp2f(mrg_ml[(w * G + g) * 2] - M);
        acc += f * mrg_o[(w * G + g) * D + d];
        L += f * mrg_ml[(w * G + g) * 2 + 1];
      }
      if (single) {
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
    __syncwarp();
    if (lane == 0) mbar_arrive(mfree);
    ++itm;
    x += sg.adv;
  }
}

}  // namespace kvq
