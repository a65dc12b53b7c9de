// Split-KV decode on the tensor cores (sm_100a tcgen05) for 8-bit keys
// (K8V4, K8V8) at head_dim 128.
//
// Same result as the CUDA-core kernel: for each sequence, KV head and query
// head g of its GQA group, o = sum_t p_t v^_t / sum_t p_t with
// p_t = 2^(s_t - m), s_t = (sigma log2 e) q . k^_t over positions t < len
// (exact softmax attention on the dequantised cache, KVSplit page, section
// "Exemplos de uso e opcoes de CLI"; k^ = d_k c_k, v^ = d_v c_v from the
// 32-element blocks of the page's memory table), with the same stream-K split
// and the same partial-result format, so the log-sum-exp combine is shared.
//
// Per 128-token tile of one (sequence, KV head):
//  scores  S[t, n] = sum over one 32-element block of c_k[t, i] * qd[n, i]
//          on tcgen05.mma kind::i8 (s8 x s8 -> exact s32 in TMEM): A = the
//          stored key codes exactly as they sit in HBM (one 3-D TMA tensor
//          load per tile, 128-byte swizzle, no conversion), B = the query as
//          two int8 digits per element, q ~= s (256 hi + lo) with
//          s = max|q| / 32512 per head (15-bit precision), rows 0..G-1 = hi,
//          G..2G-1 = lo.  One MMA per block b puts S_b in its own 16 TMEM
//          columns, because d_k varies per (token, block):
//            s_t,g = s_g sum_b d_k[t, b] (256 S_b[t, g] + S_b[t, G + g]).
//  softmax one thread per token row reads its S row (tcgen05.ld), forms the
//          G scores, and the 128 threads vote (bar.red.or) whether any score
//          exceeds the running max by more than 2^8; only then is the exact
//          tile max exchanged and O rescaled in TMEM.  p = 2^(s - m) is
//          written as fp16 into the B operand of the PV product.
//  values  one thread per token row converts its stored V codes to
//          v^ = fp16(d_v (c - 8)) (4-bit) or fp16(d_v c) (8-bit): each code
//          becomes the exact fp16 1024 + u by a byte permute, 1024 + bias is
//          subtracted exactly and one fp16 multiply by d_v rounds once.  The
//          tile is written MN-major (head_dim contiguous) with 128-byte swizzle.
//  PV      O^T[d, g] += sum_t v^[t, d] p[t, g] on tcgen05.mma kind::f16 with
//          fp32 accumulation in TMEM (M = head_dim 128, N = 16 >= G, K = 16
//          tokens per instruction, 8 per tile).
//
// CTA = 11 warps, one CTA per SM (persistent): warp 0 streams each chunk
// (TMA tensor load of the key codes, bulk copies of key scales, value codes
// and value scales) into a ring of stages; warp 1 owns TMEM and issues the
// score MMAs, warp 10 the PV MMAs; warps 2-5 (one per TMEM lane quadrant) run the softmax and the
// per-item epilogue; warps 6-9 convert V.  TMEM: two 64-column score tiles
// and two 16-column O accumulators (by item parity).  Every wait is bounded
// (2 s): on expiry the kernel records an error code, raises a CTA-wide abort
// flag, and every role leaves through the same teardown (MMAs drained, TMEM
// freed); decisions inside the softmax warpgroup are made uniform with
// bar.red so no thread waits at a named barrier for one that has left.
#include <cuda.h>
#include <cuda_fp16.h>

#include <mutex>
#include <vector>

#include "decode_common.cuh"
#include "kvq_internal.cuh"
#include "sm100_util.cuh"
#include "tcgen05_util.cuh"
#include "tma_host.h"

namespace kvq {

namespace {

constexpr int kTT = 128;       // tokens per tile: M of the score product
constexpr int kD = 128;        // head_dim
constexpr int kNB = kD / 32;   // quantisation blocks per row

template <int VB>
struct TcTraits {
  static constexpr int K_BYTES = kTT * kD;               // key codes, [128 rows][128 B] swizzled
  static constexpr int KS_ROW = kNB * 2;
  static constexpr int V_ROW = VB == 8 ? kD : kD / 2;
  static constexpr int VS_ROW = kNB * 2;
  static constexpr int OFF_KS = K_BYTES;
  static constexpr int OFF_VC = OFF_KS + kTT * KS_ROW;
  static constexpr int OFF_VS = OFF_VC + kTT * V_ROW;
  static constexpr int STAGE = (OFF_VS + kTT * VS_ROW + 1023) / 1024 * 1024;
  static constexpr int VH_BYTES = kTT * kD * 2;          // v^ tile, two [128 tokens][128 B] column blocks
  static constexpr int P_BYTES = 2 * 16 * 128;           // p, two [16 rows][64 tokens] K-major blocks
  static constexpr int QD_BYTES = 16 * 128;              // query digits [16 rows][128 B]
  static constexpr int OFF_VH = 0;
  static constexpr int OFF_P = OFF_VH + 2 * VH_BYTES;
  static constexpr int OFF_QD = OFF_P + 2 * P_BYTES;
  static constexpr int OFF_STAGE = OFF_QD + 2 * QD_BYTES;
  static constexpr int MISC = 1024;
  static constexpr int SMEM_LIMIT = 227 * 1024;
  static constexpr int NS_FIT = (SMEM_LIMIT - 1024 - OFF_STAGE - MISC) / STAGE;
  static constexpr int NS = NS_FIT > 6 ? 6 : NS_FIT;
  static constexpr int OFF_MISC = OFF_STAGE + NS * STAGE;
  static constexpr int SMEM = OFF_MISC + MISC + 1024;    // + slack for the 1024-B alignment
  static constexpr int NT = 352;
  static constexpr uint32_t TMEM_COLS = 256;
  static constexpr uint32_t S_COL = 0;                   // two 64-column score tiles
  static constexpr uint32_t O_COL = 128;                 // two 16-column O^T accumulators
  static_assert(NS >= 2, "stage ring");
  static_assert(OFF_STAGE % 1024 == 0 && STAGE % 1024 == 0, "swizzle atoms");
  static_assert(SMEM <= SMEM_LIMIT, "shared memory");
};

// Byte offset of element (row n, byte column c) in a K-major 128-byte-swizzled
// operand of 128-byte rows (8-row atoms of 1024 B).
__device__ __forceinline__ int sw128_kmajor(int n, int c) {
  return (n >> 3) * 1024 + (n & 7) * 128 + ((((c >> 4) ^ (n & 7))) << 4) + (c & 15);
}

// Exact int -> float for |x| < 2^22 (the block sums are below 32 * 127 * 128).
__device__ __forceinline__ float small_int_to_float(uint32_t x) {
  return __uint_as_float(x + 0x4B400000u) - 12582912.0f;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Four fp16 pairs {1024 + byte} for the four bytes of w (each byte < 256).
__device__ __forceinline__ void bytes_to_h1024(uint32_t w, uint32_t& p01, uint32_t& p23) {
  p01 = __byte_perm(w, 0x64646464u, 0x4140);
  p23 = __byte_perm(w, 0x64646464u, 0x4342);
}
// fp16(d (h - bias)) for a pair h = 1024 + u: the subtraction is exact, the multiply rounds once.
__device__ __forceinline__ uint32_t dequant_pair(uint32_t h, __half2 bias, __half2 d) {
  __half2 x = *reinterpret_cast<const __half2*>(&h);
  x = __hmul2(__hsub2(x, bias), d);
  return *reinterpret_cast<const uint32_t*>(&x);
}

// One token row of v^ into the MN-major swizzled tile: logical 16-B chunk q
// (elements 8q .. 8q+7) of row t lives at column block q / 8, K group t / 8.
__device__ __forceinline__ void store_vh_chunk(uint8_t* vh, int row, int q, uint4 v) {
  const int r8 = row & 7;
  *reinterpret_cast<uint4*>(vh + (q >> 3) * (kTT * 128) + (row >> 3) * 1024 + r8 * 128 + (((q & 7) ^ r8) << 4)) = v;
}

template <int VB>
__device__ __forceinline__ void dequant_v_row(const uint8_t* st, int row, bool valid, uint8_t* vh) {
  using T = TcTraits<VB>;
  if (!valid) {
#pragma unroll
    for (int q = 0; q < kD / 8; ++q) store_vh_chunk(vh, row, q, make_uint4(0, 0, 0, 0));
    return;
  }
  const uint2 sw = *reinterpret_cast<const uint2*>(st + T::OFF_VS + row * T::VS_ROW);
  const uint8_t* vc = st + T::OFF_VC + row * T::V_ROW;
  if constexpr (VB == 4) {
    const __half2 bias = __half2half2(__ushort_as_half(0x6408));   // 1032
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int bb = (i + (row >> 1)) & 3;                          // rotated: conflict-free loads / stores
      const uint4 w = *reinterpret_cast<const uint4*>(vc + 16 * bb);
      const uint32_t dbits = __byte_perm(((bb >> 1) ? sw.y : sw.x), 0, (bb & 1) ? 0x3232 : 0x1010);
      const __half2 d = *reinterpret_cast<const __half2*>(&dbits);
      const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
      uint32_t o[4][4];                                             // [output chunk][pair]
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        // bytes 4k..4k+3: low nibbles are elements 4k..4k+3, high nibbles 16+4k..16+4k+3
        uint32_t a01, a23, b01, b23;
        bytes_to_h1024(wv[k] & 0x0F0F0F0Fu, a01, a23);
        bytes_to_h1024((wv[k] >> 4) & 0x0F0F0F0Fu, b01, b23);
        o[k >> 1][2 * (k & 1)] = dequant_pair(a01, bias, d);
        o[k >> 1][2 * (k & 1) + 1] = dequant_pair(a23, bias, d);
        o[2 + (k >> 1)][2 * (k & 1)] = dequant_pair(b01, bias, d);
        o[2 + (k >> 1)][2 * (k & 1) + 1] = dequant_pair(b23, bias, d);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) store_vh_chunk(vh, row, 4 * bb + c, make_uint4(o[c][0], o[c][1], o[c][2], o[c][3]));
    }
  } else {
    const __half2 bias = __half2half2(__ushort_as_half(0x6480));   // 1152 = 1024 + 128
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ci = (i + row) & 7;                                 // 16 elements, block ci / 2
      const uint4 w = *reinterpret_cast<const uint4*>(vc + 16 * ci);
      const int bb = ci >> 1;
      const uint32_t dbits = __byte_perm(((bb >> 1) ? sw.y : sw.x), 0, (bb & 1) ? 0x3232 : 0x1010);
      const __half2 d = *reinterpret_cast<const __half2*>(&dbits);
      const uint32_t wv[4] = {w.x ^ 0x80808080u, w.y ^ 0x80808080u, w.z ^ 0x80808080u, w.w ^ 0x80808080u};
      uint32_t o[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint32_t a01, a23;
        bytes_to_h1024(wv[k], a01, a23);
        o[2 * k] = dequant_pair(a01, bias, d);
        o[2 * k + 1] = dequant_pair(a23, bias, d);
      }
      store_vh_chunk(vh, row, 2 * ci, make_uint4(o[0], o[1], o[2], o[3]));
      store_vh_chunk(vh, row, 2 * ci + 1, make_uint4(o[4], o[5], o[6], o[7]));
    }
  }
}

template <int VB, int G>
__global__ void __launch_bounds__(352, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const DecodeArgs a, const __grid_constant__ Batch b) {
  using T = TcTraits<VB>;
  constexpr int NS = T::NS;
  constexpr int B_FULL = 0, B_EMPTY = NS, B_SFULL = 2 * NS, B_SFREE = 2 * NS + 2, B_PFULL = 2 * NS + 4,
                B_VFULL = 2 * NS + 6, B_PVDONE = 2 * NS + 8, B_QFULL = 2 * NS + 10, B_OFULL = 2 * NS + 12,
                B_OFREE = 2 * NS + 14, B_DONE = 2 * NS + 16, B_DONE2 = 2 * NS + 17, NBAR = 2 * NS + 18;
  static_assert(NBAR * 8 <= 256, "barrier area");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  uint8_t* misc = smem + T::OFF_MISC;
  const uint32_t bar0 = base + T::OFF_MISC;
  auto bar = [&](int i) { return bar0 + 8u * uint32_t(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 256);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 260);
  float* red_q = reinterpret_cast<float*>(misc + 512);   // [4 quadrants][8 heads] each
  float* red_m = red_q + 32;
  float* red_l = red_q + 64;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = a.L.n_kv_heads;
  const int64_t x0 = int64_t(blockIdx.x) * a.cpc;
  const int64_t x1 = min(a.total_chunks, x0 + a.cpc);

  // p and query-digit buffers start zeroed: their rows for heads >= G are never written
  for (int i = threadIdx.x; i < (2 * T::P_BYTES + 2 * T::QD_BYTES) / 16; i += T::NT)
    reinterpret_cast<uint4*>(smem + T::OFF_P)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    for (int i = 0; i < NBAR; ++i) {
      uint32_t cnt = 1;
      if (i >= B_EMPTY && i < B_EMPTY + NS) cnt = 9;           // score MMAs + 4 softmax + 4 value warps
      else if ((i >= B_SFREE && i < B_SFREE + 2) || (i >= B_PFULL && i < B_PFULL + 4) ||
               (i >= B_QFULL && i < B_QFULL + 2) || (i >= B_OFREE && i < B_OFREE + 2))
        cnt = 4;                                               // one arrival per warp of a warpgroup
      mbar_init(bar(i), cnt);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), T::TMEM_COLS);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = l2_evict_first_policy();
      uint32_t it = 0;
      bool ok = true;
      for (int64_t x = x0; x < x1 && ok;) {
        const DecodeSeg sg = decode_find_seg(b, x, x1);
        const SeqDesc sd = b.s[sg.bi];
        for (int k = sg.k0; k < sg.k0 + sg.n; ++k) {
          const int s = it % NS;
          if (!mbar_wait(bar(B_EMPTY + s), ((it / NS) & 1) ^ 1, abort_flag)) {
            record_error(a.L.err, kErrWaitTimeout | 0x21);
            *abort_flag = 1;
            ok = false;
            break;
          }
          const int tok0 = k * a.chunk;
          const int ntok = min(a.chunk, sd.a - tok0);
          const int ncopy = min(a.chunk, (ntok + 15) & ~15);
          const int page = a.L.page_table[int64_t(sd.seq_id) * a.L.max_pages_per_seq + tok0 / a.L.page_tokens];
          if (page < 0 || page >= a.L.n_pages) {
            record_error(a.L.err, kErrBadPage);
            *abort_flag = 1;
            ok = false;
            break;
          }
          const int r = tok0 % a.L.page_tokens;
          const uint8_t* hb = a.L.head_ptr(a.layer, page, sg.h);
          const uint32_t full = bar(B_FULL + s);
          const uint32_t st = base + T::OFF_STAGE + s * T::STAGE;
          mbar_arrive_expect_tx(full, uint32_t(T::K_BYTES + ncopy * (T::KS_ROW + T::V_ROW + T::VS_ROW)));
          // key codes: rows r .. r+127 of this head block (rows past the page read as zero)
          tma_load_3d(st, &tm_k, 0, r, (a.layer * a.L.n_pages + page) * H + sg.h, full);
          bulk_g2s(st + T::OFF_KS, hb + a.L.k_scales_off + int64_t(r) * T::KS_ROW, ncopy * T::KS_ROW, full, pol);
          bulk_g2s(st + T::OFF_VC, hb + a.L.v_codes_off + int64_t(r) * T::V_ROW, ncopy * T::V_ROW, full, pol);
          bulk_g2s(st + T::OFF_VS, hb + a.L.v_scales_off + int64_t(r) * T::VS_ROW, ncopy * T::VS_ROW, full, pol);
          ++it;
        }
        x += sg.adv;
      }
      // no copy may outlive the CTA
      for (uint32_t j = it > uint32_t(NS) ? it - NS : 0; j < it; ++j) mbar_wait(bar(B_FULL + j % NS), (j / NS) & 1, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ score MMAs
    // A tcgen05.mma keeps its issuing thread ~100 cycles whatever its shape (measured; two issuing warps
    // double the rate), so score MMAs (this warp) and PV MMAs (warp 10) come from different warps.
    if (lane == 0) {
      constexpr uint32_t ID_QK = idesc_s8_s32(kTT, 16);
      uint32_t it = 0, j = 0, ii = 0;
      bool ok = true;
      for (int64_t x = x0; x < x1 && ok; ++ii) {
        const DecodeSeg sg = decode_find_seg(b, x, x1);
        const uint64_t qd0 = sdesc_k_sw128(base + T::OFF_QD + (ii & 1) * T::QD_BYTES);
        ok = mbar_wait(bar(B_QFULL + (ii & 1)), (ii >> 1) & 1, abort_flag);
        for (int k = 0; k < sg.n && ok; ++k, ++it, ++j) {
          const int s = it % NS;
          ok = mbar_wait(bar(B_FULL + s), (it / NS) & 1, abort_flag) &&
               mbar_wait(bar(B_SFREE + (j & 1)), ((j >> 1) & 1) ^ 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint64_t kd0 = sdesc_k_sw128(base + T::OFF_STAGE + s * T::STAGE);
          const uint32_t s_tm = tmem + T::S_COL + 64 * (j & 1);
#pragma unroll
          for (int bb = 0; bb < kNB; ++bb) umma_i8(s_tm + 16 * bb, kd0 + 2 * bb, qd0 + 2 * bb, ID_QK, 0u);
          umma_commit(bar(B_SFULL + (j & 1)));
          umma_commit(bar(B_EMPTY + s));
        }
        x += sg.adv;
      }
      if (!ok) {
        record_error(a.L.err, kErrWaitTimeout | 0x22);
        *abort_flag = 1;
      }
      // every MMA issued by this thread has completed before TMEM is released
      umma_commit(bar(B_DONE));
      mbar_wait(bar(B_DONE), 0, nullptr);
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------ PV MMAs
    if (lane == 0) {
      constexpr uint32_t ID_PV = idesc_f16_f32_amn(kD, 16);
      uint32_t j = 0, ii = 0;
      bool ok = true;
      for (int64_t x = x0; x < x1 && ok; ++ii) {
        const DecodeSeg sg = decode_find_seg(b, x, x1);
        const uint32_t ip = ii & 1;
        const uint32_t o_tm = tmem + T::O_COL + 16 * ip;
        ok = mbar_wait(bar(B_OFREE + ip), ((ii >> 1) & 1) ^ 1, abort_flag);
        for (int k = 0; k < sg.n && ok; ++k, ++j) {
          ok = mbar_wait(bar(B_PFULL + (j & 1)), (j >> 1) & 1, abort_flag) &&
               mbar_wait(bar(B_VFULL + (j & 1)), (j >> 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint64_t vd0 = sdesc_mn_sw128(base + T::OFF_VH + (j & 1) * T::VH_BYTES, kTT * 128, 1024);
          const uint64_t pd0 = sdesc_k_sw128(base + T::OFF_P + (j & 1) * T::P_BYTES);
#pragma unroll
          for (int kk = 0; kk < kTT / 16; ++kk)
            umma_f16(o_tm, vd0 + kk * (2048 >> 4), pd0 + (((kk >> 2) * 2048 + (kk & 3) * 32) >> 4), ID_PV,
                     (k == 0 && kk == 0) ? 0u : 1u);
          umma_commit(bar(B_PVDONE + (j & 1)));
        }
        if (ok) umma_commit(bar(B_OFULL + ip));
        x += sg.adv;
      }
      if (!ok) {
        record_error(a.L.err, kErrWaitTimeout | 0x25);
        *abort_flag = 1;
      }
      umma_commit(bar(B_DONE2));
      mbar_wait(bar(B_DONE2), 0, nullptr);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ softmax + epilogue (warps 2..5)
    const int quad = warp & 3;
    const int row = quad * 32 + lane;                 // token row of a tile; head_dim row of O
    const uint32_t lane_addr = tmem + (uint32_t(quad * 32) << 16);
    constexpr int BAR_CHECK = 1, BAR_VOTE = 2, BAR_MAX = 3, BAR_QAMAX = 4, BAR_L = 5, BAR_QDONE = 6;
    float m[G], l[G], qsc[G], qsc_next[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      m[g] = -INFINITY;
      l[g] = 0.f;
    }
    // query digits of one item into buffer `buf`; the scale per head comes back in `sc`
    auto write_q = [&](const DecodeSeg& sg, uint32_t buf, float (&sc)[G]) {
      const __half* qb = a.q + (int64_t(sg.bi) * a.n_q_heads + int64_t(sg.h) * G) * kD;
      float qv[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        qv[g] = __half2float(qb[g * kD + row]) * a.scale_log2;
        const float mx = warp_max(fabsf(qv[g]));
        if (lane == 0) red_q[quad * 8 + g] = mx;
      }
      named_barrier(BAR_QAMAX, 128);
      uint8_t* qd = smem + T::OFF_QD + buf * T::QD_BYTES;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float amax = fmaxf(fmaxf(red_q[g], red_q[8 + g]), fmaxf(red_q[16 + g], red_q[24 + g]));
        sc[g] = amax * (1.f / 32512.f);
        const float inv = amax > 0.f ? 32512.f / amax : 0.f;
        int n = __float2int_rn(qv[g] * inv);
        n = max(-32512, min(32512, n));
        const int lo = ((n + 128) & 255) - 128;
        const int hi = (n - lo) >> 8;
        qd[sw128_kmajor(g, row)] = uint8_t(hi & 255);
        qd[sw128_kmajor(G + g, row)] = uint8_t(lo & 255);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_QFULL + buf));
      named_barrier(BAR_QDONE, 128);                  // red_q is reused by the next call
    };

    uint32_t it = 0, j = 0, ii = 0;
    bool wok = true;                                   // waits since the last uniform check
    int64_t x = x0;
    DecodeSeg sg{0, 0, 0, 0};
    if (x < x1) {
      sg = decode_find_seg(b, x, x1);
      write_q(sg, 0, qsc);
    }
    while (x < x1) {
      const int64_t nx = x + sg.adv;
      DecodeSeg nsg{0, 0, 0, 0};
      if (nx < x1) {
        // the next item's digits go to the buffer of the item before this one, whose
        // score MMAs have all completed (every one of its tiles was read here)
        nsg = decode_find_seg(b, nx, x1);
        write_q(nsg, (ii + 1) & 1, qsc_next);
      }
      const SeqDesc sd = b.s[sg.bi];
      const uint32_t ip = ii & 1;
      bool ok = true;
      for (int k = 0; k < sg.n; ++k, ++it, ++j) {
        const int s = it % NS;
        bool w = __all_sync(0xffffffffu, mbar_wait(bar(B_SFULL + (j & 1)), (j >> 1) & 1, abort_flag));
        w = w && __all_sync(0xffffffffu, mbar_wait(bar(B_FULL + s), (it / NS) & 1, abort_flag));
        const uint8_t* st = smem + T::OFF_STAGE + s * T::STAGE;
        const uint2 kw = *reinterpret_cast<const uint2*>(st + T::OFF_KS + row * T::KS_ROW);
        const float2 dk01 = h2_to_f2(kw.x), dk23 = h2_to_f2(kw.y);
        const float dk[4] = {dk01.x, dk01.y, dk23.x, dk23.y};
        float acc[G];
#pragma unroll
        for (int g = 0; g < G; ++g) acc[g] = 0.f;
        if (w) {
          // two blocks (32 columns) at a time: s_g += d_k[b] (256 S_b[g] + S_b[G + g])
          tc_fence_after();
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t sr[32];
            tmem_ld32(lane_addr + T::S_COL + 64 * (j & 1) + 32 * half, sr);
            tmem_wait_ld();
#pragma unroll
            for (int bi = 0; bi < 2; ++bi)
#pragma unroll
              for (int g = 0; g < G; ++g) {
                const float fh = small_int_to_float(sr[16 * bi + g]);
                const float fl = small_int_to_float(sr[16 * bi + G + g]);
                acc[g] = fmaf(dk[2 * half + bi], fmaf(fh, 256.f, fl), acc[g]);
              }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(B_SFREE + (j & 1)));
          mbar_arrive(bar(B_EMPTY + s));
        }
        if (!bar_red_and(BAR_CHECK, 128, w && wok)) {
          ok = false;
          break;
        }
        wok = true;
        const int tok0 = (sg.k0 + k) * a.chunk;
        const bool valid = row < min(a.chunk, sd.a - tok0);
        float sc[G];
        bool need = false;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          sc[g] = valid ? acc[g] * qsc[g] : -INFINITY;
          need |= sc[g] > m[g] + 8.f;
        }
        if (bar_red_or(BAR_VOTE, 128, need)) {
          // some score moved past the running max by more than 2^8: exact tile max, rescale
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float mx = warp_max(sc[g]);
            if (lane == 0) red_m[quad * 8 + g] = mx;
          }
          named_barrier(BAR_MAX, 128);
          float alpha[G];
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float tmax = fmaxf(fmaxf(red_m[g], red_m[8 + g]), fmaxf(red_m[16 + g], red_m[24 + g]));
            const float mn = fmaxf(m[g], tmax);
            alpha[g] = exp2f(m[g] - mn);
            m[g] = mn;
            l[g] *= alpha[g];
          }
          if (k > 0) {
            // O holds this item's earlier tiles: rescale once PV of the previous tile is done
            const bool w2 = __all_sync(0xffffffffu, mbar_wait(bar(B_PVDONE + ((j - 1) & 1)), ((j - 1) >> 1) & 1, abort_flag));
            if (w2) {
              tc_fence_after();
              uint32_t o[16];
              tmem_ld16(lane_addr + T::O_COL + 16 * ip, o);
              tmem_wait_ld();
#pragma unroll
              for (int g = 0; g < G; ++g) o[g] = __float_as_uint(__uint_as_float(o[g]) * alpha[g]);
              tmem_st16(lane_addr + T::O_COL + 16 * ip, o);
              tmem_wait_st();
            }
            wok = wok && w2;
          }
        }
        float p[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          p[g] = exp2f(sc[g] - m[g]);                 // 0 for rows past the end
          l[g] += p[g];
        }
        // the p buffer of this parity was last read by PV two tiles back
        if (j >= 2) wok = wok && __all_sync(0xffffffffu, mbar_wait(bar(B_PVDONE + (j & 1)), ((j >> 1) & 1) ^ 1, abort_flag));
        uint8_t* pb = smem + T::OFF_P + (j & 1) * T::P_BYTES + (row >> 6) * 2048;
#pragma unroll
        for (int g = 0; g < G; ++g)
          *reinterpret_cast<__half*>(pb + sw128_kmajor(g, 2 * (row & 63))) = __float2half_rn(p[g]);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_PFULL + (j & 1)));
      }
      if (!ok) break;
      // ---- item epilogue: O^T row `row` (head_dim index) for every head
      bool w = __all_sync(0xffffffffu, mbar_wait(bar(B_OFULL + ip), (ii >> 1) & 1, abort_flag));
      uint32_t o[16];
      if (w) {
        tc_fence_after();
        tmem_ld16(lane_addr + T::O_COL + 16 * ip, o);
        tmem_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_OFREE + ip));
      if (!bar_red_and(BAR_CHECK, 128, w && wok)) break;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float v = warp_sum(l[g]);
        if (lane == 0) red_l[quad * 8 + g] = v;
      }
      named_barrier(BAR_L, 128);
      const int item = sg.bi * H + sg.h;
      const int nch = sd.c;
      const int64_t off = int64_t(sd.b) + int64_t(sg.h) * nch;
      const bool single = (off / a.cpc) == ((off + nch - 1) / a.cpc);
      const int64_t slot = int64_t(blockIdx.x) + item;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float L = red_l[g] + red_l[8 + g] + red_l[16 + g] + red_l[24 + g];
        const float ov = __uint_as_float(o[g]);
        if (single) {
          a.out[(int64_t(sg.bi) * a.n_q_heads + sg.h * G + g) * kD + row] = __float2half_rn(ov / L);
        } else {
          a.ws_o[(slot * G + g) * kD + row] = ov;
          if (row == 0) {
            a.ws_ml[(slot * G + g) * 2] = m[g];
            a.ws_ml[(slot * G + g) * 2 + 1] = L;
          }
        }
        m[g] = -INFINITY;
        l[g] = 0.f;
        qsc[g] = qsc_next[g];
      }
      x = nx;
      sg = nsg;
      ++ii;
    }
    if (x < x1) {
      record_error(a.L.err, kErrWaitTimeout | 0x23);
      *abort_flag = 1;
    }
  } else {
    // ------------------------------------------------------------ V conversion (warps 6..9)
    const int row = (warp & 3) * 32 + lane;
    uint32_t it = 0, j = 0;
    bool ok = true;
    for (int64_t x = x0; x < x1 && ok;) {
      const DecodeSeg sg = decode_find_seg(b, x, x1);
      const SeqDesc sd = b.s[sg.bi];
      for (int k = 0; k < sg.n; ++k, ++it, ++j) {
        const int s = it % NS;
        bool w = mbar_wait(bar(B_FULL + s), (it / NS) & 1, abort_flag);
        // the v^ buffer of this parity was last read by PV two tiles back
        if (w && j >= 2) w = mbar_wait(bar(B_PVDONE + (j & 1)), ((j >> 1) & 1) ^ 1, abort_flag);
        ok = __all_sync(0xffffffffu, w);
        if (!ok) break;
        const int tok0 = (sg.k0 + k) * a.chunk;
        const bool valid = row < min(a.chunk, sd.a - tok0);
        dequant_v_row<VB>(smem + T::OFF_STAGE + s * T::STAGE, row, valid, smem + T::OFF_VH + (j & 1) * T::VH_BYTES);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(B_VFULL + (j & 1)));
          mbar_arrive(bar(B_EMPTY + s));
        }
      }
      x += sg.adv;
    }
    if (!ok) {
      if (lane == 0) record_error(a.L.err, kErrWaitTimeout | 0x24);
      *abort_flag = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, T::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host
struct MapEntry {
  const void* pool;
  int64_t head_block;
  int n_blocks, page_tokens;
  CUtensorMap map;
};

// Key-code tensor map of a cache: [head blocks][page_tokens rows][128 B], box
// [1][128][128 B], 128-byte swizzle.  Encoded once per pool.
bool key_map(const Layout& L, CUtensorMap* out) {
  static std::mutex mu;
  static std::vector<MapEntry> maps;
  const int64_t nhb = int64_t(L.n_layers) * L.n_pages * L.n_kv_heads;
  std::lock_guard<std::mutex> lock(mu);
  for (const MapEntry& e : maps)
    if (e.pool == L.pool && e.head_block == L.head_block && e.n_blocks == nhb && e.page_tokens == L.page_tokens) {
      *out = e.map;
      return true;
    }
  MapEntry e{L.pool, L.head_block, int(nhb), L.page_tokens, {}};
  const cuuint64_t dims[3] = {cuuint64_t(kD), cuuint64_t(L.page_tokens), cuuint64_t(nhb)};
  const cuuint64_t strides[2] = {cuuint64_t(kD), cuuint64_t(L.head_block)};
  const cuuint32_t box[3] = {cuuint32_t(kD), cuuint32_t(kTT), 1};
  if (!make_tensor_map(&e.map, CU_TENSOR_MAP_DATA_TYPE_UINT8, L.pool, 3, dims, strides, box)) return false;
  if (maps.size() >= 16) maps.erase(maps.begin());
  maps.push_back(e);
  *out = e.map;
  return true;
}

template <int VB, int G>
cudaError_t launch_tc(const CUtensorMap& tm, const DecodeArgs& a, const Batch& b, int n_cta, cudaStream_t s) {
  using T = TcTraits<VB>;
  static bool configured = false;
  if (!configured) {
    const cudaError_t e =
        cudaFuncSetAttribute(decode_tc_kernel<VB, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, T::SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  decode_tc_kernel<VB, G><<<n_cta, T::NT, T::SMEM, s>>>(tm, a, b);
  return cudaGetLastError();
}

}  // namespace

bool decode_tc_supported(const Layout& L, int G) {
  return L.decode_tc && L.k_bits == 8 && (L.v_bits == 4 || L.v_bits == 8) && L.head_dim == kD &&
         (G == 1 || G == 2 || G == 4 || G == 8) &&
         int64_t(L.n_layers) * L.n_pages * L.n_kv_heads < (int64_t(1) << 31);
}

int decode_tc_tile_tokens() { return kTT; }

cudaError_t launch_decode_tc(const Layout& L, int layer, const Batch& b, const DecodePlan& plan, int n_q_heads,
                             const void* q, void* out, float scale_log2, void* ws, cudaStream_t s) {
  const int G = n_q_heads / L.n_kv_heads;
  CUtensorMap tm;
  if (!key_map(L, &tm)) return cudaErrorInvalidValue;
  DecodeArgs a;
  a.L = L;
  a.layer = layer;
  a.n_q_heads = n_q_heads;
  a.q = static_cast<const __half*>(q);
  a.out = static_cast<__half*>(out);
  const int64_t slots = int64_t(plan.max_ctas) + plan.n_items;
  a.ws_o = static_cast<float*>(ws);
  a.ws_ml = a.ws_o + slots * G * kD;
  a.scale_log2 = scale_log2;
  a.total_chunks = plan.total_chunks;
  a.cpc = plan.chunks_per_cta;
  a.chunk = plan.chunk_tokens;
#define KVQ_TC(VB_, G_) \
  if (L.v_bits == VB_ && G == G_) return launch_tc<VB_, G_>(tm, a, b, plan.n_cta, s);
  KVQ_TC(4, 1) KVQ_TC(4, 2) KVQ_TC(4, 4) KVQ_TC(4, 8)
  KVQ_TC(8, 1) KVQ_TC(8, 2) KVQ_TC(8, 4) KVQ_TC(8, 8)
#undef KVQ_TC
  return cudaErrorInvalidValue;
}

}  // namespace kvq
